"""Data-parallel orchestration on two gloo ranks (CPU, no GPU).

dp_step (random_gradient_projection_b200/data_parallel.py) runs, on every rank,
accumulate -> one all-reduce of all S_l (back to back) -> apply(batch_total = B * world).  Here each
rank drives a stand-in context that computes its shard with the fp64 oracle, so the
test checks the orchestration itself: which tensors are reduced, in which order, and
the global batch used for the average.  Two ranks of 3 samples each must reproduce the
single-process oracle step on all 6 samples, and the two replicas must agree exactly.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.grape_oracle as O
import workloads as W


def _workload():
    return W.Workload("dp", ((24, 16), (16, 12)), r=8, B=6, T=5, dtype="f32", C=0.9,
                      sigma=0.7, steps=2)


class OracleShard:
    """Implements the methods dp_step calls, for the samples `rows` of the batch."""

    def __init__(self, w, rows, W0):
        self.w, self.rows = w, list(rows)
        self.layers = list(w.layers)
        self.B = len(self.rows)
        self.h = O.Hyper.of(w)
        self.state = O.State.init(W0, w.r)
        self.S = None

    def accumulate(self, A, Gout, step, stream=None):
        Ps = [O.projection_matrix(self.h.seed, l, step, di, self.h.r)
              for l, (di, _) in enumerate(self.layers)]
        R = O.projected_per_sample(A, Gout, Ps, range(self.B))
        norms = [np.sqrt(sum(np.sum(R[i][l] ** 2) for l in range(len(Ps)))) for i in range(self.B)]
        c = [O.clip_factor(n, self.h.C) for n in norms]
        self.P = Ps
        # like the library: every S_l a view into one flat buffer, in layer order
        parts = [sum(c[i] * R[i][l] for i in range(self.B)) for l in range(len(Ps))]
        self.S_flat = torch.from_numpy(np.concatenate([p.reshape(-1) for p in parts]))
        self.S, at = [], 0
        for p_ in parts:
            self.S.append(self.S_flat[at:at + p_.size].view(p_.shape))
            at += p_.size

    def S_tensor(self, l):
        return self.S[l]

    def S_all_tensor(self):
        return self.S_flat

    def apply(self, Wt, step, batch_total, stream=None):
        t = step + 1
        for l, (di, do) in enumerate(self.layers):
            xi = O.noise_matrix(self.h.seed, l, step, self.h.r, do)
            g = (self.S[l].numpy() + self.h.sigma * self.h.C * xi) / batch_total
            self.state.m[l], self.state.v[l], d = O.adam(self.state.m[l], self.state.v[l], g, t,
                                                         self.h.beta1, self.h.beta2, self.h.eps)
            Wt[l] -= torch.from_numpy(self.h.lr * (self.P[l] @ d))


class PerLayerShard(OracleShard):
    """The same shard without the flat S buffer: dp_step reduces S_l layer by layer."""

    def __getattribute__(self, name):
        if name == "S_all_tensor":
            raise AttributeError(name)
        return super().__getattribute__(name)


def _rank(rank, world, port, out, shards=None, per_layer=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from random_gradient_projection_b200.data_parallel import dp_step
    w = _workload()
    sizes = shards or [w.B // world] * world
    start = sum(sizes[:rank])
    rows = range(start, start + sizes[rank])
    W0 = W.make_weights(w)
    g = (PerLayerShard if per_layer else OracleShard)(w, rows, W0)
    Wt = [torch.from_numpy(x.astype(np.float64)) for x in W0]
    for s in range(w.steps):
        x = W.make_step_inputs(w, s, samples=list(rows))
        A = [x.as_f64(a) for a in x.A]
        G = [x.as_f64(gg) for gg in x.Gout]
        dp_step(g, A, G, Wt, s, batch_total=sum(sizes) if shards else None)
    out[rank] = [t.numpy().copy() for t in Wt]
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_dp_step_equals_full_batch_oracle():
    world = 2
    port = 29500 + os.getpid() % 1000
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    w = _workload()
    ref = O.run(w, w.steps)["state"]
    for l in range(w.n_layers):
        assert np.array_equal(out[0][l], out[1][l])          # replicas identical
        assert np.allclose(out[0][l], ref.W[l], rtol=0, atol=1e-13), l


@pytest.mark.parametrize("per_layer", [False, True], ids=["one_allreduce", "per_layer"])
def test_three_uneven_ranks_equal_full_batch_oracle(per_layer):
    """Shards of 3, 2 and 1 samples with batch_total = 6, reduced either as one flat
    buffer or layer by layer: every replica equals the single-process oracle step."""
    world, shards = 3, [3, 2, 1]
    port = 30500 + os.getpid() % 1000 + (7 if per_layer else 0)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out, shards, per_layer), nprocs=world,
                       start_method="spawn", join=True)
    w = _workload()
    ref = O.run(w, w.steps)["state"]
    for l in range(w.n_layers):
        for r in range(1, world):
            assert np.array_equal(out[0][l], out[r][l])
        assert np.allclose(out[0][l], ref.W[l], rtol=0, atol=1e-13), l
