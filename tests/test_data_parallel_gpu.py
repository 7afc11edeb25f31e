"""Data parallelism through the library itself (needs a B200).

Two ranks, each a process with its own context on the same GPU, run dp_step
(random_gradient_projection_b200/data_parallel.py): grape_accumulate over the rank's
shard of the batch, one all-reduce of the device buffer that holds every S_l, then
grape_apply with the global batch.  The ranks' kernels never wait on each other: they
meet only in the all-reduce, between steps, which gloo does on the host (the buffer is
copied out, summed and copied back; with NCCL, one process per GPU, it is summed in
place).

Stitched together (norms and clip factors of rank 0's samples, then rank 1's), the
ranks' intermediates must match the fp64 oracle's step on the whole batch, and the two
replicas must end with the same weights, bit for bit.  Shards of equal and of unequal
size (batch_total passed to dp_step).
"""
import os
import socket
import tempfile
from datetime import timedelta

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

import workloads as W  # noqa: E402
from harness import compare, run_oracle, to_device  # noqa: E402

STEPS = 2


def _workload(B):
    return W.Workload("dp_gpu", ((256, 512), (512, 256)), r=128, B=B, T=40, dtype="bf16", C=1.0,
                      sigma=0.8, steps=STEPS)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, B, shards, out_dir):
    try:
        _run_rank(rank, world, port, B, shards, out_dir)
    except BaseException:
        import traceback
        with open(os.path.join(out_dir, f"rank{rank}.err"), "w") as f:
            f.write(traceback.format_exc())
        raise


def _run_rank(rank, world, port, B, shards, out_dir):
    import torch.distributed as dist
    from random_gradient_projection_b200 import GrapeStep, grape
    from random_gradient_projection_b200.data_parallel import dp_step
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    gloo_all_reduce = dist.all_reduce

    def all_reduce_via_host(t, op=dist.ReduceOp.SUM, group=None, async_op=False):
        h = t.cpu()
        gloo_all_reduce(h, op=op, group=group)
        t.copy_(h)

    dist.all_reduce = all_reduce_via_host   # dp_step looks it up at call time
    try:
        torch.cuda.set_device(0)
        w = _workload(B)
        off, sh = sum(shards[:rank]), shards[rank]
        g = GrapeStep.for_workload(w.replace(B=sh), path=grape.GRAPE_PATH_TC)
        Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
        out = {}
        for s in range(STEPS):
            # this rank's samples of the whole batch (each sample has its own streams)
            x = W.make_step_inputs(w, s, samples=range(off, off + sh))
            A = [to_device(a, w.dtype) for a in x.A]
            G = [to_device(a, w.dtype) for a in x.Gout]
            dp_step(g, A, G, Wd, s, batch_total=B)
            torch.cuda.synchronize()
            out[f"norms{s}"], out[f"clip{s}"] = g.norms(), g.clip()
            for l in range(w.n_layers):
                for k, f in (("S", g.S), ("m", g.m), ("v", g.v), ("dR", g.dR)):
                    out[f"{k}{s}_{l}"] = f(l)
        for l, x in enumerate(Wd):
            out[f"W{l}"] = x.cpu().numpy()
        g.close()
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), **out)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shards", [(3, 3), (4, 2)], ids=["even", "uneven"])
def test_dp_step_on_two_ranks_matches_oracle_on_the_whole_batch(shards):
    import torch.multiprocessing as mp
    B = sum(shards)
    w = _workload(B)
    with tempfile.TemporaryDirectory() as d:
        try:
            mp.start_processes(_rank, args=(2, _free_port(), B, shards, d), nprocs=2, join=True,
                               start_method="spawn")
        except Exception:
            for k in range(2):   # the first rank to fail is the one to read
                e = os.path.join(d, f"rank{k}.err")
                if os.path.exists(e):
                    print(f"---- rank {k}\n" + open(e).read())
            raise
        r = [dict(np.load(os.path.join(d, f"rank{k}.npz"))) for k in range(2)]
    for l in range(w.n_layers):
        assert np.array_equal(r[0][f"W{l}"], r[1][f"W{l}"]), "the replicas diverged"
    trace = []
    for s in range(STEPS):
        trace.append({
            "norms": np.concatenate([r[0][f"norms{s}"], r[1][f"norms{s}"]]),
            "clip": np.concatenate([r[0][f"clip{s}"], r[1][f"clip{s}"]]),
            **{k: [r[0][f"{k}{s}_{l}"] for l in range(w.n_layers)] for k in ("S", "m", "v", "dR")},
        })
        for k in ("S", "m", "v", "dR"):   # every rank holds the reduced S and the same state
            for l in range(w.n_layers):
                assert np.array_equal(r[0][f"{k}{s}_{l}"], r[1][f"{k}{s}_{l}"]), (k, s, l)
    lib = {"trace": trace, "W": [r[0][f"W{l}"] for l in range(w.n_layers)]}
    worst = compare(w, lib, run_oracle(w, STEPS), 2e-2, STEPS)
    print(shards, {k: f"{v:.2e}" for k, v in worst.items()})
