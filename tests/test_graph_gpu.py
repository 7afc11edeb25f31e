"""CUDA-graph replay of grape_step (grape_set_graph) through the C ABI (needs a B200).

A replay must compute exactly what the ordinary launches compute: the same P (its key
rewritten per step), the same noise and Adam step, on every pointer set.  Each test runs
the same steps twice, once with graphs and once without, and compares W, m and v bitwise,
and the graph run is also checked against the fp64 oracle.
"""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W
from harness import compare, snapshot, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeStep, grape  # noqa: E402

SIMT, TC = grape.GRAPE_PATH_SIMT, grape.GRAPE_PATH_TC


def _inputs(w, n_sets):
    sets = []
    for k in range(n_sets):
        x = W.make_step_inputs(w, k, threads=8)
        sets.append(([to_device(a, w.dtype) for a in x.A], [to_device(a, w.dtype) for a in x.Gout]))
    return sets


def _run(w, path, steps, graph, sets, stream=None, setup=None):
    g = GrapeStep.for_workload(w, path=path)
    if setup:
        setup(g)
    g.set_graph(graph)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    counts = []
    for s in range(steps):
        A, G = sets[s % len(sets)]
        c0 = g.launch_count()
        g.step(A, G, Ws, s, stream)
        counts.append(g.launch_count() - c0)
    torch.cuda.synchronize()
    out = {"W": [x.cpu().numpy() for x in Ws], "m": [g.m(l) for l in range(w.n_layers)],
           "v": [g.v(l) for l in range(w.n_layers)], "norms": g.norms(), "counts": counts}
    g.close()
    return out


CASES = {
    "tc_mlp2": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=64), TC, None),
    "tc_mlp2_refresh3": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=64, refresh=3), TC, None),
    "tc_ghost": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=64), TC,
                 lambda g: g.set_norm_method(grape.GRAPE_NORM_GHOST)),
    # the stored aggregation: the replayed node is the fused aggregation + noise + Adam
    "tc_mlp2_stored": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=64), TC,
                       lambda g: g.set_aggregation(grape.GRAPE_AGG_STORE)),
    "simt_tiny": (W.get("tiny_f32"), SIMT, None),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_graph_replay_is_bitwise_the_ordinary_step(case):
    w, path, setup = CASES[case]
    sets = _inputs(w, 2)
    steps = 6                      # each pointer set: captured at first sight, then replayed
    eager = _run(w, path, steps, False, sets, setup=setup)
    graph = _run(w, path, steps, True, sets, setup=setup)
    for l in range(w.n_layers):
        assert np.array_equal(eager["W"][l], graph["W"][l]), l
        assert np.array_equal(eager["m"][l], graph["m"][l]) and np.array_equal(eager["v"][l], graph["v"][l])
    assert np.array_equal(eager["norms"], graph["norms"])
    # every step, captured or replayed, launches the kernels of an ordinary step with P
    # generated
    full = max(eager["counts"])
    assert all(c == full for c in graph["counts"])


@pytest.mark.parametrize("size", ["reduced", "bench"])
def test_graph_on_a_side_stream_matches_oracle(size):
    """Two persistent input buffers, refilled with each step's inputs: the pointers repeat
    (steps 0-1 captured, 2-5 replayed) while the contents follow the oracle.
    ``bench`` is the benchmarked workload at full size (4 x 1024^2, B = 64, T = 128) in the
    launch configuration bench.py times: CUDA-graph replay."""
    w = W.get("mlp4x1024") if size == "bench" else W.scaled(W.get("mlp4x1024"), n_layers=2, B=4)
    steps = 6
    bufs = _inputs(w, 2)
    side = torch.cuda.Stream()
    g = GrapeStep.for_workload(w, path=TC)
    g.set_graph(True)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    trace = []
    for s in range(steps):
        x = W.make_step_inputs(w, s, threads=8)
        A, G = bufs[s % 2]
        for d, a in zip(A, x.A):
            d.copy_(to_device(a, w.dtype))
        for d, a in zip(G, x.Gout):
            d.copy_(to_device(a, w.dtype))
        torch.cuda.synchronize()
        g.step(A, G, Ws, s, side)
        side.synchronize()
        trace.append(snapshot(g, w.n_layers))
    lib = {"trace": trace, "W": [x.cpu().numpy() for x in Ws]}
    g.close()
    res = O.run(w, steps)
    worst = compare(w, lib, {"trace": res["trace"], "state": res["state"]}, 2e-2, steps)
    print("graph replay vs oracle", {k: f"{v:.2e}" for k, v in worst.items()})


def test_graph_survives_norm_method_switch_and_disable():
    w = W.scaled(W.get("mlp4x1024"), n_layers=1, B=2, T=32)
    sets = _inputs(w, 1)
    g = GrapeStep.for_workload(w, path=TC)
    g.set_graph(True)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    A, G = sets[0]
    for s in range(3):
        g.step(A, G, Ws, s)
    g.set_norm_method(grape.GRAPE_NORM_GHOST)   # drops the captured graph
    for s in range(3, 6):
        g.step(A, G, Ws, s)
    g.set_graph(False)
    g.step(A, G, Ws, 6)
    torch.cuda.synchronize()
    ref = GrapeStep.for_workload(w, path=TC)
    Wr = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    for s in range(7):
        if s == 3:
            ref.set_norm_method(grape.GRAPE_NORM_GHOST)
        ref.step(A, G, Wr, s)
    torch.cuda.synchronize()
    assert np.array_equal(Ws[0].cpu().numpy(), Wr[0].cpu().numpy())
    g.close()
    ref.close()
