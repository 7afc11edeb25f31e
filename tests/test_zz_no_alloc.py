"""The no-allocation entry point (needs a B200).

grape_layer_sqnorms_static computes the per-sample squared projected norms of one
layer with only the library's static device scratch.  It serves callers that must
not allocate device memory: code running under a framework whose caching allocator
already holds the GPU's memory (a side cudaMalloc can fail or fragment that pool),
and latency-critical code that cannot pay for cudaMalloc / cudaFree, which may
synchronise the device.

Its result is checked two ways, on two calls in a row each time: against the fp64
oracle's per-sample projected norms of the same inputs, squared, and against what a
grape_step on a one-layer context computes (there the per-sample norm is the square
root of exactly this quantity).

This file is collected last, so a failure here comes after every other test has run;
it passes on its own in a fresh process as well as after the rest of the suite.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

import oracle.grape_oracle as O  # noqa: E402
import workloads as W  # noqa: E402
from harness import rel_fro, to_device  # noqa: E402
from random_gradient_projection_b200 import GrapeStep, grape  # noqa: E402

TOL = 2e-2   # the bf16 tensor-core tolerance of the parity tests

CASES = {
    # one 1024 x 1024 layer, r = 128 (the 128-wide projection tile), T a multiple of 64
    "mlp_r128": (W.scaled(W.get("mlp4x1024"), n_layers=1, B=8, T=128), 1),
    # r = 256 (the 256-wide projection tile) and T = 197, off the 64-row TMA box
    "r256_T197": (W.Workload("static_r256", ((1024, 256),), r=256, B=4, T=197, dtype="bf16",
                             C=1.0, sigma=1.0, steps=2), 1),
    # a context with a projection-refresh period: the entry point takes the key s // K
    "refresh2": (W.scaled(W.get("mlp4x1024"), n_layers=1, B=4, T=64, refresh=2), 2),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_static_sqnorms_match_oracle_and_grape_step_on_two_calls(case):
    w, K = CASES[case]
    d_in, d_out = w.layers[0]
    g = GrapeStep.for_workload(w, path=grape.GRAPE_PATH_TC)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    out = torch.full((w.B,), -1.0, device="cuda")
    h = O.Hyper.of(w)
    for s in (2, 3):   # two calls in a row: different steps, different inputs
        x = W.make_step_inputs(w, s)
        A, G = to_device(x.A[0], "bf16"), to_device(x.Gout[0], "bf16")
        g.step([A], [G], Wd, s)
        grape.grape_layer_sqnorms_static(A, G, d_in, d_out, w.r, w.B, w.T, w.seed, 0, s // K, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)) and np.all(got > 0)
        ref = O.sample_norms([x.as_f64(x.A[0])], [x.as_f64(x.Gout[0])], s, h, [d_in]) ** 2
        ctx = g.norms().astype(np.float64) ** 2   # one layer: n_i^2 is its squared norm
        e_orc, e_ctx = rel_fro(got, ref), rel_fro(got, ctx)
        print(f"{case} step {s}: vs oracle {e_orc:.2e}, vs grape_step {e_ctx:.2e}")
        assert e_orc <= TOL and e_ctx <= TOL
    g.close()


def test_static_sqnorms_reject_problems_beyond_the_scratch():
    A = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(grape.GrapeError) as e:
        # AP alone would need 64 * 4096 * 256 * 2 bytes = 128 MiB
        grape.grape_layer_sqnorms_static(A, A, 4096, 4096, 256, 64, 4096, 0, 0, 0, A)
    assert e.value.code == grape.GRAPE_EINVAL
    assert "static scratch" in str(e.value)
