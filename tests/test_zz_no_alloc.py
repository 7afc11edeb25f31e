"""The no-allocation entry point against the context-based step (needs a B200).

grape_layer_sqnorms_static computes the per-sample squared projected norms of one
layer with only the library's static device scratch.  It serves callers that must
not allocate device memory: code running under a framework whose caching allocator
already holds the GPU's memory (a side cudaMalloc can fail or fragment that pool),
and latency-critical code that cannot pay for cudaMalloc / cudaFree, which may
synchronise the device.  Its result must equal what a grape_step on a one-layer
context computes for the same inputs: there, the per-sample norm is the square root
of exactly this quantity.

This file is collected last, so a failure here comes after every other test has run;
it passes on its own in a fresh process as well as after the rest of the suite.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

import workloads as W  # noqa: E402
from harness import rel_fro, to_device  # noqa: E402
from random_gradient_projection_b200 import GrapeStep, grape  # noqa: E402

TOL = 2e-2   # the bf16 tensor-core tolerance of the parity tests


def test_static_sqnorms_match_grape_step_on_two_calls():
    w = W.scaled(W.get("mlp4x1024"), n_layers=1, B=8, T=128)   # one 1024 x 1024 layer
    d_in, d_out = w.layers[0]
    g = GrapeStep.for_workload(w, path=grape.GRAPE_PATH_TC)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    out = torch.full((w.B,), -1.0, device="cuda")
    for s in range(2):   # two calls in a row: different steps, different inputs
        x = W.make_step_inputs(w, s)
        A, G = to_device(x.A[0], "bf16"), to_device(x.Gout[0], "bf16")
        g.step([A], [G], Wd, s)
        grape.grape_layer_sqnorms_static(A, G, d_in, d_out, w.r, w.B, w.T, w.seed, 0, s, out)
        torch.cuda.synchronize()
        ref = g.norms().astype(np.float64) ** 2   # one layer: n_i^2 is its squared norm
        got = out.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)) and np.all(got > 0)
        err = rel_fro(got, ref)
        print(f"call {s}: relative Frobenius difference {err:.2e}")
        assert err <= TOL
    g.close()


def test_static_sqnorms_reject_problems_beyond_the_scratch():
    A = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(grape.GrapeError) as e:
        # AP alone would need 64 * 4096 * 256 * 2 bytes = 128 MiB
        grape.grape_layer_sqnorms_static(A, A, 4096, 4096, 256, 64, 4096, 0, 0, 0, A)
    assert e.value.code == grape.GRAPE_EINVAL
    assert "static scratch" in str(e.value)
