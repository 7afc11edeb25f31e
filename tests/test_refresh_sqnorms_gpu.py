"""Projection-refresh period K and the Hutchinson per-sample norm estimate, through the C ABI
(needs a B200), against the fp64 oracle.

* refresh: several steps with K = 2, 3 and K larger than the run, whole-step parity
  (S, norms, clip decisions, m, v, W), and the launch count showing that a step inside a
  period does not regenerate P while the P it uses is unchanged;
* Hutchinson: ``grape_sqnorms`` against the oracle's explicit-O estimator on the same P,
  against the step's own norms, on ragged T, several tiles and both paths, and with m,
  v and W left untouched.
"""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W
from harness import compare, rel_fro, run_library, run_oracle, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeError, GrapeStep, grape  # noqa: E402

SIMT, TC = grape.GRAPE_PATH_SIMT, grape.GRAPE_PATH_TC

REFRESH = {
    "tiny_f32_K2": (W.scaled(W.get("tiny_f32"), refresh=2), SIMT, 5, 1e-5),
    "tiny_f32_K3": (W.scaled(W.get("tiny_f32"), refresh=3), SIMT, 5, 1e-5),
    "mlp_2x1024_K2": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=4, refresh=2), TC, 4, 2e-2),
    "vit_ragged_K10": (W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768)), B=3, refresh=10),
                       TC, 3, 2e-2),
}


@pytest.mark.parametrize("case", sorted(REFRESH))
def test_refresh_period_matches_oracle(case):
    w, path, steps, tol = REFRESH[case]
    lib = run_library(w, steps, path)
    orc = run_oracle(w, steps)
    worst = compare(w, lib, orc, tol, steps)
    print(case, {k: f"{v:.2e}" for k, v in worst.items()})


@pytest.mark.parametrize("path", [SIMT, TC])
def test_refresh_skips_generation_and_keeps_P(path):
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=2, T=64, refresh=3)
    g = GrapeStep.for_workload(w, path=path)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0, threads=8)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    counts, Ps = [], []
    for s in range(4):
        c0 = g.launch_count()
        g.step(A, G, Ws, s)
        torch.cuda.synchronize()
        counts.append(g.launch_count() - c0)
        Ps.append(g.P(0))
    gen = 1    # P generation is one launch on both paths
    assert counts[1] == counts[0] - gen and counts[2] == counts[0] - gen and counts[3] == counts[0]
    assert np.array_equal(Ps[0], Ps[1]) and np.array_equal(Ps[1], Ps[2])
    assert not np.array_equal(Ps[2], Ps[3])
    # P of key 1 is the oracle's projection for step field 1 (bf16 on the tensor path)
    ref = O.projection_matrix(w.seed, 0, 1, w.layers[0][0], w.r)
    assert rel_fro(Ps[3], ref) < (5e-3 if path == TC else 1e-6)
    # setting the period again forces a fresh P on the next step
    g.set_refresh_period(3)
    c0 = g.launch_count()
    g.step(A, G, Ws, 4)
    torch.cuda.synchronize()
    assert g.launch_count() - c0 == counts[0]
    with pytest.raises(GrapeError):
        g.set_refresh_period(0)
    g.close()


SQN = {
    "tiny_f32": (W.get("tiny_f32"), SIMT, 1e-5),
    "mlp_2x1024_B4": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=4), TC, 2e-2),
    "vit_qkv_down_B3_T197": (W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768)), B=3), TC, 2e-2),
    "r512_T130": (W.scaled(W.get("llm7b_slice"), layers=((512, 1024),), r=512, B=2, T=130), TC, 2e-2),
    "mlp_K2_step3": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=64, refresh=2), TC, 2e-2),
    # the DP-SGD-RC page's sketch width k = 32, on odd fp32 shapes (CUDA-core path)
    "f32_k32_T100": (W.scaled(W.get("tiny_f32"), layers=((256, 192), (96, 130)), r=32, B=5, T=100),
                     SIMT, 1e-5),
}


@pytest.mark.parametrize("case", sorted(SQN))
def test_sqnorms_match_hutchinson_oracle(case):
    w, path, tol = SQN[case]
    step = 3
    g = GrapeStep.for_workload(w, path=path)
    x = W.make_step_inputs(w, step, threads=8)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    got = g.sqnorms(A, G, step).cpu().numpy().astype(np.float64)
    ref = O.hutchinson_sample_sqnorms([x.as_f64(a) for a in x.A], [x.as_f64(a) for a in x.Gout], step,
                                      O.Hyper.of(w), [di for di, _ in w.layers])
    err = rel_fro(got, ref)
    print(case, f"rel err {err:.2e}")
    assert err <= tol
    assert np.all(got >= 0)
    g.close()


@pytest.mark.parametrize("path", [SIMT, TC])
def test_sqnorms_equal_the_steps_norms_and_touch_no_state(path):
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=32)
    g = GrapeStep.for_workload(w, path=path)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0, threads=8)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    g.step(A, G, Ws, 0)
    torch.cuda.synchronize()
    n_step, m0, W0 = g.norms(), g.m(0), Ws[0].cpu().numpy()
    sq = g.sqnorms(A, G, 0).cpu().numpy()
    torch.cuda.synchronize()
    # the same kernels on the same P: the sum of the same partials in the same order
    assert np.allclose(sq, n_step.astype(np.float64) ** 2, rtol=2e-6, atol=0)
    assert np.array_equal(g.m(0), m0) and np.array_equal(Ws[0].cpu().numpy(), W0)
    assert np.array_equal(g.norms(), n_step)
    g.close()


def test_sqnorms_rejects_bad_output():
    w = W.scaled(W.get("mlp4x1024"), n_layers=1, B=2, T=16)
    g = GrapeStep.for_workload(w)
    x = W.make_step_inputs(w, 0, threads=8)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    with pytest.raises(GrapeError):
        grape.grape_sqnorms(g.ctx, A, G, 0, None)
    g.close()
