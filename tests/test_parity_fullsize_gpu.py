"""Parity at the full layer shapes of the ViT-B, 7B-slice and long-context workloads
(needs a B200).

* sub-batch: the same layer stacks, token counts, seeds and hyper-parameters with
  B' = 2 samples, one step through the C ABI against the whole fp64 oracle step;
* full batch, in the launch configuration the benchmark uses for that workload:
  one step at the workload's own B; the per-sample norms of the first and last
  sample are recomputed one by one by the oracle, and properties that hold at any
  size are checked on every sample (clip bound, clip decisions, finite S).
"""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W
from harness import compare, rel_fro, run_library, run_oracle, to_device

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeStep, grape  # noqa: E402

TC = grape.GRAPE_PATH_TC
NAMES = ["vit_b", "llm7b_slice", "longctx"]


@pytest.mark.parametrize("name", NAMES)
def test_full_shapes_sub_batch(name):
    w = W.get(name).replace(B=2)
    lib = run_library(w, 1, TC)
    orc = run_oracle(w, 1)
    worst = compare(w, lib, orc, 2e-2, 1)
    print(name, "B'=2", {k: f"{v:.2e}" for k, v in worst.items()})


@pytest.mark.parametrize("name", NAMES)
def test_full_batch_sampled(name):
    w = W.get(name)
    g = GrapeStep.for_workload(w, path=TC)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0, threads=16)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    g.step(A, G, Wd, 0)
    torch.cuda.synchronize()
    norms, clip = g.norms(), g.clip()
    assert np.all(np.isfinite(norms)) and np.all(norms > 0)
    assert np.all(clip * norms <= w.C * (1 + 1e-6))
    assert np.all(clip[norms <= w.C] == 1.0)
    for l in (0, w.n_layers - 1):
        assert np.all(np.isfinite(g.S(l)))
    del A, G
    # the first and the last sample, one by one in fp64
    samples = [0, w.B - 1]
    xs = W.make_step_inputs(w, 0, samples=samples, threads=16)
    ref = O.sample_norms([xs.as_f64(a) for a in xs.A], [xs.as_f64(gg) for gg in xs.Gout], 0,
                         O.Hyper.of(w), [di for di, _ in w.layers])
    err = rel_fro(norms[samples], ref)
    print(name, "full batch, norms of samples", samples, f"rel err {err:.2e}")
    assert err <= 2e-2
    away = np.abs(ref - w.C) / w.C > 1e-3
    assert np.array_equal((clip[samples] < 1)[away], (ref > w.C)[away])
    g.close()
