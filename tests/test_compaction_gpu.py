"""Live-token compaction (grape_enable_compaction / grape_step_masked) through the C ABI
(needs a B200), against the fp64 oracle on the full, uncompacted inputs.

* the long-context recipe (a Bernoulli(0.1) loss mask zeroes 90 % of Gout rows):
  whole-step parity over several steps on both paths, ragged T_full and T_cap;
* a mask stricter than the zero rows: masked tokens whose Gout is not zero are still
  dropped (oracle: the step on apply_token_mask(Gout, mask));
* edge cases: a sample with no kept token, one at exactly the capacity, and a sample
  over the capacity (reported as GRAPE_EINVAL by the next synchronising call);
* the full long-context shape (B = 8, T = 8192, capacity 1024): sampled norms.
"""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W
from harness import compare, rel_fro, snapshot, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeError, GrapeStep, grape  # noqa: E402

SIMT, TC = grape.GRAPE_PATH_SIMT, grape.GRAPE_PATH_TC


def _run(w, T_cap, steps, path, mask_fn=None):
    """Library: compacted steps; oracle: the same steps on the full inputs with the mask
    applied to Gout.  ``mask_fn(s, generator_mask)`` gives the mask passed in."""
    g = GrapeStep.for_workload(w.replace(T=T_cap), path=path)
    g.enable_compaction(w.T)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    h = O.Hyper.of(w)
    st = O.State.init(W.make_weights(w), w.r)
    lib_trace, orc_trace, counts = [], [], []
    for s in range(steps):
        x = W.make_step_inputs(w, s, threads=8)
        mask = (x.mask != 0) if mask_fn is None else mask_fn(s, x.mask != 0)
        A = [to_device(a, w.dtype) for a in x.A]
        G = [to_device(a, w.dtype) for a in x.Gout]
        g.step_masked(A, G, Wd, torch.from_numpy(mask.astype(np.uint8)).cuda(), s)
        torch.cuda.synchronize()
        counts.append(g.live_counts())
        lib_trace.append(snapshot(g, w.n_layers))
        Gm = O.apply_token_mask([x.as_f64(a) for a in x.Gout], mask)
        orc_trace.append(O.step(st, [x.as_f64(a) for a in x.A], Gm, s, h))
        assert np.array_equal(counts[-1], np.minimum(mask.sum(axis=1), T_cap))
    lib = {"trace": lib_trace, "W": [t.cpu().numpy() for t in Wd]}
    g.close()
    return lib, {"trace": orc_trace, "state": st}, counts


CASES = {
    # long-context recipe, reduced: T_full = 1000 (ragged), about 100 kept tokens per sample
    "longctx_2layers_T1000": (W.scaled(W.get("longctx"), layers=((2048, 2048), (2048, 6144)), B=3, T=1000),
                              192, 3),
    "tiny_f32_masked": (W.scaled(W.get("tiny_f32"), mask_p=0.5), 12, 3),
}
PAIRS = [("longctx_2layers_T1000", TC), ("longctx_2layers_T1000", SIMT), ("tiny_f32_masked", SIMT)]


@pytest.mark.parametrize("case,path", PAIRS, ids=[f"{c}-{'tc' if p == TC else 'simt'}" for c, p in PAIRS])
def test_masked_step_matches_oracle(case, path):
    w, T_cap, steps = CASES[case]
    tol = 1e-5 if (w.dtype == "f32" and path == SIMT) else 2e-2
    lib, orc, counts = _run(w, T_cap, steps, path)
    worst = compare(w, lib, orc, tol, steps)
    print(case, "kept tokens", [c.tolist() for c in counts], {k: f"{v:.2e}" for k, v in worst.items()})


def test_mask_drops_tokens_with_nonzero_gout():
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=96)

    def stricter(s, m):
        m = m.copy()
        m[:, ::3] = False          # drop every third token although its Gout is not zero
        return m
    lib, orc, counts = _run(w, 72, 2, TC, stricter)
    worst = compare(w, lib, orc, 2e-2, 2)
    print("stricter mask", {k: f"{v:.2e}" for k, v in worst.items()})


@pytest.mark.parametrize("path", [SIMT, TC])
def test_empty_full_and_overflowing_samples(path):
    w = W.scaled(W.get("mlp4x1024"), n_layers=1, B=3, T=80)
    T_cap = 64

    def edges(s, m):
        m = np.zeros_like(m)
        m[1, 5:5 + T_cap] = True   # exactly at the capacity
        m[2, ::7] = True           # 12 kept tokens; sample 0 keeps none
        return m
    lib, orc, counts = _run(w, T_cap, 1, path, edges)
    assert counts[0].tolist() == [0, T_cap, 12]
    assert lib["trace"][0]["norms"][0] == 0.0 and lib["trace"][0]["clip"][0] == 1.0
    compare(w, lib, orc, 2e-2, 1)
    # over the capacity: the next synchronising call reports it, and the flag clears
    g = GrapeStep.for_workload(w.replace(T=T_cap), path=path)
    g.enable_compaction(w.T)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0, threads=8)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    full = torch.ones((w.B, w.T), dtype=torch.uint8, device="cuda")
    g.step_masked(A, G, Wd, full, 0)
    with pytest.raises(GrapeError) as e:
        g.live_counts()
    assert e.value.code == grape.GRAPE_EINVAL
    assert g.live_counts().tolist() == [T_cap] * w.B
    with pytest.raises(GrapeError):
        g.enable_compaction(w.T)               # only once
    g.close()


def test_full_longctx_masked_sampled_norms():
    w = W.get("longctx")
    T_cap = 1024
    g = GrapeStep.for_workload(w.replace(T=T_cap), path=TC)
    g.enable_compaction(w.T)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0, threads=16)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    g.step_masked(A, G, Wd, torch.from_numpy((x.mask != 0).astype(np.uint8)).cuda(), 0)
    torch.cuda.synchronize()
    counts = g.live_counts()
    assert np.array_equal(counts, (x.mask != 0).sum(axis=1))
    norms = g.norms()
    del A, G
    samples = [0, w.B - 1]
    xs = W.make_step_inputs(w, 0, samples=samples, threads=16)
    ref = O.sample_norms([xs.as_f64(a) for a in xs.A], [xs.as_f64(a) for a in xs.Gout], 0, O.Hyper.of(w),
                         [di for di, _ in w.layers])
    err = rel_fro(norms[samples], ref)
    print("longctx masked, kept", counts.tolist(), f"norms rel err {err:.2e}")
    assert err <= 2e-2
    g.close()
