"""The parity comparison itself (CPU): it accepts the oracle against itself and rejects
plausible mistakes of the update that leave S, m and v untouched.

The "library" side here is another oracle run, in the trace format the GPU tests build,
so the check can be shown to fail without a faulty kernel."""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W
from harness import compare, rel_fro

# small bf16 stack: two layers, two 128-row back-projection tiles in the first
WL = W.Workload("cmp", ((256, 128), (256, 256)), r=32, B=4, T=16, dtype="bf16", C=1.0,
                sigma=0.8, steps=2)
STEPS = 2


def as_library(res):
    """An oracle run shaped like the library's trace: fp32 host copies, dR per step."""
    f32 = lambda xs: [np.asarray(x, dtype=np.float32) for x in xs]   # noqa: E731
    trace = [{"norms": np.asarray(t["norms"], np.float32), "clip": np.asarray(t["clip"], np.float32),
              "S": f32(t["S"]), "m": f32(t["m"]), "v": f32(t["v"]), "dR": f32(t["dR"])}
             for t in res["trace"]]
    return {"trace": trace, "W": f32(res["state"].W)}


@pytest.fixture(scope="module")
def reference():
    res = O.run(WL, STEPS)
    return {"trace": res["trace"], "state": res["state"]}


def test_oracle_against_itself_passes(reference):
    worst = compare(WL, as_library(O.run(WL, STEPS)), reference, 2e-2, STEPS)
    assert worst["S"] < 1e-6 and worst["dR"] < 1e-6 and worst["dW"] < 1e-5


def test_learning_rate_off_by_a_quarter_fails(reference):
    """lr x 1.25 on the library side leaves S, m, v and dR as they are; the updated W still
    agrees to well inside the tolerance, because W_0 dominates it; W - W_0 does not."""
    lib = as_library(O.run(WL.replace(lr=WL.lr * 1.25), STEPS))
    W_only = max(rel_fro(lib["W"][l], reference["state"].W[l]) for l in range(WL.n_layers))
    assert W_only < 2e-2          # what the W check alone would accept
    with pytest.raises(AssertionError, match="of dW"):
        compare(WL, lib, reference, 2e-2, STEPS)


def test_missing_first_moment_bias_correction_fails(reference, monkeypatch):
    """dR = m / (sqrt(v_hat) + eps): the first moment left uncorrected in dR only."""
    def adam_no_bc1(m, v, g, t, beta1, beta2, eps):
        m = beta1 * m + (1.0 - beta1) * g
        v = beta2 * v + (1.0 - beta2) * g * g
        return m, v, m / (np.sqrt(v / (1.0 - beta2 ** t)) + eps)
    monkeypatch.setattr(O, "adam", adam_no_bc1)
    lib = as_library(O.run(WL, STEPS))
    monkeypatch.undo()
    with pytest.raises(AssertionError, match="of dR"):
        compare(WL, lib, reference, 2e-2, STEPS)


def test_wrong_projection_on_one_back_projection_tile_fails(reference):
    """The first 128 rows of layer 0's update back-projected through another step's P."""
    lib = as_library(O.run(WL, STEPS))
    w2 = WL.replace(seed=WL.seed + 1)
    other_update = O.run(w2, STEPS)["state"].W[0] - W.make_weights(w2)[0]
    W0 = W.make_weights(WL)[0]
    lib["W"][0][:128] = (W0[:128] + other_update[:128]).astype(np.float32)
    with pytest.raises(AssertionError, match="of dW"):
        compare(WL, lib, reference, 2e-2, STEPS)


def test_noise_free_first_step_leaves_only_sign_decisions_out():
    """sigma = 0: dR at t = 1 is the sign of S; elements whose sign an S within the
    tolerance does not fix are left out of the dR check and their directions out of the
    W - W_0 check, and an S perturbed within tolerance still passes."""
    w = WL.replace(sigma=0.0)
    ref = O.run(w, 1)
    rng = np.random.default_rng(3)

    def perturbed_adam(m, v, g, t, beta1, beta2, eps):
        g = g + rng.standard_normal(g.shape) * 3e-3 * np.sqrt(np.mean(g * g))
        return O_adam(m, v, g, t, beta1, beta2, eps)
    O_adam = O.adam
    O.adam = perturbed_adam
    try:
        lib = as_library(O.run(w, 1))
    finally:
        O.adam = O_adam
    worst = compare(w, lib, {"trace": ref["trace"], "state": ref["state"]}, 2e-2, 1)
    assert 0.0 < worst["dR_left_out"] <= 0.05
