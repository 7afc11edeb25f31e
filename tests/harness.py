"""Shared helpers of the parity tests: run a workload through the library and the oracle
on the same seeded inputs and compare."""
from __future__ import annotations

import numpy as np

import oracle.grape_oracle as O
import workloads as W

# An element of the Adam direction dR is compared only where the oracle's own Adam
# denominator sqrt(v_hat) exceeds KAPPA times the per-element error of the averaged
# gradient g that the tolerance allows (tol * rms(S) / batch).  Below it the direction is
# a decision the arithmetic cannot take reliably: at t = 1, dR = g / (|g| + eps) is the
# sign of g, and an S within tolerance can flip it where |g| is that small.
KAPPA = 2.0


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def to_device(x, dtype: str):
    """A stored input array (uint16 bf16 patterns or float32) as a CUDA tensor."""
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def snapshot(g, n_layers: int) -> dict:
    """The last step's intermediates of a GrapeStep, copied to the host."""
    return {"norms": g.norms(), "clip": g.clip(),
            "S": [g.S(l) for l in range(n_layers)],
            "m": [g.m(l) for l in range(n_layers)],
            "v": [g.v(l) for l in range(n_layers)],
            "dR": [g.dR(l) for l in range(n_layers)]}


def run_library(w, steps: int, path: int, capture=True, setup=None):
    """Run ``steps`` steps through the C ABI; return per-step intermediates and final state.
    ``setup(g)`` configures the context before the first step."""
    import torch
    from random_gradient_projection_b200 import GrapeStep
    g = GrapeStep.for_workload(w, path=path)
    if setup:
        setup(g)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    trace = []
    for s in range(steps):
        x = W.make_step_inputs(w, s, threads=8)
        A = [to_device(a, w.dtype) for a in x.A]
        G = [to_device(a, w.dtype) for a in x.Gout]
        g.step(A, G, Ws, s)
        torch.cuda.synchronize()
        if capture:
            trace.append(snapshot(g, w.n_layers))
    out = {"trace": trace, "W": [x.cpu().numpy() for x in Ws], "path": g.path}
    g.close()
    return out


def run_oracle(w, steps: int):
    res = O.run(w, steps)
    return {"trace": res["trace"], "state": res["state"]}


def well_conditioned(w, ot: dict, l: int, t: int, tol: float, divisor: int) -> np.ndarray:
    """Elements of layer l's dR at Adam step t that an S within ``tol`` determines."""
    S = np.asarray(ot["S"][l], dtype=np.float64)
    rms_S = np.linalg.norm(S) / np.sqrt(max(S.size, 1))
    v_hat = np.asarray(ot["v"][l], dtype=np.float64) / (1.0 - w.beta2 ** t)
    return np.sqrt(v_hat) > KAPPA * tol * rms_S / divisor


def _undetermined_projector(P_cols):
    """x -> x minus its least-squares component in span(P_cols) (d_in x k), or None."""
    if not P_cols:
        return None
    V = np.stack(P_cols, axis=1)
    return lambda x: x - V @ np.linalg.lstsq(V, x, rcond=None)[0]


def delta_w_error(w, lib_W, orc_trace, st, tol: float, steps: int, divisor: int) -> float:
    """Relative Frobenius error of the library's update W - W_0 against the oracle's.

    Each column n of W - W_0 = -lr sum_t P_t dR_t is a combination of the columns of P_t;
    the directions P_t[:, j] of the dR elements that the S tolerance leaves undetermined
    (``well_conditioned`` false) are projected out of both sides, column by column, before
    the comparison.  With noise they are a handful of elements, usually none."""
    W0 = W.make_weights(w)
    num = den = 0.0
    for l in range(w.n_layers):
        d_lib = np.asarray(lib_W[l], dtype=np.float64) - W0[l]
        d_orc = np.asarray(st.W[l], dtype=np.float64) - W0[l]
        bad_cols = {}
        for s in range(steps):
            ot = orc_trace[s]
            bad = ~well_conditioned(w, ot, l, s + 1, tol, divisor)
            for j, n in zip(*np.nonzero(bad)):
                bad_cols.setdefault(int(n), []).append(ot["P"][l][:, j])
        for n, cols in bad_cols.items():
            proj = _undetermined_projector(cols)
            d_lib[:, n] = proj(d_lib[:, n])
            d_orc[:, n] = proj(d_orc[:, n])
        num += float(np.sum((d_lib - d_orc) ** 2))
        den += float(np.sum(d_orc ** 2))
    return float(np.sqrt(num / den)) if den > 0 else float(np.sqrt(num))


def compare(w, lib, orc, tol: float, steps: int, divisor=None):
    """Assert the library's step matches the oracle's within ``tol`` (relative Frobenius):

    * per step: the norms, S (the clipped sum), m and v, and the Adam direction dR on the
      elements an S within ``tol`` determines (``well_conditioned``; at most 5 % of them
      may be left out, which only a noise-free first step comes near);
    * at the end: the update W - W_0 (directions of left-out dR elements projected out)
      and W itself;
    and that clip decisions agree away from C.  ``divisor`` is the batch the noisy sum is
    averaged over (B by default)."""
    worst = {}
    st = orc["state"]
    div = divisor or w.B
    left_out = 0.0
    for s in range(steps):
        lt, ot = lib["trace"][s], orc["trace"][s]
        n_o = np.asarray(ot["norms"])
        worst["norms"] = max(worst.get("norms", 0.0), rel_fro(lt["norms"], n_o))
        away = np.abs(n_o - w.C) / w.C > 1e-3
        assert np.array_equal((lt["clip"] < 1)[away], (np.asarray(ot["clip"]) < 1)[away]), \
            f"step {s}: clip decisions differ"
        for l in range(w.n_layers):
            worst["S"] = max(worst.get("S", 0.0), rel_fro(lt["S"][l], ot["S"][l]))
            worst["m"] = max(worst.get("m", 0.0), rel_fro(lt["m"][l], ot["m"][l]))
            worst["v"] = max(worst.get("v", 0.0), rel_fro(lt["v"][l], ot["v"][l]))
            ok = well_conditioned(w, ot, l, s + 1, tol, div)
            left_out = max(left_out, 1.0 - float(np.mean(ok)))
            worst["dR"] = max(worst.get("dR", 0.0),
                              rel_fro(np.asarray(lt["dR"][l])[ok], np.asarray(ot["dR"][l])[ok]))
    worst["dW"] = delta_w_error(w, lib["W"], orc["trace"], st, tol, steps, div)
    for l in range(w.n_layers):
        worst["W"] = max(worst.get("W", 0.0), rel_fro(lib["W"][l], st.W[l]))
    for k, e in worst.items():
        assert e <= tol, f"{w.name}: relative Frobenius error of {k} = {e:.3e} > {tol:.1e}"
    assert left_out <= 0.05, f"{w.name}: {left_out:.1%} of dR left out as undetermined"
    worst["dR_left_out"] = left_out
    return worst
