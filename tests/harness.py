"""Shared helpers of the parity tests: run a workload through the library and the oracle
on the same seeded inputs and compare."""
from __future__ import annotations

import numpy as np

import oracle.grape_oracle as O
import workloads as W


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


def run_library(w, steps: int, path: int, capture=True):
    """Run ``steps`` steps through the C ABI; return per-step intermediates and final state."""
    import torch
    from random_gradient_projection_b200 import GrapeStep
    g = GrapeStep.for_workload(w, path=path)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    trace = []
    for s in range(steps):
        x = W.make_step_inputs(w, s, threads=8)
        A = [to_device(a, w.dtype) for a in x.A]
        G = [to_device(a, w.dtype) for a in x.Gout]
        g.step(A, G, Ws, s)
        torch.cuda.synchronize()
        if capture:
            trace.append({"norms": g.norms(), "clip": g.clip(),
                          "S": [g.S(l) for l in range(w.n_layers)],
                          "m": [g.m(l) for l in range(w.n_layers)],
                          "v": [g.v(l) for l in range(w.n_layers)],
                          "dR": [g.dR(l) for l in range(w.n_layers)]})
    out = {"trace": trace, "W": [x.cpu().numpy() for x in Ws], "path": g.path}
    g.close()
    return out


def run_oracle(w, steps: int):
    res = O.run(w, steps)
    return {"trace": res["trace"], "state": res["state"]}


def compare(w, lib, orc, tol: float, steps: int):
    """Assert the library's step matches the oracle's within ``tol`` (relative Frobenius) on
    S (the clipped sum), m, v and W, and that clip decisions agree away from C."""
    worst = {}
    st = orc["state"]
    for s in range(steps):
        lt, ot = lib["trace"][s], orc["trace"][s]
        n_o = np.asarray(ot["norms"])
        worst["norms"] = max(worst.get("norms", 0.0), rel_fro(lt["norms"], n_o))
        away = np.abs(n_o - w.C) / w.C > 1e-3
        assert np.array_equal((lt["clip"] < 1)[away], (np.asarray(ot["clip"]) < 1)[away]), \
            f"step {s}: clip decisions differ"
        for l in range(w.n_layers):
            worst["S"] = max(worst.get("S", 0.0), rel_fro(lt["S"][l], ot["S"][l]))
    for l in range(w.n_layers):
        worst["m"] = max(worst.get("m", 0.0), rel_fro(lib["trace"][-1]["m"][l], st.m[l]))
        worst["v"] = max(worst.get("v", 0.0), rel_fro(lib["trace"][-1]["v"][l], st.v[l]))
        worst["W"] = max(worst.get("W", 0.0), rel_fro(lib["W"][l], st.W[l]))
    for k, e in worst.items():
        assert e <= tol, f"{w.name}: relative Frobenius error of {k} = {e:.3e} > {tol:.1e}"
    return worst
