"""The oracle reproduces its stored expected values for the tiny fp32 workload."""
import json
import os

import numpy as np

import oracle.grape_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_f32_oracle.json")


def test_tiny_f32_golden():
    g = json.load(open(GOLDEN))
    w = W.get("tiny_f32")
    res = O.run(w, w.steps)
    for t, gt in zip(res["trace"], g["steps"]):
        assert np.allclose(t["norms"], gt["norms"], rtol=1e-12)
        assert np.array_equal(t["clip"] < 1, np.array(gt["clip"]) < 1)
        for s, gs in zip(t["S"], gt["S"]):
            assert np.allclose(s, gs, rtol=1e-11, atol=1e-14)
    st = res["state"]
    for name in ("W", "m", "v"):
        for a, b in zip(getattr(st, name), g[name]):
            assert np.allclose(a, b, rtol=1e-11, atol=1e-15), name


def test_tiny_f32_clips_some_not_all():
    """The input recipe puts samples on both sides of C."""
    g = json.load(open(GOLDEN))
    c = np.array([s["clip"] for s in g["steps"]])
    assert (c < 1).any() and (c == 1).any()
