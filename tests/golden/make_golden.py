"""Write the oracle's expected values for the tiny fp32 workload (64x32 layer, r=8,
B=4, T=16, three steps) to ``tiny_f32_oracle.json``.

Calls only ``oracle/`` and ``workloads``.  The pages print no worked example, so
these values are regression anchors for the oracle and the expected values of
the GPU parity test on that workload, not a pin against the pages.
Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle.grape_oracle as O  # noqa: E402
import workloads as W  # noqa: E402


def main():
    w = W.get("tiny_f32")
    res = O.run(w, w.steps)
    st = res["state"]
    out = {
        "workload": w.name,
        "source": "oracle/grape_oracle.py run() on workloads.get('tiny_f32'), "
                  "method of 'Memory-Efficient Differentially Private Training with Gradient "
                  "Random Projection', Resumen Tecnico > Metodologia",
        "steps": [{"norms": t["norms"].tolist(), "clip": t["clip"].tolist(),
                   "S": [s.tolist() for s in t["S"]]} for t in res["trace"]],
        "W": [x.tolist() for x in st.W],
        "m": [x.tolist() for x in st.m],
        "v": [x.tolist() for x in st.v],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32_oracle.json")
    with open(path, "w") as f:
        json.dump(out, f)
    print("wrote", path)


if __name__ == "__main__":
    main()
