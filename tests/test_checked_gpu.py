"""The bounds-checked build (GRAPE_CHECKED) on the tensor-core path (needs a B200).

tests/checked_cases.py runs in a fresh process with GRAPE_LIB=checked: ragged T and
d_in, r = 512, two launch groups, the cluster aggregation, the norm kernel with
(A_i P)^T in TMEM and the fused aggregation + Adam, ghost norms, a masked step and the
entry point with static scratch.  Every TMA box must pass its check: a failed
check raises from the library (or gives NaN from the static entry point) and fails the
run, and the results still match the oracle.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_every_tma_box_passes_the_bounds_check():
    from random_gradient_projection_b200 import build
    build.build(checked=True)
    env = dict(os.environ, GRAPE_LIB="checked")
    out = subprocess.run([sys.executable, os.path.join(HERE, "checked_cases.py")], env=env,
                         capture_output=True, text=True, timeout=600)
    print(out.stdout[-3000:])
    assert out.returncode == 0, out.stderr[-3000:]
    assert "ALL OK" in out.stdout
