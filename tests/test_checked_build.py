"""The bounds-checked variant of the library builds, exports the same C ABI, and leaves
the default build untouched (CPU only; nvcc cross-compiles)."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "random_gradient_projection_b200", "csrc")


def _exports(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    return set(re.findall(r"\sT\s(grape_\w+)$", out, flags=re.M))


def test_checked_library_exports_the_same_abi():
    from random_gradient_projection_b200 import build
    default, checked = build.build(), build.build(checked=True)
    assert checked.endswith("libgrape_checked.so")
    assert _exports(checked) == _exports(default) != set()


@pytest.mark.parametrize("checked", [False, True], ids=["default", "checked"])
def test_the_check_exists_only_in_the_checked_build(checked):
    """Preprocess tc.cu for the device: the box check is in the checked build's kernels and
    nowhere in the default build's."""
    from random_gradient_projection_b200 import build
    cmd = [build.nvcc(), *build.ARCH, "-std=c++17", "-I", os.path.join(ROOT, "include"), "-E",
           "-D__CUDA_ARCH__=1000", os.path.join(CSRC, "tc.cu")]
    if checked:
        cmd.insert(1, "-DGRAPE_CHECKED")
    pre = subprocess.run(cmd, capture_output=True, text=True)
    assert pre.returncode == 0, pre.stderr[-2000:]
    calls = len(re.findall(r"\bbox_ok\s*\(", pre.stdout))
    copies = len(re.findall(r"ptx::tma_(?:load|store)_\w+\(", open(os.path.join(CSRC, "tc.cu")).read()))
    if checked:
        assert copies >= 11 and calls == copies + 1   # the definition and one check per TMA copy
    else:
        assert calls == 0 and "extA" not in pre.stdout
