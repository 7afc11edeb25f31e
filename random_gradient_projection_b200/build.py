"""Build libgrape.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m random_gradient_projection_b200.build [--force] [--verbose]

The library links the CUDA runtime statically and reaches the driver API
(tensor-map encoding) through cudaGetDriverEntryPoint, so it needs no
libcuda at link time and cross-compiles on a machine without a GPU.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libgrape.so")
# bounds-checked variant (-DGRAPE_CHECKED): every TMA box start is checked in the kernels
LIB_CHECKED = os.path.join(HERE, "libgrape_checked.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in sources() + headers() + [__file__])


def build(force: bool = False, verbose: bool = False, extra=None, checked: bool = False) -> str:
    """Build libgrape.so, or with ``checked`` the bounds-checked libgrape_checked.so."""
    lib = LIB_CHECKED if checked else LIB
    if not force and up_to_date(lib):
        return lib
    flags = ["-DGRAPE_CHECKED"] if checked else []
    cmd = [nvcc(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-cudart", "static", "-I", os.path.join(ROOT, "include"),
           "-Xptxas", "-warn-spills", *flags, *(extra or []), *sources(), "-ldl", "-o", lib + ".tmp"]
    if verbose:
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print registers / spills per kernel")
    ap.add_argument("--checked", action="store_true",
                    help="build the bounds-checked libgrape_checked.so (GRAPE_LIB=checked loads it)")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_v else None
    print(build(force=a.force or a.ptxas_v, verbose=a.verbose or a.ptxas_v, extra=extra, checked=a.checked))


if __name__ == "__main__":
    sys.exit(main())
