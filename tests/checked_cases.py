"""Tensor-core cases run through the bounds-checked library (GRAPE_LIB=checked).

Run as a script by tests/test_checked_gpu.py in a fresh process, because the binding
chooses its library at import.  Each case runs whole steps and reads the results back;
reading synchronises and raises GrapeError if any kernel found a TMA box outside its
tensor.  The results must still match the oracle, since a skipped copy would show.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import torch  # noqa: E402

import workloads as W  # noqa: E402
from harness import compare, run_library, run_oracle, to_device  # noqa: E402
from random_gradient_projection_b200 import GrapeStep, grape  # noqa: E402

TC = grape.GRAPE_PATH_TC

CASES = {
    # ragged T, r = 512 (256-wide projection tiles), two N tiles
    "r512_T130": W.Workload("r512", ((1024, 2816), (2816, 1024)), r=512, B=2, T=130, dtype="bf16",
                            C=1.0, sigma=0.6, steps=2),
    # d_in off the k-block and the back-projection tile
    "ragged_d_in": W.Workload("ragged_din", ((520, 256), (136, 512)), r=128, B=3, T=40, dtype="bf16",
                              C=1.0, sigma=0.8, steps=2),
    # two launch groups
    "20_layers": W.Workload("twenty", tuple([(256, 256), (512, 256)] * 10), r=128, B=3, T=64,
                            dtype="bf16", C=1.0, sigma=1.0, steps=2),
    # T = 197, d_out = 2304: the cluster aggregation over few output tiles
    "vit_B3": W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768)), B=3),
}


def main():
    assert grape.LIB_PATH.endswith("libgrape_checked.so"), grape.LIB_PATH
    for name, w in CASES.items():
        lib = run_library(w, 2, TC)
        worst = compare(w, lib, run_oracle(w, 2), 2e-2, 2)
        print("checked", name, {k: f"{v:.1e}" for k, v in worst.items()}, flush=True)

    # the norm kernel with (A_i P)^T in TMEM and the fused aggregation + noise + Adam:
    # stored R_i at T = 512 (the default there), and the ragged T = 130 forced onto it
    w = W.Workload("r512_T512", ((512, 1024), (1024, 512)), r=512, B=2, T=512, dtype="bf16", C=1.0,
                   sigma=1.0, steps=2)
    worst = compare(w, run_library(w, 2, TC), run_oracle(w, 2), 2e-2, 2)
    print("checked r512_T512", {k: f"{v:.1e}" for k, v in worst.items()}, flush=True)
    os.environ["GRAPE_NORM_TMEM"] = "1"   # read when a context is created
    w = CASES["r512_T130"]
    lib = run_library(w, 2, TC, setup=lambda g: g.set_aggregation(grape.GRAPE_AGG_STORE))
    del os.environ["GRAPE_NORM_TMEM"]
    worst = compare(w, lib, run_oracle(w, 2), 2e-2, 2)
    print("checked r512_T130 stored, TMEM norms", {k: f"{v:.1e}" for k, v in worst.items()}, flush=True)

    # ghost norms (T <= 128)
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=100)
    g = GrapeStep.for_workload(w, path=TC)
    g.set_norm_method(grape.GRAPE_NORM_GHOST)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0)
    g.step([to_device(a, w.dtype) for a in x.A], [to_device(a, w.dtype) for a in x.Gout], Wd, 0)
    n = g.norms()
    g.close()
    print("checked ghost", n, flush=True)

    # a masked step over compacted rows
    w = W.scaled(W.get("longctx"), layers=((2048, 2048),), B=2, T=600)
    g = GrapeStep.for_workload(w.replace(T=128), path=TC)
    g.enable_compaction(w.T)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0)
    mask = torch.from_numpy((x.mask != 0).astype(np.uint8)).cuda()
    g.step_masked([to_device(a, w.dtype) for a in x.A], [to_device(a, w.dtype) for a in x.Gout], Wd, mask, 0)
    print("checked masked", g.norms(), flush=True)
    g.close()

    # the entry point with static scratch
    w = W.scaled(W.get("mlp4x1024"), n_layers=1, B=2, T=96)
    x = W.make_step_inputs(w, 0)
    out = torch.empty(w.B, dtype=torch.float32, device="cuda")
    grape.grape_layer_sqnorms_static(to_device(x.A[0], w.dtype), to_device(x.Gout[0], w.dtype), 1024, 1024,
                                     w.r, w.B, w.T, w.seed, 0, 0, out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    print("checked static", out.cpu().numpy(), flush=True)
    print("ALL OK", flush=True)


if __name__ == "__main__":
    main()
