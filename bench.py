#!/usr/bin/env python
"""Throughput of the DP-GRAPE step on one node.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (default): the largest single-GPU configuration, a 7B-LLM-shaped slice of four
decoder blocks (per block Q, K, V, O 4096 x 4096, gate and up 4096 x 11008, down
11008 x 4096: 28 linear layers), r = 512, B = 16 samples of T = 512 tokens, bf16 A and
Gout, fp32 W and Adam moments (``workloads`` name ``llm7b_slice``; ``--workload`` picks
another).  A "step" is one full pass of the method over one batch:
regenerate P, project, per-sample norms, clip, aggregate, noise + projected
Adam, back-projection onto W.  Inputs are synthetic (seeded, see ``workloads``)
and rotate over several distinct per-step sets whose total is far larger than
the 126 MB L2, each set alone already larger than L2.

Prints one JSON line (rank 0).  With N > 1 (launched by torch.distributed.run)
every rank runs its own B samples (weak scaling); every layer's S, back to back in
one buffer, is summed over the ranks by a single NCCL all-reduce between the
aggregation and Adam.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "DP-GRAPE step samples/s (tokens/s) on 1 B200; % of tensor-pipe/HBM roofline"
# --mode sqnorms: the Hutchinson per-sample gradient-norm estimate alone (grape_sqnorms)
METRIC_SQNORMS = ("Hutchinson per-sample gradient-norm estimates/s (samples/s) on 1 B200; "
                  "% of tensor-pipe/HBM roofline")
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INPUT_SETS = 4          # distinct per-step input sets (2 when one set exceeds 1 GB)
L2_BYTES = 126 * 1000 * 1000


def layer_summary(w) -> str:
    """'4x1024x1024' for a uniform stack, else the count and the distinct shapes."""
    shapes = sorted(set(w.layers), key=w.layers.index)
    if len(shapes) == 1:
        return f"{w.n_layers}x{shapes[0][0]}x{shapes[0][1]}"
    return f"{w.n_layers} layers of " + ", ".join(f"{a}x{b}" for a, b in shapes)



def workload_of(args):
    """The workload the arguments name, reduced by --layers / --batch if given (its name
    then records the reduction)."""
    w = WL.get(args.workload)
    if args.layers or args.batch:
        kw = {}
        if args.layers:
            kw["n_layers"] = args.layers
        if args.batch:
            kw["B"] = args.batch
        w = WL.scaled(w, **kw)
        w = w.replace(name=f"{w.name}[{w.n_layers} layers, B={w.B}]")
    return w


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llm7b_slice", choices=sorted(WL.WORKLOADS))
    ap.add_argument("--mode", default="step", choices=["step", "sqnorms"],
                    help="step: the whole DP-GRAPE step; sqnorms: per-sample norm estimates only")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel of grape_step from the host instead of replaying a "
                         "CUDA graph of the step (grape_set_graph)")
    ap.add_argument("--norm", default="direct", choices=["direct", "ghost"],
                    help="per-sample norms by R_i tiles (direct) or by the ghost Gram identity")
    ap.add_argument("--agg", default="auto", choices=["auto", "recompute", "store"],
                    help="aggregation S = sum_i c_i R_i: a second contraction over the stacked rows "
                         "(recompute), a weighted sum of the R_i the norm kernel stored (store), or "
                         "the library's choice by tokens per sample (auto)")
    ap.add_argument("--mask-capacity", type=int, default=0,
                    help="run masked steps (grape_step_masked) keeping at most this many loss "
                         "tokens per sample; the workload's own token mask is passed in")
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--layers", type=int, default=0,
                    help="keep only the workload's first N layers (a reduced case for profiling)")
    ap.add_argument("--batch", type=int, default=0,
                    help="samples per batch instead of the workload's B (a reduced case for profiling)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------------------
# clocks during the timed region (NVML, polled from a thread)
# ---------------------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.nv, self.err = None, str(e)

    def _poll(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.005)

    def sample(self):
        if not self.nv:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in self.REASONS.items():
                if mask & bit:
                    self.reasons.add(name)
        except Exception:  # noqa: BLE001
            pass

    def __enter__(self):
        self.t = threading.Thread(target=self._poll, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self.t.join()
        self.sample()

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvml unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------
# roofline bookkeeping
# ---------------------------------------------------------------------------------------

def peaks():
    try:
        p = json.load(open(PEAKS_FILE))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:  # noqa: BLE001
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0, "source": "fallback"}


def phase_work(w, path: str, agg: str = "recompute"):
    """Algorithmic bytes and flops of one launch of each phase (all layers in one call).

    Bytes count each operand once at its storage width: the minimum traffic of that phase.
    With the stored aggregation (``agg`` "store") the norm phase also writes every R_i
    (bf16, B r d_out per layer) and the aggregation reads them back once: a pass over
    memory with no contraction.
    """
    el = 4 if w.dtype == "f32" else 2
    ap_el = 4 if path == "simt" else 2
    dr_el = 4 if path == "simt" else 2
    p_el = 4 if path == "simt" else 2          # fp32 P on the CUDA cores, bf16 on the tensor path
    rows = w.B * w.T
    out = {}
    out["gen_P"] = {"bytes": sum(di * w.r * p_el for di, _ in w.layers), "flops": 0}
    out["project"] = {"bytes": sum(rows * di * el + rows * w.r * ap_el for di, _ in w.layers),
                      "flops": sum(2 * rows * di * w.r for di, _ in w.layers)}
    out["norm"] = {"bytes": sum(rows * do * el + rows * w.r * ap_el for _, do in w.layers),
                   "flops": sum(2 * rows * w.r * do for _, do in w.layers)}
    out["clip"] = {"bytes": 8 * w.B, "flops": 0}
    out["aggregate"] = {"bytes": sum(rows * do * el + rows * w.r * ap_el + 4 * w.r * do
                                     for _, do in w.layers),
                        "flops": sum(2 * rows * w.r * do for _, do in w.layers)}
    out["adam"] = {"bytes": sum(w.r * do * (4 + 16 + dr_el) for _, do in w.layers), "flops": 0}
    if agg == "store":
        r_bytes = sum(2 * w.B * w.r * do for _, do in w.layers)
        out["norm"]["bytes"] += r_bytes
        out["aggregate"] = {"bytes": r_bytes + sum(4 * w.r * do for _, do in w.layers), "flops": 0}
        # a one-process step sums the R_i inside noise + Adam: R_i read, S written (kept
        # for inspection), m and v read and written, dR written; S is not read back
        out["aggregate_adam"] = {"bytes": r_bytes + sum(w.r * do * (4 + 16 + dr_el) for _, do in w.layers),
                                 "flops": 0}
    out["backproject"] = {"bytes": sum(8 * di * do + di * w.r * ap_el + w.r * do * dr_el
                                       for di, do in w.layers),
                          "flops": sum(2 * di * w.r * do for di, do in w.layers)}
    # live-token compaction (--mask-capacity): scan the mask, read and write the kept rows
    out["compact"] = {"bytes": w.B * w.T + sum(2 * rows * (di + do) * el for di, do in w.layers),
                      "flops": 0}
    return out


def phase_roofline(work, seconds: float, pk, path: str) -> dict:
    """The roofline of one phase's launch: the bound its algorithmic work puts nearest
    (dense bf16 tensor FLOPs at the sustained measured peak, since the phases are timed
    inside a seconds-long run of steps, or bytes at the measured HBM copy bandwidth) and
    what the measured time achieves against it.  The CUDA-core path is bound by fp32 FFMA
    issue: 148 SMs x 128 lanes x 2 flop x the maximum SM clock."""
    if path != "tc":
        peak = 148 * 128 * 2 * pk["sm_max_mhz"] * 1e6 / 1e12
        achieved = work["flops"] / seconds / 1e12
        return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x max SM clock"}
    t_tc = work["flops"] / (pk["bf16_tflops_sustained"] * 1e12)
    t_hbm = work["bytes"] / (pk["hbm_gbs"] * 1e9)
    if t_tc > t_hbm:
        achieved = work["flops"] / seconds / 1e12
        peak = pk["bf16_tflops_sustained"]
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": f"{pk['source']} sustained dense bf16"}
    achieved = work["bytes"] / seconds / 1e9
    peak = pk["hbm_gbs"]
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": f"{pk['source']} HBM copy"}


def sqnorms_work(w):
    """Work of the norm estimate alone: FLOPs of AP = A P and of the per-sample
    (A_i P)^T Gout_i, bytes of A and Gout read once and of the B outputs."""
    el = 4 if w.dtype == "f32" else 2
    flops = sum(2 * w.B * w.T * w.r * (di + do) for di, do in w.layers)
    byts = sum(w.B * w.T * (di + do) * el for di, do in w.layers) + 4 * w.B
    return flops, byts


def step_work(w):
    """The method's own work per step: FLOPs of the factored projection and back-projection,
    bytes of A and Gout read once, W read + written, m and v read + written."""
    el = 4 if w.dtype == "f32" else 2
    flops = sum(2 * w.B * w.T * w.r * (di + do) + 2 * di * w.r * do for di, do in w.layers)
    byts = sum(w.B * w.T * (di + do) * el + 8 * di * do + 16 * w.r * do for di, do in w.layers)
    return flops, byts


KERNEL_SOURCES = {"tc": ("tc.cu", "tc_ptx.cuh", "philox.cuh"), "simt": ("simt.cu", "philox.cuh")}


def kernel_source_sha(path: str) -> str:
    """Hash of the kernel sources' code (the path's .cu file and the device headers it
    includes): comments and blank lines stripped, so that a comment edit does not orphan
    counters taken from unchanged code."""
    import re
    csrc = os.path.join(ROOT, "random_gradient_projection_b200", "csrc")
    src = "\n".join(open(os.path.join(csrc, n)).read() for n in KERNEL_SOURCES[path])
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(l.rstrip() for l in src.splitlines() if l.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def traffic_for(kernel: str, workload: str, path: str, mode: str = "step"):
    try:
        t = json.load(open(TRAFFIC_FILE))
    except Exception:  # noqa: BLE001
        return None
    rec = t.get(f"{path}:{kernel}:{workload}" + ("" if mode == "step" else f":{mode}"))
    if not rec or rec.get("source_sha") != kernel_source_sha(path):
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------------------
# the oracle on the host cores (baseline arm and cpu_baseline)
# ---------------------------------------------------------------------------------------

def _oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def _oracle_call(O, w, st, h, s, nb, mode) -> float:
    """Seconds of one oracle step (or norm pass) over the first ``nb`` samples of step s's
    inputs; drawing the inputs is not timed."""
    x = WL.make_step_inputs(w, s, samples=list(range(nb)), threads=8)
    A = [x.as_f64(a) for a in x.A]
    G = [x.as_f64(g) for g in x.Gout]
    t0 = time.perf_counter()
    if mode == "sqnorms":
        O.sample_norms(A, G, s, h, [di for di, _ in w.layers])
    else:
        O.step(st, A, G, s, h)
    return time.perf_counter() - t0


def oracle_samples_per_s(w, target_s: float, max_steps: int = 1000, sub_batch=None, mode="step"):
    """Time the fp64 oracle, as it stands, on samples of the workload's batch.

    Each timed call is one oracle step over ``sub_batch`` samples; calls repeat until
    ``target_s`` of CPU work has been timed.  Without ``sub_batch`` a first call over one
    sample sizes the calls to about a third of the target each (at most the whole batch),
    so that a large workload still gives a bounded sample.  Input drawing is outside the
    timed calls.  Returns (samples/s, samples timed, seconds, threads, samples per call)."""
    import oracle.grape_oracle as O
    h = O.Hyper.of(w)
    st = O.State.init(WL.make_weights(w), w.r)
    done, spent, s = 0, 0.0, 0
    nb = sub_batch
    if nb is None:
        t1 = _oracle_call(O, w, st, h, s, 1, mode)
        spent, done, s = t1, 1, 1
        nb = max(1, min(w.B, int(target_s / 3.0 / max(t1, 1e-9))))
    # a target of 0 s means: exactly max_steps calls (the reference arm's warm-up)
    while (spent < target_s or target_s <= 0) and s < max_steps:
        spent += _oracle_call(O, w, st, h, s, nb, mode)
        done += nb
        s += 1
    return (done / spent if spent > 0 else 0.0), done, spent, _oracle_threads(), nb


def run_reference(args, rank: int, world: int):
    """--impl reference: the fp64 oracle timed on the host cores (rank 0 only).

    Each step is the oracle's step over the first ``sub`` samples of that step's batch,
    ``sub`` sized from one untimed single-sample call so that the whole run of
    warm-up and timed steps takes about two minutes (at most 4 samples per step)."""
    if rank != 0:
        return
    w = workload_of(args)
    import oracle.grape_oracle as O
    h = O.Hyper.of(w)
    t1 = _oracle_call(O, w, O.State.init(WL.make_weights(w), w.r), h, 0, 1, args.mode)
    per_step = 120.0 / max(1, args.steps + args.warmup)
    sub = max(1, min(w.B, 4, int(per_step / max(t1, 1e-9))))
    # warm-up calls (untimed), then K timed calls of a bounded sub-batch each
    oracle_samples_per_s(w, 0.0, max_steps=max(1, args.warmup), sub_batch=sub, mode=args.mode)
    st = O.State.init(WL.make_weights(w), w.r)
    times = [_oracle_call(O, w, st, h, s, sub, args.mode) for s in range(args.steps)]
    total = sum(times)
    value = sub * len(times) / total
    cores = _oracle_threads()
    sample = f"{sub} of {w.B} samples per step, all {w.n_layers} layers, fp64 numpy oracle"
    line = {
        "impl": "reference", "metric": METRIC if args.mode == "step" else METRIC_SQNORMS,
        "value": value, "unit": "samples/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "layers": layer_summary(w),
                   "r": w.r, "B": w.B, "T": w.T, "tokens_per_s": value * w.T},
        "cpu_baseline": {"value": value, "unit": "samples/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "samples/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

def main(argv=None):
    args = parse(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} needs {args.gpus} ranks, one per GPU, but {world} "
                         f"{'was' if world == 1 else 'were'} launched: run it under "
                         f"`python -m torch.distributed.run --nproc-per-node {args.gpus} ...`")
    assert args.warmup >= 3, "at least 3 warm-up steps"

    import torch
    import torch.distributed as dist
    from random_gradient_projection_b200 import GrapeStep, grape
    from random_gradient_projection_b200.data_parallel import dp_step

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    w = workload_of(args)
    path = {"auto": grape.GRAPE_PATH_AUTO, "simt": grape.GRAPE_PATH_SIMT,
            "tc": grape.GRAPE_PATH_TC}[args.path]
    masked = args.mask_capacity > 0
    if masked and (args.mode != "step" or world > 1):
        raise SystemExit("--mask-capacity runs the single-GPU step only")
    g = GrapeStep.for_workload(w.replace(T=args.mask_capacity) if masked else w, path=path)
    if masked:
        g.enable_compaction(w.T)
    if args.norm == "ghost":
        g.set_norm_method(grape.GRAPE_NORM_GHOST)
    g.set_aggregation({"auto": grape.GRAPE_AGG_AUTO, "recompute": grape.GRAPE_AGG_RECOMPUTE,
                       "store": grape.GRAPE_AGG_STORE}[args.agg])
    agg_name = "store" if g.aggregation == grape.GRAPE_AGG_STORE else "recompute"
    if not args.no_graph:
        g.set_graph(True)      # grape_step replays one CUDA graph per input set
    path_name = {grape.GRAPE_PATH_SIMT: "simt", grape.GRAPE_PATH_TC: "tc"}[g.path]
    Wd = [torch.from_numpy(x).to(dev) for x in WL.make_weights(w)]

    # distinct per-step input sets; ranks draw different samples (input seed only)
    win = w.replace(seed=w.seed + 7919 * rank)
    # (each set's graph is captured at its first step, so every set is first seen in the
    # warm-up: no capture falls in the timed region)
    n_sets = min(INPUT_SETS if w.input_bytes() < (1 << 30) else 2, args.warmup)
    sets = []
    for k in range(n_sets):
        x = WL.make_step_inputs(win, k, threads=16)
        conv = (lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)) \
            if w.dtype == "bf16" else torch.from_numpy
        sets.append(([conv(a).to(dev) for a in x.A], [conv(a).to(dev) for a in x.Gout],
                     torch.from_numpy((x.mask != 0).astype(np.uint8)).to(dev)))
    set_bytes = w.input_bytes()

    sq_out = torch.empty(w.B, dtype=torch.float32, device=dev)
    # the plain step over each input set, its buffers checked and marshalled once
    bound = [g.bind(A, G, Wd, torch.cuda.current_stream()) for A, G, _ in sets]

    def one(s):
        A, G, M = sets[s % n_sets]
        if masked:
            g.step_masked(A, G, Wd, M, s)
        elif args.mode == "sqnorms":
            g.sqnorms(A, G, s, out=sq_out)     # per-sample estimates only (no exchange needed)
        elif world > 1:
            dp_step(g, A, G, Wd, s)
        else:
            bound[s % n_sets].step(s)

    def barrier():
        if world > 1:
            dist.barrier()

    step = 0
    for _ in range(args.warmup):
        one(step)
        step += 1
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps --------------------------------------------------
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = g.launch_count()
    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    with sampler:
        e0.record(stream)
        for _ in range(args.steps):
            one(step)
            step += 1
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    launches = g.launch_count() - launches0
    ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_per_step = ms / args.steps
    samples_per_s = world * w.B * args.steps / (ms / 1e3)

    # ---- the same steps from a cold L2: a 256 MB write before each step, each step timed
    # alone with events (the write is outside the timed intervals) ------------------------
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    cold_ms = 0.0
    n_cold = min(args.steps, 50)
    for _ in range(n_cold):
        flush.fill_(step & 0xFF)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        one(step)
        c1.record(stream)
        step += 1
        torch.cuda.synchronize()
        cold_ms += c0.elapsed_time(c1)
    if world > 1:
        t = torch.tensor([cold_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        cold_ms = float(t.item())
    del flush

    # ---- per-phase device time (same K steps, events between phases) --------------------
    g.profile(True)
    for _ in range(args.steps):
        one(step)
        step += 1
    phases = g.profile_read()
    g.profile(False)

    pk = peaks()
    w_run = w.replace(T=args.mask_capacity) if masked else w   # rows the GEMM phases see
    work = phase_work(w_run, path_name, agg_name)
    if masked:
        work["compact"]["bytes"] = w.B * w.T + (work["compact"]["bytes"] - w_run.B * w_run.T)
    per_phase = {}
    for name, (pms, calls) in phases.items():
        if calls == 0:
            continue
        avg_s = pms / calls / 1e3
        per_phase[name] = {"ms_per_launch": pms / calls, "share": None,
                           "GB/s": work[name]["bytes"] / avg_s / 1e9,
                           "TFLOP/s": work[name]["flops"] / avg_s / 1e12}
    tot = sum(v["ms_per_launch"] for v in per_phase.values())
    for v in per_phase.values():
        v["share"] = v["ms_per_launch"] / tot if tot > 0 else None
    for name, v in per_phase.items():
        v["roofline"] = phase_roofline(work[name], v["ms_per_launch"] / 1e3, pk, path_name)
    dom = max(per_phase, key=lambda k: per_phase[k]["ms_per_launch"])
    dom_roof = per_phase[dom]["roofline"]
    traffic = traffic_for(dom, w.name, path_name, args.mode)
    if masked:
        # the live-token lower bound: the method's work over the kept tokens only
        kept = float(np.mean([m.float().sum(dim=1).mean().item() for _, _, m in sets]))
        flops, byts = step_work(w.replace(T=max(1, int(round(kept)))))
    else:
        flops, byts = step_work(w) if args.mode == "step" else sqnorms_work(w)
    t_roof = max(flops / (pk["bf16_tflops_sustained"] * 1e12), byts / (pk["hbm_gbs"] * 1e9))

    # ---- end to end through the public API: host buffers, copies in the timed region ----
    e2e = None
    if args.e2e_steps > 0:
        x = WL.make_step_inputs(win, 0, threads=16)
        hostA = [torch.from_numpy(a.view(np.int16) if w.dtype == "bf16" else a).pin_memory()
                 for a in x.A]
        hostG = [torch.from_numpy(a.view(np.int16) if w.dtype == "bf16" else a).pin_memory()
                 for a in x.Gout]
        norms = torch.empty(w.B, dtype=torch.float32).pin_memory()
        if masked:
            dA, dG, dM = sets[0]
            hostM = torch.from_numpy((x.mask != 0).astype(np.uint8)).pin_memory()

            def e2e_one(s):
                for d, h_ in zip(dA, hostA):
                    d.view(torch.int16 if w.dtype == "bf16" else d.dtype).copy_(h_, non_blocking=True)
                for d, h_ in zip(dG, hostG):
                    d.view(torch.int16 if w.dtype == "bf16" else d.dtype).copy_(h_, non_blocking=True)
                dM.copy_(hostM, non_blocking=True)
                g.step_masked(dA, dG, Wd, dM, s)
                g.norms()                          # synchronises and reads the B norms back
        elif args.mode == "sqnorms":
            # public call with device buffers: copy the step's inputs in, estimate, copy out
            dA, dG, _ = sets[0]

            def e2e_one(s):
                for d, h_ in zip(dA, hostA):
                    d.view(torch.int16 if w.dtype == "bf16" else d.dtype).copy_(h_, non_blocking=True)
                for d, h_ in zip(dG, hostG):
                    d.view(torch.int16 if w.dtype == "bf16" else d.dtype).copy_(h_, non_blocking=True)
                g.sqnorms(dA, dG, s, out=sq_out)
                norms.copy_(sq_out, non_blocking=True)
                torch.cuda.current_stream().synchronize()
        elif world > 1:
            # the data-parallel step: this rank's inputs copied in, dp_step (with its
            # all-reduce), the norms read back
            dA, dG, _ = sets[0]

            def e2e_one(s):
                for d, h_ in zip(dA, hostA):
                    d.view(torch.int16 if w.dtype == "bf16" else d.dtype).copy_(h_, non_blocking=True)
                for d, h_ in zip(dG, hostG):
                    d.view(torch.int16 if w.dtype == "bf16" else d.dtype).copy_(h_, non_blocking=True)
                dp_step(g, dA, dG, Wd, s)
                g.norms()                          # synchronises and reads the B norms back
        else:
            def e2e_one(s):
                g.step_host(hostA, hostG, Wd, s, norms)   # synchronises its stream
        e2e_one(step)    # first call allocates the staging
        step += 1
        barrier()
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            e2e_one(step)
            step += 1
        el = time.perf_counter() - t0
        if world > 1:
            t = torch.tensor([el], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            el = float(t.item())
        e2e = {"value": world * w.B * args.e2e_steps / el, "unit": "samples/s",
               "h2d_bytes_per_step": set_bytes + (w.B * w.T if masked else 0), "d2h_bytes_per_step": 4 * w.B,
               "steps": args.e2e_steps,
               "note": ("pinned host A/Gout and the token mask copied in, grape_step_masked, the B "
                        "norms copied out, every step") if masked else
                       ("pinned host A/Gout copied in on every rank, dp_step (accumulate, one "
                        "all-reduce of S, apply), the B norms copied out, every step")
                       if world > 1 and args.mode == "step" else
                       ("grape_step_host: pinned host A/Gout copied in, per-sample norms copied out, "
                        "every step") if args.mode == "step" else
                       ("pinned host A/Gout copied in, grape_sqnorms, the B estimates copied out, "
                        "every step")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, secs, cores, nb = oracle_samples_per_s(w, args.cpu_seconds, mode=args.mode)
        cpu = {"value": v, "unit": "samples/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} samples of {w.name} (oracle steps over {nb} of its B={w.B} "
                         f"samples, after one over a single sample), {secs:.1f} s of fp64 numpy "
                         f"oracle time; every oracle step also draws each layer's P and noise "
                         f"in numpy, a cost per step that a sample of few samples does not "
                         f"spread"}

    if rank == 0:
        line = {
            "metric": METRIC if args.mode == "step" else METRIC_SQNORMS,
            "value": samples_per_s, "unit": "samples/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "layers": layer_summary(w),
                       "r": w.r, "B_per_gpu": w.B, "global_batch": w.B * world, "T": w.T,
                       "path": path_name, "parallelism": f"dp{world}", "mode": args.mode,
                       "mask_capacity": args.mask_capacity or None, "norm": args.norm,
                       "aggregation": agg_name if args.mode == "step" else None,
                       "cuda_graph": (not args.no_graph) and args.mode == "step" and not masked and world == 1,
                       "l2": (f"inputs rotate over {n_sets} distinct sets of "
                              f"{set_bytes / 1e6:.0f} MB each (> 126 MB L2)")
                             if set_bytes > L2_BYTES else
                             (f"inputs ({n_sets} sets of {set_bytes / 1e6:.3f} MB) fit in L2; "
                              "cold_l2 times steps after a 256 MB write"),
                       "tokens_per_s": samples_per_s * w.T,
                       "cold_l2": {"ms_per_step": cold_ms / n_cold,
                                   "value": world * w.B * n_cold / (cold_ms / 1e3),
                                   "how": f"{n_cold} steps, each after a 256 MB write, timed one by one"}},
            "roofline": {"bound": dom_roof["bound"], "kernel": dom, "achieved": dom_roof["achieved"],
                         "peak": dom_roof["peak"], "unit": dom_roof["unit"], "frac": dom_roof["frac"],
                         "traffic": traffic, "peak_source": dom_roof["peak_source"]},
            "step_roofline": {"t_roof_us": t_roof * 1e6, "frac": t_roof / (ms_per_step / 1e3),
                              "flops": flops, "bytes": byts,
                              "peaks": f"{pk['source']}: HBM copy and sustained dense bf16"},
            "phases": per_phase,
            "gpu_launches": launches,
            "clocks": sampler.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    g.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
