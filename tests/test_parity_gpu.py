"""Parity of the CUDA library with the fp64 oracle, through the C ABI (needs a B200)."""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W
from harness import compare, rel_fro, run_library, run_oracle, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeError, GrapeStep, grape  # noqa: E402

SIMT, TC = grape.GRAPE_PATH_SIMT, grape.GRAPE_PATH_TC

# ---------------------------------------------------------------------------------
# the generator
# ---------------------------------------------------------------------------------


@pytest.mark.parametrize("seed,layer,step,stream", [(0, 0, 0, 0), (1, 3, 7, 1),
                                                     (0x0123456789ABCDEF, 27, 12345, 0),
                                                     (2**64 - 1, 2**32 - 1, 2**31, 1)])
def test_philox_words_bit_exact(seed, layer, step, stream):
    n = 100_003
    out = torch.empty(4 * n, dtype=torch.int32, device="cuda")
    grape.grape_philox_words(seed, layer, step, stream, n, out)
    got = out.cpu().numpy().view(np.uint32).reshape(n, 4)
    ref = O.philox_words(seed, layer, step, stream, n)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("n", [1, 3, 4, 4097, 1 << 20])
def test_gaussian_matches_oracle(n):
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    grape.grape_gaussian(42, 5, 9, 1, n, out)
    got = out.cpu().numpy().astype(np.float64)
    ref = O.gaussian_stream(42, 5, 9, 1, n)
    # fp32 log / sqrt / sincospi of the same words: a few fp32 ulps of |z| <= 6.7
    assert np.max(np.abs(got - ref)) < 2e-5
    assert rel_fro(got, ref) < 1e-6


@pytest.mark.parametrize("layers,r,step", [(((256, 512), (520, 256)), 128, 0),
                                           (((648, 512), (1024, 256)), 512, 3)],
                         ids=["r128", "r512_step3"])
def test_bf16_projection_matches_oracle_element_by_element(layers, r, step):
    """The tensor-core path draws P_l in bf16 with the special-function unit's log and
    sine/cosine.  Each element must be the oracle's fp64 N(0, 1/r) value of the same
    Philox words, up to bf16 rounding (2^-8 of |P|, a bound on the half ulp) plus the
    intrinsics' error: at most about 1e-3 in z (the log's absolute error near u1 = 1
    under the square root), so 1e-3 / sqrt(r) in P.  A wrong stream, layer, step or
    element index, a swapped cosine and sine or a flipped sign misses this by orders of
    magnitude."""
    w = W.Workload("p_bf16", layers, r=r, B=2, T=16, dtype="bf16", C=1.0, sigma=0.5,
                   steps=step + 1)
    g = GrapeStep.for_workload(w, path=TC)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, step)
    g.step([to_device(a, w.dtype) for a in x.A], [to_device(a, w.dtype) for a in x.Gout], Ws, step)
    torch.cuda.synchronize()
    h = O.Hyper.of(w)
    for l, (d_in, _) in enumerate(layers):
        got = g.P(l).astype(np.float64)
        ref = O.projection_matrix(h.seed, l, h.projection_key(step), d_in, r)
        bound = 2.0**-8 * np.abs(ref) + 1.01e-3 / np.sqrt(r)
        err = np.abs(got - ref)
        print(l, f"max err / bound {np.max(err / bound):.3f}, rel fro {rel_fro(got, ref):.2e}")
        assert np.all(err <= bound), (l, np.unravel_index(np.argmax(err / bound), err.shape))
        assert rel_fro(got, ref) < 2.0**-8
    g.close()


# ---------------------------------------------------------------------------------
# full steps against the oracle
# ---------------------------------------------------------------------------------

CASES = {
    # name: (workload, steps)
    "tiny_f32": (W.get("tiny_f32"), 3),
    # MLP layers at reduced batch: several 64/128 tiles
    "mlp_2x1024_B4": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=4), 3),
    # ViT shapes with the ragged T = 197 and d_out = 2304, 768
    "vit_qkv_down_B3": (W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768)), B=3), 2),
    # sparse loss tokens, C = 0.5, T = 1000 (ragged)
    "longctx_1layer_T1000": (W.scaled(W.get("longctx"), layers=((2048, 2048),), B=2, T=1000), 2),
    # r = 512 (two 256-wide N tiles, four 128-row M tiles), ragged T
    "r512_T130": (W.Workload("r512", ((1024, 2816), (2816, 1024)), r=512, B=2, T=130,
                             dtype="bf16", C=1.0, sigma=0.6, steps=2), 2),
    # more layers than one launch group holds (16)
    "20_layers": (W.Workload("twenty", tuple([(256, 256), (512, 256)] * 10), r=128, B=3, T=64,
                             dtype="bf16", C=1.0, sigma=1.0, steps=2), 2),
    # degenerate shapes (CUDA-core path only: r not a multiple of 128)
    "T1_B1": (W.Workload("T1_B1", ((96, 40),), r=16, B=1, T=1, dtype="bf16", C=1.0,
                         sigma=0.5, steps=2), 2),
    "r_equals_d_in": (W.Workload("r_eq_din", ((64, 32), (64, 48)), r=64, B=3, T=9,
                                 dtype="f32", C=1.0, sigma=1.0, steps=2), 2),
    "odd_sizes": (W.Workload("odd", ((37, 19), (53, 7)), r=5, B=5, T=13, dtype="f32",
                             C=0.7, sigma=0.3, steps=2), 2),
    "no_noise": (W.scaled(W.get("tiny_f32"), sigma=0.0), 3),
    "no_noise_bf16": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=4, T=64, sigma=0.0), 2),
    "T1_bf16_tc": (W.Workload("T1_tc", ((256, 256),), r=128, B=5, T=1, dtype="bf16", C=1.0,
                              sigma=0.5, steps=2), 2),
    # tensor-core path with d_in off the 64-wide k-block and the 128-row back-projection
    # tile (d_in % 8 == 0 is all it needs): a ragged last k-block in the projection and a
    # ragged last M tile of W, both at the edge of their TMA boxes
    "ragged_d_in_tc": (W.Workload("ragged_din", ((520, 256), (136, 512)), r=128, B=3, T=40,
                                  dtype="bf16", C=1.0, sigma=0.8, steps=2), 2),
    # the norm kernel's one 256-column block of (A_i P)^T in TMEM (T in 257..512): eight
    # 64-token chunks, the last one ragged, r = 256 (groups of two CTAs)
    "r256_T500": (W.Workload("r256_T500", ((512, 768), (768, 512)), r=256, B=3, T=500,
                             dtype="bf16", C=1.0, sigma=0.7, steps=2), 2),
    # r = 512 (the back-projection with P in TMEM) with d_in off the 128-row block: the
    # last block of P is partly past d_in (8 of its 128 rows)
    "r512_ragged_d_in": (W.Workload("r512_ragged", ((520, 256), (648, 512)), r=512, B=2, T=40,
                                    dtype="bf16", C=1.0, sigma=0.8, steps=2), 2),
    # the per-layer shape of the 7B-slice workload at small widths: r = 512, T = 512
    "r512_T512": (W.Workload("r512_T512", ((512, 1024), (1024, 512)), r=512, B=2, T=512,
                             dtype="bf16", C=1.0, sigma=1.0, steps=2), 2),
}


def _tc_ok(w):
    return (w.dtype == "bf16" and w.r % 128 == 0 and (w.r <= 256 or w.r % 256 == 0)
            and all(di % 8 == 0 and do % 256 == 0 for di, do in w.layers))


def _tol(w, path):
    if w.dtype == "f32":
        return 1e-5
    return 1e-4 if path == SIMT else 2e-2


PAIRS = [(c, SIMT) for c in sorted(CASES)] + [(c, TC) for c in sorted(CASES) if _tc_ok(CASES[c][0])]


@pytest.mark.parametrize("case,path", PAIRS, ids=[f"{c}-{'tc' if p == TC else 'simt'}" for c, p in PAIRS])
def test_step_matches_oracle(case, path):
    w, steps = CASES[case]
    lib = run_library(w, steps, path)
    assert lib["path"] == path
    orc = run_oracle(w, steps)
    worst = compare(w, lib, orc, _tol(w, path), steps)
    print(case, "tc" if path == TC else "simt", {k: f"{v:.2e}" for k, v in worst.items()})


STORE_CASES = ["mlp_2x1024_B4", "vit_qkv_down_B3", "longctx_1layer_T1000", "r512_T130", "20_layers",
               "ragged_d_in_tc", "T1_bf16_tc", "no_noise_bf16", "r256_T500", "r512_T512"]


@pytest.mark.parametrize("case", STORE_CASES)
@pytest.mark.parametrize("agg", [grape.GRAPE_AGG_STORE, grape.GRAPE_AGG_RECOMPUTE], ids=["store", "recompute"])
def test_aggregation_methods_match_oracle(case, agg):
    """Both aggregations, forced whatever GRAPE_AGG_AUTO would pick for the shape: S from
    the R_i the norm kernel stored (bf16), and S from the second contraction over the
    stacked rows, each against the oracle's sum of the clipped R_i."""
    w, steps = CASES[case]
    lib = run_library(w, steps, TC, setup=lambda g: g.set_aggregation(agg))
    orc = run_oracle(w, steps)
    worst = compare(w, lib, orc, 2e-2, steps)
    print(case, "store" if agg == grape.GRAPE_AGG_STORE else "recompute",
          {k: f"{v:.2e}" for k, v in worst.items()})


# (the TMEM norm kernel takes T <= 512 and only with the stored aggregation)
TMEM_NORM_CASES = ["T1_bf16_tc", "r512_T130", "vit_qkv_down_B3", "20_layers", "ragged_d_in_tc", "r256_T500"]


@pytest.mark.parametrize("case", TMEM_NORM_CASES)
def test_both_norm_kernels_match_oracle_and_each_other(case, monkeypatch):
    """With the stored aggregation the norms run on the kernel that keeps (A_i P)^T in
    TMEM for 256 < T <= 512 and on the streamed kernel otherwise.  GRAPE_NORM_TMEM=1 and
    =0 force one or the other for every T up to 512: T = 1, a ragged last 64-token chunk,
    more layers than one launch holds, r = 128 / 256 / 512.  Each against the oracle,
    and against each other: the same bf16 products summed in fp32 in another order, so
    the norms and the S built from the stored R_i agree far inside the parity
    tolerance."""
    w, steps = CASES[case]
    store = lambda g: g.set_aggregation(grape.GRAPE_AGG_STORE)   # noqa: E731
    runs = {}
    for mode in ("0", "1"):
        monkeypatch.setenv("GRAPE_NORM_TMEM", mode)
        runs[mode] = run_library(w, steps, TC, setup=store)
    monkeypatch.delenv("GRAPE_NORM_TMEM")
    orc = run_oracle(w, steps)
    for mode, lib in runs.items():
        worst = compare(w, lib, orc, 2e-2, steps)
        print(case, "tmem" if mode == "1" else "streamed", {k: f"{v:.2e}" for k, v in worst.items()})
    for t in range(steps):
        a, b = runs["0"]["trace"][t], runs["1"]["trace"][t]
        assert rel_fro(a["norms"], b["norms"]) < 1e-4, t
        for l in range(w.n_layers):
            assert rel_fro(a["S"][l], b["S"][l]) < 1e-3, (t, l)


@pytest.mark.parametrize("case", ["r512_T130", "vit_qkv_down_B3", "r256_T500"])
def test_projection_kernels_give_the_same_bits(case, monkeypatch):
    """For r >= 256 the projection runs in 256-row tiles (two 128-row MMAs sharing each P
    stage); GRAPE_PROJECT_WIDE=0 keeps the 128-row tiles.  Every AP element is the same
    chain of 128 x 256 x 16 MMAs over the same k order either way, so the two give the
    same bits, through to W.  The cases have a last tile whose second half is past the
    stacked rows (r512_T130: 260 rows, vit_qkv_down_B3: 591)."""
    w, steps = CASES[case]
    monkeypatch.setenv("GRAPE_PROJECT_WIDE", "0")
    narrow = run_library(w, steps, TC)
    monkeypatch.delenv("GRAPE_PROJECT_WIDE")
    wide = run_library(w, steps, TC)
    for t in range(steps):
        assert np.array_equal(narrow["trace"][t]["norms"], wide["trace"][t]["norms"]), t
        for l in range(w.n_layers):
            assert np.array_equal(narrow["trace"][t]["S"][l], wide["trace"][t]["S"][l]), (t, l)
    for l in range(w.n_layers):
        assert np.array_equal(narrow["W"][l], wide["W"][l]), l


def test_auto_aggregation_follows_tokens_per_sample():
    """AUTO stores R_i from T = 256 tokens per sample on; the ghost norm forms no R_i and
    so recomputes; the CUDA-core path refuses STORE."""
    base = W.Workload("agg_auto", ((256, 256),), r=128, B=2, T=255, dtype="bf16", C=1.0,
                      sigma=1.0, steps=1)
    g = GrapeStep.for_workload(base, path=TC)
    assert g.aggregation == grape.GRAPE_AGG_RECOMPUTE
    g.close()
    g = GrapeStep.for_workload(base.replace(T=256), path=TC)
    assert g.aggregation == grape.GRAPE_AGG_STORE
    g.close()
    g = GrapeStep.for_workload(base.replace(T=64), path=TC)
    g.set_aggregation(grape.GRAPE_AGG_STORE)
    assert g.aggregation == grape.GRAPE_AGG_STORE
    g.set_norm_method(grape.GRAPE_NORM_GHOST)
    assert g.aggregation == grape.GRAPE_AGG_RECOMPUTE
    g.close()
    g = GrapeStep.for_workload(base, path=SIMT)
    with pytest.raises(GrapeError) as e:
        g.set_aggregation(grape.GRAPE_AGG_STORE)
    assert e.value.code == grape.GRAPE_EUNSUPPORTED
    g.close()


def test_bench_workload_full_size_tc():
    """The benchmarked workload (4 x 1024^2, r = 128, B = 64, T = 128) at full size on the
    tensor-core path, two steps, against the oracle on the whole batch."""
    w = W.get("mlp4x1024")
    lib = run_library(w, 2, TC)
    orc = run_oracle(w, 2)
    worst = compare(w, lib, orc, 2e-2, 2)
    print("mlp4x1024 full", {k: f"{v:.2e}" for k, v in worst.items()})


def test_auto_path_picks_tensor_cores_for_bf16():
    g = GrapeStep.for_workload(W.scaled(W.get("mlp4x1024"), n_layers=1, B=2, T=16))
    assert g.path == TC
    g.close()


def test_tiny_f32_matches_golden():
    """The fp32 workload against the stored oracle values (tests/golden)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_f32_oracle.json")))
    w = W.get("tiny_f32")
    lib = run_library(w, w.steps, grape.GRAPE_PATH_AUTO)
    assert lib["path"] == SIMT
    assert rel_fro(lib["W"][0], g["W"][0]) < 1e-5
    assert rel_fro(lib["trace"][-1]["m"][0], g["m"][0]) < 1e-5
    assert rel_fro(lib["trace"][-1]["v"][0], g["v"][0]) < 1e-5
    for s in range(w.steps):
        assert rel_fro(lib["trace"][s]["S"][0], g["steps"][s]["S"][0]) < 1e-5
        assert rel_fro(lib["trace"][s]["norms"], g["steps"][s]["norms"]) < 1e-5


# ---------------------------------------------------------------------------------
# properties of the library itself
# ---------------------------------------------------------------------------------

def _inputs(w, s):
    x = W.make_step_inputs(w, s)
    return [to_device(a, w.dtype) for a in x.A], [to_device(a, w.dtype) for a in x.Gout]


@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_bitwise_reproducible(path):
    """Fixed-order reductions: two runs of the same steps give identical bits."""
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=64)
    a = run_library(w, 2, path)
    b = run_library(w, 2, path)
    for l in range(w.n_layers):
        assert np.array_equal(a["W"][l], b["W"][l])
        assert np.array_equal(a["trace"][-1]["m"][l], b["trace"][-1]["m"][l])


@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_clipped_norm_bound(path):
    """Every clip factor brings the sample to norm <= C; unclipped samples keep 1."""
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=16, T=32)
    lib = run_library(w, 1, path)
    n, c = lib["trace"][0]["norms"], lib["trace"][0]["clip"]
    assert np.all(c * n <= w.C * (1 + 1e-6))
    assert np.all(c[n <= w.C] == 1.0)
    assert (c < 1).any() and (c == 1).any()


@pytest.mark.parametrize("path,agg", [(SIMT, None), (TC, None), (TC, grape.GRAPE_AGG_STORE)],
                         ids=["simt", "tc", "tc-stored"])
def test_accumulate_apply_equals_step(path, agg):
    """The data-parallel split gives the step's bits.  With the stored aggregation a step
    sums the R_i inside its noise + Adam kernel, and the split keeps the two apart: the
    same arithmetic in the same order."""
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=32)
    W0 = W.make_weights(w)
    g1, g2 = GrapeStep.for_workload(w, path=path), GrapeStep.for_workload(w, path=path)
    if agg is not None:
        g1.set_aggregation(agg)
        g2.set_aggregation(agg)
    W1 = [torch.from_numpy(x).cuda() for x in W0]
    W2 = [torch.from_numpy(x).cuda() for x in W0]
    for s in range(2):
        A, G = _inputs(w, s)
        g1.step(A, G, W1, s)
        g2.accumulate(A, G, s)
        g2.apply(W2, s)
    torch.cuda.synchronize()
    for l in range(w.n_layers):
        assert torch.equal(W1[l], W2[l])
        for f in ("S", "m", "v", "dR"):
            assert np.array_equal(getattr(g1, f)(l), getattr(g2, f)(l)), (f, l)


@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_apply_needs_the_accumulated_projection(path):
    """apply(s) back-projects with the P the aggregation of S used: it is refused before
    any accumulation, for a step of another key, and after sqnorms replaced P; W is left
    untouched by a refused call, and a step of the same refresh key is accepted."""
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=32)
    g = GrapeStep.for_workload(w, path=path)
    Wd = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    before = [x.clone() for x in Wd]
    A, G = _inputs(w, 0)
    with pytest.raises(GrapeError) as e:
        g.apply(Wd, 0)
    assert e.value.code == grape.GRAPE_EINVAL
    g.accumulate(A, G, 0)
    with pytest.raises(GrapeError):
        g.apply(Wd, 1)
    g.sqnorms(A, G, 1)                       # draws P of step 1 into the scratch
    with pytest.raises(GrapeError):
        g.apply(Wd, 0)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(Wd, before))
    g.accumulate(A, G, 0)
    g.apply(Wd, 0)                           # the matching pair runs
    g.set_refresh_period(2)
    g.accumulate(A, G, 2)
    g.apply(Wd, 3)                           # 2 // 2 == 3 // 2: the same P
    torch.cuda.synchronize()
    g.close()


@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_step_host_equals_step(path):
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=32)
    W0 = W.make_weights(w)
    g1, g2 = GrapeStep.for_workload(w, path=path), GrapeStep.for_workload(w, path=path)
    W1 = [torch.from_numpy(x).cuda() for x in W0]
    W2 = [torch.from_numpy(x).cuda() for x in W0]
    for s in range(2):
        x = W.make_step_inputs(w, s)
        A = [to_device(a, w.dtype) for a in x.A]
        G = [to_device(a, w.dtype) for a in x.Gout]
        g1.step(A, G, W1, s)
        hostA = [torch.from_numpy(a.view(np.int16)).pin_memory() for a in x.A]
        hostG = [torch.from_numpy(a.view(np.int16)).pin_memory() for a in x.Gout]
        norms = np.zeros(w.B, dtype=np.float32)
        g2.step_host(hostA, hostG, W2, s, norms)
        assert np.array_equal(norms, g1.norms())
    torch.cuda.synchronize()
    for l in range(w.n_layers):
        assert torch.equal(W1[l], W2[l])


@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_checkpoint_resume_bitwise(path):
    """Stop after step 1, move m and v to a fresh context, continue: identical W.
    P is not state (it is regenerated from seed, layer and step)."""
    w = W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=32)
    W0 = W.make_weights(w)
    ref = GrapeStep.for_workload(w, path=path)
    Wr = [torch.from_numpy(x).cuda() for x in W0]
    for s in range(3):
        A, G = _inputs(w, s)
        ref.step(A, G, Wr, s)
    first = GrapeStep.for_workload(w, path=path)
    Wc = [torch.from_numpy(x).cuda() for x in W0]
    for s in range(2):
        A, G = _inputs(w, s)
        first.step(A, G, Wc, s)
    saved = []
    for l, (di, do) in enumerate(w.layers):
        m = torch.empty(w.r, do, device="cuda")
        v = torch.empty(w.r, do, device="cuda")
        first.get_state(l, m, v)
        saved.append((m, v))
    first.close()
    second = GrapeStep.for_workload(w, path=path)
    for l, (m, v) in enumerate(saved):
        second.set_state(l, m, v)
    A, G = _inputs(w, 2)
    second.step(A, G, Wc, 2)
    torch.cuda.synchronize()
    for l in range(w.n_layers):
        assert torch.equal(Wr[l], Wc[l])


def test_moment_memory_is_projected():
    """Optimizer state is O(r x layers): the context holds far less than 2 x 4 bytes x W."""
    w = W.get("mlp4x1024")
    g = GrapeStep.for_workload(w, path=SIMT)
    full_adam = sum(2 * 4 * di * do for di, do in w.layers)
    moments = sum(2 * 4 * w.r * do for _, do in w.layers)
    assert moments * 8 == full_adam         # r = d/8 here
    assert g.device_bytes() < full_adam     # moments plus the whole workspace
    g.close()


@pytest.mark.parametrize("case", ["mlp_tc", "mlp_simt", "tiny_f32", "vit_tc", "r512_two_groups"])
def test_device_bytes_equal_the_host_plan(case):
    """grape_context_bytes, computed on the host, is what grape_create allocates, including
    the projection's tile schedules (r >= 256; one per launch group of 16 layers)."""
    w, path = {"mlp_tc": (W.get("mlp4x1024"), TC), "mlp_simt": (W.get("mlp4x1024"), SIMT),
               "tiny_f32": (W.get("tiny_f32"), SIMT),
               "vit_tc": (W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768)), B=3), TC),
               "r512_two_groups": (W.Workload("r512_18", tuple([(512, 256), (1024, 512)] * 9), r=512, B=2,
                                              T=300, dtype="bf16", C=1.0, sigma=1.0, steps=1), TC)}[case]
    g = GrapeStep.for_workload(w, path=path)
    dt = grape.GRAPE_BF16 if w.dtype == "bf16" else grape.GRAPE_F32
    assert g.device_bytes() == grape.grape_context_bytes(w.layers, w.r, w.B, w.T, dt, path)
    g.close()


def test_errors_are_reported():
    w = W.get("tiny_f32")
    g = GrapeStep.for_workload(w)
    x = W.make_step_inputs(w, 0)
    A = [to_device(a, "f32") for a in x.A]
    G = [to_device(a, "f32") for a in x.Gout]
    Wt = [torch.zeros(64, 32, device="cuda")]
    with pytest.raises(GrapeError) as e:
        g.step([A[0].data_ptr() + 4], G, Wt, 0)      # misaligned
    assert e.value.code == grape.GRAPE_EINVAL
    with pytest.raises(GrapeError) as e:
        g.step(A, G, Wt, -1)
    assert e.value.code == grape.GRAPE_EINVAL
    g.step(A, G, Wt, 0)                              # still usable afterwards
    torch.cuda.synchronize()
    g.close()


def test_allocation_failure_is_reported(monkeypatch):
    monkeypatch.setenv("GRAPE_FAULT_ALLOC", "1")
    with pytest.raises(GrapeError) as e:
        GrapeStep.for_workload(W.get("tiny_f32"))
    assert e.value.code == grape.GRAPE_ENOMEM


@pytest.mark.parametrize("path", [SIMT, TC])
def test_S_all_is_every_layer_back_to_back(path):
    w = W.scaled(W.get("mlp4x1024"), layers=((1024, 1024), (1024, 512 * 2), (768, 2304)), B=2, T=32)
    if path == SIMT:
        w = w.replace(layers=((24, 16), (16, 12), (12, 20)), r=8, dtype="f32")
    g = GrapeStep.for_workload(w, path=path)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0, threads=8)
    g.accumulate([to_device(a, w.dtype) for a in x.A], [to_device(a, w.dtype) for a in x.Gout], 0)
    torch.cuda.synchronize()
    flat = g.S_all_tensor().cpu().numpy()
    at = 0
    for l, (_, do) in enumerate(w.layers):
        n = w.r * do
        assert np.array_equal(flat[at:at + n].reshape(w.r, do), g.S(l)), l
        at += n
    assert at == flat.size
    g.close()
