"""The C-ABI library loads and exports what include/grape.h declares (no GPU needed)."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "grape.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"GRAPE_API\s+[\w\s\*]*?\b(grape_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from random_gradient_projection_b200 import build, grape
    build.build()
    return grape.load()


def test_header_declares_the_boundary():
    names = declared()
    for must in ("grape_create", "grape_step", "grape_destroy", "grape_step_host",
                 "grape_accumulate", "grape_apply", "grape_get_state", "grape_set_state"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    from random_gradient_projection_b200 import grape
    out = subprocess.run(["nm", "-D", "--defined-only", grape.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(grape_\w+)$", out, flags=re.M))
    missing = [n for n in declared() if n not in exported]
    assert not missing, missing
    for n in declared():
        assert hasattr(lib, n)
    # the binding wraps exactly the declared set
    assert sorted(grape.EXPORTS) == declared()


@pytest.mark.parametrize("kw,msg", [
    (dict(layers=[(64, 32)], r=80), "r must be <= d_in"),
    (dict(layers=[], r=8), "n_layers"),
    (dict(layers=[(64, 32)], r=8, C=0.0), "C must be"),
    (dict(layers=[(64, 32)], r=8, sigma=-1.0), "sigma"),
    (dict(layers=[(64, 32)], r=8, B=0), "B and T"),
    (dict(layers=[(64, 32)], r=8, beta1=1.0), "adam"),
    (dict(layers=[(64, 32)], r=8, dtype=7), "in_dtype"),
    (dict(layers=[(64, 32)] * 65, r=8), "n_layers"),
    (dict(layers=[(64, 32)], r=8, B=1 << 16, T=1 << 14), "B*T too large"),
    (dict(layers=[(64, 0)], r=8), "d_in and d_out"),
    (dict(layers=[(64, 32)], r=0), "r must be >= 1"),
    (dict(layers=[(64, 32)], r=8, eps=0.0), "adam"),
    (dict(layers=[(64, 32)], r=8, path=3), "path"),
])
def test_create_validates_before_touching_the_device(lib, kw, msg):
    from random_gradient_projection_b200 import grape
    args = dict(layers=[(64, 32)], r=8, C=1.0, sigma=1.0, seed=0, lr=1e-3, beta1=0.9,
                beta2=0.999, eps=1e-8, B=4, T=16, dtype=grape.GRAPE_F32, path=0)
    args.update(kw)
    with pytest.raises(grape.GrapeError) as e:
        grape.grape_create(**args)
    assert e.value.code == grape.GRAPE_EINVAL
    assert msg in str(e.value)


def test_generator_entry_points_validate(lib):
    from random_gradient_projection_b200 import grape
    with pytest.raises(grape.GrapeError) as e:
        grape.grape_philox_words(0, 0, 0, 0, 16, 8, stream=0)   # misaligned output
    assert e.value.code == grape.GRAPE_EINVAL
    grape.grape_gaussian(0, 0, 0, 0, 0, 0, stream=0)              # empty request is a no-op


def test_refresh_and_sqnorms_validate_the_handle(lib):
    """Both reject a NULL handle on the host, before any device work."""
    assert lib.grape_set_refresh_period(None, 2) == 1          # GRAPE_EINVAL
    assert b"ctx" in lib.grape_global_error()
    assert lib.grape_sqnorms(None, None, None, 0, None, None) == 1


def test_selftest_validates_its_limits(lib):
    """Bad limits are refused on the host, before any device work."""
    assert lib.grape_selftest_wait_timeout(-1, 10, None) == 1          # GRAPE_EINVAL
    assert lib.grape_selftest_wait_timeout(10, 5, None) == 1
    assert lib.grape_selftest_wait_timeout(2_000_000_000, 3_000_000_000, None) == 1


def _header_constants():
    """Every GRAPE_* integer the header defines, by #define or in an enum."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    vals = {k: int(v) for k, v in re.findall(r"#define\s+(GRAPE_[A-Z0-9_]+)\s+(\d+)\b", src)}
    for body in re.findall(r"enum\s+\w+\s*\{(.*?)\}", src, flags=re.S):
        vals.update({k: int(v) for k, v in re.findall(r"(GRAPE_[A-Z0-9_]+)\s*=\s*(\d+)", body)})
    return vals


def test_binding_constants_equal_the_header():
    """grape.py restates the header's codes, paths, dtypes, debug items, norm methods and
    phase order; a drift would mislabel results without any error."""
    from random_gradient_projection_b200 import grape
    hdr = _header_constants()
    named = [k for k in hdr if hasattr(grape, k)]
    assert len(named) >= 20, named
    for k in named:
        assert getattr(grape, k) == hdr[k], k
    phases = sorted((v, k) for k, v in hdr.items() if k.startswith("GRAPE_PHASE_"))
    assert len(grape.PHASES) == hdr["GRAPE_N_PHASES"] == len(phases)
    short = {"GEN_P": "gen_P", "BACKPROJECT": "backproject"}
    for (v, k), name in zip(phases, grape.PHASES):
        tail = k[len("GRAPE_PHASE_"):]
        assert short.get(tail, tail.lower()) == name, (k, name)


def test_context_bytes_is_the_documented_arena(lib):
    """grape_context_bytes needs no device.  For the bench workload (4 x 1024^2, r = 128,
    B = 64, T = 128, bf16, tensor-core path), block by block, each rounded up to 256 B:
    every S_l 4 r sum(d_out) = 2 MiB; per layer P 2 d_in r = 256 KiB, AP 2 B T r = 2 MiB,
    m and v 4 r d_out = 512 KiB each, dR 2 r d_out = 256 KiB; then the norm partials
    (B x 32 slots x 4 B: one per 128 x 128 tile of each R_i, 8 per layer), norms, clip
    factors and the 256-byte error word."""
    from random_gradient_projection_b200 import grape
    layers = [(1024, 1024)] * 4
    KiB, MiB = 1024, 1 << 20
    per_layer = 256 * KiB + 2 * MiB + 2 * 512 * KiB + 256 * KiB
    expect = 2 * MiB + 4 * per_layer + 64 * 32 * 4 + 256 + 256 + 256
    assert grape.grape_context_bytes(layers, 128, 64, 128, grape.GRAPE_BF16) == expect == 16_786_176
    # the fp32 CUDA-core path: fp32 P, AP and dR, one 64 x 64 partial slot per layer here
    tiny = grape.grape_context_bytes([(64, 32)], 8, 4, 16, grape.GRAPE_F32)
    assert tiny == 1024 + 2048 + 2048 + 1024 + 1024 + 1024 + 3 * 256


def test_context_bytes_counts_the_stored_R_i_when_auto_chooses_them(lib):
    """GRAPE_AGG_AUTO stores every R_i (B x r x d_out bf16) on the tensor-core path from
    T = 256 tokens per sample: one more token adds B r 2 bytes of AP and the store's
    B r d_out 2 bytes; the CUDA-core path never stores."""
    from random_gradient_projection_b200 import grape
    a = grape.grape_context_bytes([(1024, 1024)], 128, 4, 255, grape.GRAPE_BF16)
    b = grape.grape_context_bytes([(1024, 1024)], 128, 4, 256, grape.GRAPE_BF16)
    assert b - a == 4 * 128 * 2 + 4 * 128 * 1024 * 2
    c = grape.grape_context_bytes([(1024, 1024)], 128, 4, 255, grape.GRAPE_BF16, grape.GRAPE_PATH_SIMT)
    d = grape.grape_context_bytes([(1024, 1024)], 128, 4, 256, grape.GRAPE_BF16, grape.GRAPE_PATH_SIMT)
    assert d - c == 4 * 128 * 4


def test_context_bytes_grows_with_r_times_d_out_not_d_in_times_d_out(lib):
    """Optimizer state is O(r x layers): doubling d_in changes only P (d_in r), never the
    moments; the moments alone are 8 r d_out per layer."""
    from random_gradient_projection_b200 import grape
    a = grape.grape_context_bytes([(1024, 1024)], 128, 8, 64, grape.GRAPE_BF16)
    b = grape.grape_context_bytes([(2048, 1024)], 128, 8, 64, grape.GRAPE_BF16)
    assert b - a == 1024 * 128 * 2                       # P grows by d_in r bf16, nothing else
    c = grape.grape_context_bytes([(1024, 2048)], 128, 8, 64, grape.GRAPE_BF16)
    assert c - a >= 8 * 128 * 1024                       # m and v grow with d_out


@pytest.mark.parametrize("kw,code", [
    (dict(layers=[(64, 32)], r=80), 1),
    (dict(layers=[(64, 32)], r=8, dtype=0, path=2), 5),
    (dict(layers=[], r=8), 1),
])
def test_context_bytes_validates_like_create(lib, kw, code):
    from random_gradient_projection_b200 import grape
    args = dict(layers=[(64, 32)], r=8, B=4, T=16, dtype=grape.GRAPE_BF16, path=0)
    args.update(kw)
    with pytest.raises(grape.GrapeError) as e:
        grape.grape_context_bytes(**args)
    assert e.value.code == code
