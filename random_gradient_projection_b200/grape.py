"""ctypes binding of libgrape.so (the C ABI in include/grape.h).

Argument marshalling only: every step of the method runs in the library's
CUDA kernels.  The functions keep the C names; ``GrapeStep`` is a small
owner of a context that accepts torch tensors.  Importing this module fails
loudly when the library has not been built: there is no other code path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
# GRAPE_LIB=checked loads the bounds-checked build (libgrape_checked.so) instead
LIB_PATH = os.path.join(HERE, "libgrape_checked.so" if os.environ.get("GRAPE_LIB") == "checked"
                        else "libgrape.so")

GRAPE_OK, GRAPE_EINVAL, GRAPE_ENOMEM, GRAPE_ECUDA, GRAPE_ETIMEOUT, GRAPE_EUNSUPPORTED = range(6)
GRAPE_MAX_LAYERS = 64
GRAPE_F32, GRAPE_BF16 = 0, 1
GRAPE_PATH_AUTO, GRAPE_PATH_SIMT, GRAPE_PATH_TC = 0, 1, 2
(GRAPE_DBG_NORMS, GRAPE_DBG_CLIP, GRAPE_DBG_S, GRAPE_DBG_P, GRAPE_DBG_DR, GRAPE_DBG_M,
 GRAPE_DBG_V) = range(7)

# the entry points include/grape.h declares
EXPORTS = (
    "grape_create", "grape_step", "grape_step_host", "grape_accumulate", "grape_S_ptr",
    "grape_apply", "grape_get_state", "grape_set_state", "grape_debug", "grape_device_bytes",
    "grape_path_of", "grape_last_error", "grape_global_error", "grape_destroy",
    "grape_philox_words", "grape_gaussian", "grape_profile", "grape_profile_read",
    "grape_launch_count", "grape_layer_sqnorms_static", "grape_set_refresh_period", "grape_sqnorms",
    "grape_enable_compaction", "grape_step_masked", "grape_live_counts", "grape_set_norm_method",
    "grape_set_graph", "grape_selftest_wait_timeout", "grape_S_all", "grape_context_bytes",
    "grape_set_aggregation", "grape_aggregation_of",
)
GRAPE_NORM_DIRECT, GRAPE_NORM_GHOST = 0, 1
GRAPE_AGG_AUTO, GRAPE_AGG_RECOMPUTE, GRAPE_AGG_STORE = 0, 1, 2
PHASES = ("gen_P", "project", "norm", "clip", "aggregate", "adam", "backproject", "compact",
          "aggregate_adam")   # GRAPE_N_PHASES


class grape_layer(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int32), ("d_out", ctypes.c_int32)]


class grape_adam(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double)]


class GrapeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"grape error {code}: {msg}")
        self.code = code


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m random_gradient_projection_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, u32, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64
    pp = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "grape_create": ([ctypes.POINTER(grape_layer), i32, i32, ctypes.c_double, ctypes.c_double, u64,
                          ctypes.POINTER(grape_adam), i32, i32, i32, i32, ctypes.POINTER(vp)], i32),
        "grape_step": ([vp, pp, pp, pp, i64, vp], i32),
        "grape_step_host": ([vp, pp, pp, pp, i64, vp, vp], i32),
        "grape_accumulate": ([vp, pp, pp, i64, vp], i32),
        "grape_S_ptr": ([vp, i32, ctypes.POINTER(vp)], i32),
        "grape_apply": ([vp, pp, i64, i64, vp], i32),
        "grape_get_state": ([vp, i32, vp, vp, vp], i32),
        "grape_set_state": ([vp, i32, vp, vp, vp], i32),
        "grape_debug": ([vp, i32, i32, vp], i32),
        "grape_device_bytes": ([vp, ctypes.POINTER(u64)], i32),
        "grape_context_bytes": ([ctypes.POINTER(grape_layer), i32, i32, i32, i32, i32, i32,
                                 ctypes.POINTER(u64)], i32),
        "grape_path_of": ([vp, ctypes.POINTER(i32)], i32),
        "grape_last_error": ([vp], ctypes.c_char_p),
        "grape_global_error": ([], ctypes.c_char_p),
        "grape_destroy": ([vp], None),
        "grape_philox_words": ([u64, u32, u32, u32, i64, vp, vp], i32),
        "grape_gaussian": ([u64, u32, u32, u32, i64, vp, vp], i32),
        "grape_profile": ([vp, i32], i32),
        "grape_profile_read": ([vp, vp, vp], i32),
        "grape_launch_count": ([vp, ctypes.POINTER(u64)], i32),
        "grape_layer_sqnorms_static": ([vp, vp, i32, i32, i32, i32, i32, u64, u32, u32, vp, vp], i32),
        "grape_set_refresh_period": ([vp, i32], i32),
        "grape_sqnorms": ([vp, pp, pp, i64, vp, vp], i32),
        "grape_enable_compaction": ([vp, i32], i32),
        "grape_step_masked": ([vp, pp, pp, pp, vp, i64, vp], i32),
        "grape_live_counts": ([vp, vp], i32),
        "grape_set_norm_method": ([vp, i32], i32),
        "grape_set_graph": ([vp, i32], i32),
        "grape_selftest_wait_timeout": ([i64, i64, ctypes.POINTER(i32)], i32),
        "grape_S_all": ([vp, ctypes.POINTER(vp), ctypes.POINTER(i64)], i32),
        "grape_set_aggregation": ([vp, i32], i32),
        "grape_aggregation_of": ([vp, ctypes.POINTER(i32)], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


def _ptr(x) -> int:
    """Address of a torch tensor, an int, or None (0)."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _array(ptrs) -> ctypes.Array:
    return (ctypes.c_void_p * len(ptrs))(*[_ptr(p) for p in ptrs])


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, ctx=None):
    if rc != GRAPE_OK:
        L = lib()
        msg = (L.grape_last_error(ctx) if ctx else L.grape_global_error()) or b""
        raise GrapeError(rc, msg.decode())


# ---- the C names, marshalled ------------------------------------------------

def grape_create(layers: Sequence[Sequence[int]], r: int, C: float, sigma: float, seed: int,
                 lr: float, beta1: float, beta2: float, eps: float, B: int, T: int,
                 dtype: int, path: int = GRAPE_PATH_AUTO) -> int:
    arr = (grape_layer * len(layers))(*[grape_layer(int(a), int(b)) for a, b in layers])
    adam = grape_adam(lr, beta1, beta2, eps)
    out = ctypes.c_void_p()
    _check(lib().grape_create(arr, len(layers), r, C, sigma, seed & (2**64 - 1), ctypes.byref(adam),
                              B, T, dtype, path, ctypes.byref(out)))
    return out.value


def grape_step(ctx: int, A, Gout, W, step: int, stream=None):
    _check(lib().grape_step(ctx, _array(A), _array(Gout), _array(W), step, _stream(stream)), ctx)


def grape_step_host(ctx: int, A_host, Gout_host, W, step: int, norms_host=None, stream=None):
    _check(lib().grape_step_host(ctx, _array(A_host), _array(Gout_host), _array(W), step,
                                 _ptr(norms_host), _stream(stream)), ctx)


def grape_accumulate(ctx: int, A, Gout, step: int, stream=None):
    _check(lib().grape_accumulate(ctx, _array(A), _array(Gout), step, _stream(stream)), ctx)


def grape_set_refresh_period(ctx: int, period: int):
    _check(lib().grape_set_refresh_period(ctx, period), ctx)


def grape_sqnorms(ctx: int, A, Gout, step: int, sqnorms_dev, stream=None):
    _check(lib().grape_sqnorms(ctx, _array(A), _array(Gout), step, _ptr(sqnorms_dev), _stream(stream)), ctx)


def grape_selftest_wait_timeout(short_ns: int, long_ns: int):
    """(status code, bits) of the bounded-wait self-test; GRAPE_ETIMEOUT with bits 3 is correct."""
    bits = ctypes.c_int32(0)
    rc = lib().grape_selftest_wait_timeout(short_ns, long_ns, ctypes.byref(bits))
    return rc, bits.value


def grape_set_graph(ctx: int, enable: bool):
    _check(lib().grape_set_graph(ctx, 1 if enable else 0), ctx)


def grape_set_norm_method(ctx: int, method: int):
    _check(lib().grape_set_norm_method(ctx, method), ctx)


def grape_set_aggregation(ctx: int, method: int):
    _check(lib().grape_set_aggregation(ctx, method), ctx)


def grape_aggregation_of(ctx: int) -> int:
    out = ctypes.c_int32()
    _check(lib().grape_aggregation_of(ctx, ctypes.byref(out)), ctx)
    return out.value


def grape_enable_compaction(ctx: int, T_full: int):
    _check(lib().grape_enable_compaction(ctx, T_full), ctx)


def grape_step_masked(ctx: int, A, Gout, W, mask_dev, step: int, stream=None):
    _check(lib().grape_step_masked(ctx, _array(A), _array(Gout), _array(W), _ptr(mask_dev), step,
                                   _stream(stream)), ctx)


def grape_live_counts(ctx: int, B: int) -> np.ndarray:
    out = np.zeros(B, dtype=np.int32)
    _check(lib().grape_live_counts(ctx, out.ctypes.data), ctx)
    return out


def grape_S_all(ctx: int):
    """(device address, element count) of all S_l, back to back in layer order."""
    ptr, n = ctypes.c_void_p(), ctypes.c_int64()
    _check(lib().grape_S_all(ctx, ctypes.byref(ptr), ctypes.byref(n)), ctx)
    return ptr.value, n.value


def grape_S_ptr(ctx: int, layer: int) -> int:
    out = ctypes.c_void_p()
    _check(lib().grape_S_ptr(ctx, layer, ctypes.byref(out)), ctx)
    return out.value


def grape_apply(ctx: int, W, step: int, batch_total: int = 0, stream=None):
    _check(lib().grape_apply(ctx, _array(W), step, batch_total, _stream(stream)), ctx)


def grape_get_state(ctx: int, layer: int, m, v, stream=None):
    _check(lib().grape_get_state(ctx, layer, _ptr(m), _ptr(v), _stream(stream)), ctx)


def grape_set_state(ctx: int, layer: int, m, v, stream=None):
    _check(lib().grape_set_state(ctx, layer, _ptr(m), _ptr(v), _stream(stream)), ctx)


def grape_debug(ctx: int, what: int, layer: int, shape) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _check(lib().grape_debug(ctx, what, layer, out.ctypes.data), ctx)
    return out


def grape_context_bytes(layers: Sequence[Sequence[int]], r: int, B: int, T: int, dtype: int,
                        path: int = GRAPE_PATH_AUTO) -> int:
    """Bytes grape_create would allocate for these arguments (host only, no device call)."""
    arr = (grape_layer * len(layers))(*[grape_layer(int(a), int(b)) for a, b in layers])
    out = ctypes.c_uint64()
    _check(lib().grape_context_bytes(arr, len(layers), r, B, T, dtype, path, ctypes.byref(out)))
    return out.value


def grape_device_bytes(ctx: int) -> int:
    out = ctypes.c_uint64()
    _check(lib().grape_device_bytes(ctx, ctypes.byref(out)), ctx)
    return out.value


def grape_path_of(ctx: int) -> int:
    out = ctypes.c_int32()
    _check(lib().grape_path_of(ctx, ctypes.byref(out)), ctx)
    return out.value


def grape_profile(ctx: int, enable: bool):
    _check(lib().grape_profile(ctx, 1 if enable else 0), ctx)


def grape_profile_read(ctx: int):
    """{phase name: (milliseconds, calls)} since profiling was switched on."""
    ms = np.zeros(len(PHASES), dtype=np.float64)
    cnt = np.zeros(len(PHASES), dtype=np.int64)
    _check(lib().grape_profile_read(ctx, ms.ctypes.data, cnt.ctypes.data), ctx)
    return {name: (float(ms[k]), int(cnt[k])) for k, name in enumerate(PHASES)}


def grape_launch_count(ctx: int) -> int:
    out = ctypes.c_uint64()
    _check(lib().grape_launch_count(ctx, ctypes.byref(out)), ctx)
    return out.value


def grape_layer_sqnorms_static(A, Gout, d_in: int, d_out: int, r: int, B: int, T: int, seed: int,
                               layer: int, step: int, sqnorms_out, stream=None):
    """Per-sample squared projected norms of one bf16 layer; uses only the library's
    static device scratch (no allocation).  See include/grape.h."""
    _check(lib().grape_layer_sqnorms_static(_ptr(A), _ptr(Gout), d_in, d_out, r, B, T,
                                            seed & (2**64 - 1), layer, step, _ptr(sqnorms_out),
                                            _stream(stream)))


def grape_destroy(ctx: int):
    lib().grape_destroy(ctx)


def grape_philox_words(seed: int, layer: int, step: int, stream_id: int, n_blocks: int, out,
                       stream=None):
    _check(lib().grape_philox_words(seed & (2**64 - 1), layer, step, stream_id, n_blocks, _ptr(out),
                                    _stream(stream)))


def grape_gaussian(seed: int, layer: int, step: int, stream_id: int, n: int, out, stream=None):
    _check(lib().grape_gaussian(seed & (2**64 - 1), layer, step, stream_id, n, _ptr(out),
                                _stream(stream)))


# ---- buffer checks of the context owner below ---------------------------------

def _need(x, nbytes: int, el: int, what: str, cuda: Optional[bool]):
    """Refuse a torch tensor or numpy array that cannot serve as `nbytes` contiguous bytes
    of `el`-byte elements from its start, or that lies on the wrong side of the host /
    device split (cuda None: either side).  The kernels read and write whole buffers
    from plain addresses, so a short or strided buffer would be accessed out of bounds.
    Raw integer addresses pass unchecked."""
    if x is None or isinstance(x, int):
        return
    if isinstance(x, np.ndarray):
        ok = (x.flags.c_contiguous and x.itemsize == el and x.nbytes >= nbytes and cuda is not True)
    else:
        ok = (x.is_contiguous() and x.element_size() == el and x.numel() * el >= nbytes
              and (cuda is None or x.is_cuda == cuda))
    if not ok:
        where = {True: "a CUDA", False: "a host", None: "a"}[cuda]
        raise ValueError(f"{what}: need {where} contiguous buffer of at least {nbytes} bytes of "
                         f"{el}-byte elements, got {getattr(x, 'shape', None)} "
                         f"{getattr(x, 'dtype', type(x).__name__)}")


# ---- a context owner for torch tensors ---------------------------------------

class _DeviceArray:
    """Wraps a library-owned device buffer for torch.as_tensor (no copy)."""

    def __init__(self, ptr: int, shape, typestr: str = "<f4"):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


class GrapeStep:
    """One DP-GRAPE context: a fixed layer stack, batch shape and hyper-parameters."""

    def __init__(self, layers, r, C, sigma, seed, B, T, dtype="bf16", lr=1e-3, beta1=0.9,
                 beta2=0.999, eps=1e-8, path=GRAPE_PATH_AUTO):
        self.layers = [tuple(int(x) for x in l) for l in layers]
        self.r, self.B, self.T = int(r), int(B), int(T)
        self.dtype = GRAPE_BF16 if dtype in ("bf16", GRAPE_BF16) else GRAPE_F32
        self.T_full = 0   # tokens per sample of masked inputs (enable_compaction)
        self.ctx = grape_create(self.layers, self.r, C, sigma, seed, lr, beta1, beta2, eps, B, T,
                                self.dtype, path)

    def _inputs(self, A, Gout, T=None, cuda=True):
        el = 2 if self.dtype == GRAPE_BF16 else 4
        rows = self.B * (T or self.T)
        if len(A) != len(self.layers) or len(Gout) != len(self.layers):
            raise ValueError(f"need {len(self.layers)} A and Gout buffers")
        for l, (d_in, d_out) in enumerate(self.layers):
            _need(A[l], rows * d_in * el, el, f"A[{l}]", cuda)
            _need(Gout[l], rows * d_out * el, el, f"Gout[{l}]", cuda)

    def _weights(self, W):
        if len(W) != len(self.layers):
            raise ValueError(f"need {len(self.layers)} W buffers")
        for l, (d_in, d_out) in enumerate(self.layers):
            _need(W[l], d_in * d_out * 4, 4, f"W[{l}]", True)

    @classmethod
    def for_workload(cls, w, path=GRAPE_PATH_AUTO, B=None):
        g = cls(w.layers, w.r, w.C, w.sigma, w.seed, B or w.B, w.T, w.dtype, w.lr, w.beta1,
                w.beta2, w.eps, path)
        if getattr(w, "refresh", 1) != 1:
            g.set_refresh_period(w.refresh)
        return g

    def set_graph(self, enable: bool = True):
        """Replay grape_step through CUDA graphs (one per set of A, Gout, W pointers)."""
        grape_set_graph(self.ctx, enable)

    def set_norm_method(self, method: int):
        """GRAPE_NORM_DIRECT (default) or GRAPE_NORM_GHOST (tensor-core path)."""
        grape_set_norm_method(self.ctx, method)

    def set_aggregation(self, method: int):
        """GRAPE_AGG_AUTO (the default), GRAPE_AGG_RECOMPUTE or GRAPE_AGG_STORE."""
        grape_set_aggregation(self.ctx, method)

    @property
    def aggregation(self) -> int:
        """The aggregation the next step uses: GRAPE_AGG_RECOMPUTE or GRAPE_AGG_STORE."""
        return grape_aggregation_of(self.ctx)

    def enable_compaction(self, T_full: int):
        """Inputs of T_full tokens per sample, compacted to this context's T kept tokens."""
        grape_enable_compaction(self.ctx, T_full)
        self.T_full = int(T_full)

    def step_masked(self, A, Gout, W, mask, step: int, stream=None):
        """The step over the tokens ``mask`` (uint8 / bool device tensor, B x T_full) keeps."""
        self._inputs(A, Gout, self.T_full)
        self._weights(W)
        _need(mask, self.B * self.T_full, 1, "mask", True)
        grape_step_masked(self.ctx, A, Gout, W, mask, step, stream)

    def live_counts(self) -> np.ndarray:
        return grape_live_counts(self.ctx, self.B)

    def set_refresh_period(self, period: int):
        grape_set_refresh_period(self.ctx, period)

    def sqnorms(self, A, Gout, step: int, out=None, stream=None):
        """Per-sample squared norm estimates sum_l ||(A_il P_l)^T Gout_il||^2 (B floats on
        the device); `out` is a torch float32 tensor of B elements, or one is allocated."""
        if out is None:
            import torch
            out = torch.empty(self.B, dtype=torch.float32, device=A[0].device)
        self._inputs(A, Gout)
        _need(out, self.B * 4, 4, "out", True)
        grape_sqnorms(self.ctx, A, Gout, step, out, stream)
        return out

    def close(self):
        if self.ctx:
            grape_destroy(self.ctx)
            self.ctx = 0

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001  interpreter shutdown
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def path(self) -> int:
        return grape_path_of(self.ctx)

    def device_bytes(self) -> int:
        return grape_device_bytes(self.ctx)

    def profile(self, enable: bool = True):
        grape_profile(self.ctx, enable)

    def profile_read(self):
        return grape_profile_read(self.ctx)

    def launch_count(self) -> int:
        return grape_launch_count(self.ctx)

    def step(self, A, Gout, W, step: int, stream=None):
        self._inputs(A, Gout)
        self._weights(W)
        grape_step(self.ctx, A, Gout, W, step, stream)

    def bind(self, A, Gout, W, stream=None) -> "BoundStep":
        """grape_step on fixed buffers: checks A, Gout and W once, marshals their
        addresses and the stream once, and returns an object whose ``step(s)`` makes
        only the C call.  For loops that step over the same buffers; the tensors are
        kept referenced, and must not be resized while the binding is in use."""
        self._inputs(A, Gout)
        self._weights(W)
        return BoundStep(self, A, Gout, W, stream)

    def step_host(self, A_host, Gout_host, W, step: int, norms_host=None, stream=None):
        self._inputs(A_host, Gout_host, cuda=False)
        self._weights(W)
        _need(norms_host, self.B * 4, 4, "norms_host", False)
        grape_step_host(self.ctx, A_host, Gout_host, W, step, norms_host, stream)

    def accumulate(self, A, Gout, step: int, stream=None):
        self._inputs(A, Gout)
        grape_accumulate(self.ctx, A, Gout, step, stream)

    def apply(self, W, step: int, batch_total: int = 0, stream=None):
        self._weights(W)
        grape_apply(self.ctx, W, step, batch_total, stream)

    def S_tensor(self, layer: int):
        """S_l as a torch tensor sharing the library's memory (for all-reduce)."""
        import torch
        ptr = grape_S_ptr(self.ctx, layer)
        return torch.as_tensor(_DeviceArray(ptr, (self.r, self.layers[layer][1])), device="cuda")

    def S_all_tensor(self):
        """Every S_l as one flat torch tensor sharing the library's memory (layer order):
        one all-reduce sums all layers over the ranks."""
        import torch
        ptr, n = grape_S_all(self.ctx)
        return torch.as_tensor(_DeviceArray(ptr, (n,)), device="cuda")

    def get_state(self, layer: int, m, v, stream=None):
        if 0 <= layer < len(self.layers):   # the library refuses other layers
            n = self.r * self.layers[layer][1] * 4
            _need(m, n, 4, "m", True)
            _need(v, n, 4, "v", True)
        grape_get_state(self.ctx, layer, m, v, stream)

    def set_state(self, layer: int, m, v, stream=None):
        if 0 <= layer < len(self.layers):   # the library refuses other layers
            n = self.r * self.layers[layer][1] * 4
            _need(m, n, 4, "m", True)
            _need(v, n, 4, "v", True)
        grape_set_state(self.ctx, layer, m, v, stream)

    # intermediates of the last step (host copies)
    def norms(self):
        return grape_debug(self.ctx, GRAPE_DBG_NORMS, 0, (self.B,))

    def clip(self):
        return grape_debug(self.ctx, GRAPE_DBG_CLIP, 0, (self.B,))

    def S(self, l):
        return grape_debug(self.ctx, GRAPE_DBG_S, l, (self.r, self.layers[l][1]))

    def P(self, l):
        return grape_debug(self.ctx, GRAPE_DBG_P, l, (self.layers[l][0], self.r))

    def dR(self, l):
        return grape_debug(self.ctx, GRAPE_DBG_DR, l, (self.r, self.layers[l][1]))

    def m(self, l):
        return grape_debug(self.ctx, GRAPE_DBG_M, l, (self.r, self.layers[l][1]))

    def v(self, l):
        return grape_debug(self.ctx, GRAPE_DBG_V, l, (self.r, self.layers[l][1]))


class BoundStep:
    """grape_step with its buffers and stream marshalled once (GrapeStep.bind)."""

    def __init__(self, owner: GrapeStep, A, Gout, W, stream=None):
        self.owner = owner
        self._keep = (list(A), list(Gout), list(W))   # the buffers outlive the binding
        self._args = (_array(A), _array(Gout), _array(W))
        self._stream = _stream(stream)

    def step(self, step: int):
        A, G, W = self._args
        _check(lib().grape_step(self.owner.ctx, A, G, W, step, self._stream), self.owner.ctx)
