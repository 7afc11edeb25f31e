"""The Python binding refuses buffers the kernels would access out of bounds (CPU only).

The C ABI takes plain addresses and cannot see a buffer's size, so GrapeStep checks
every torch tensor or numpy array it forwards: element count, element size,
contiguity and host/device side.  These tests build a GrapeStep without a library
context (creating one needs a GPU) and call the checks directly.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeStep, grape  # noqa: E402
from random_gradient_projection_b200.grape import _need  # noqa: E402


def _shell(layers=((64, 32), (32, 48)), r=8, B=3, T=5, dtype=grape.GRAPE_BF16):
    g = GrapeStep.__new__(GrapeStep)
    g.layers, g.r, g.B, g.T, g.dtype, g.T_full, g.ctx = list(layers), r, B, T, dtype, 0, 0
    return g


def _host(n, dtype):
    return torch.zeros(n, dtype=dtype)


def test_need_accepts_exact_and_larger_buffers():
    _need(_host(10, torch.bfloat16), 20, 2, "x", False)
    _need(_host(11, torch.int16), 20, 2, "x", False)          # raw 16-bit patterns
    _need(np.zeros(5, np.float32), 20, 4, "x", False)
    _need(None, 20, 4, "x", True)
    _need(12345, 20, 4, "x", True)                             # raw addresses pass


@pytest.mark.parametrize("bad", ["short", "strided", "elsize", "side"])
def test_need_refuses(bad):
    x = {"short": _host(9, torch.bfloat16),
         "strided": _host(40, torch.bfloat16)[::2],
         "elsize": _host(10, torch.float32),
         "side": _host(10, torch.bfloat16)}[bad]
    with pytest.raises(ValueError):
        _need(x, 20, 2, "x", True if bad == "side" else False)


def test_need_refuses_numpy_on_the_device_side_and_strided_arrays():
    with pytest.raises(ValueError):
        _need(np.zeros(8, np.float32), 16, 4, "x", True)
    with pytest.raises(ValueError):
        _need(np.zeros(16, np.float32)[::2], 16, 4, "x", False)


def test_step_inputs_are_checked_per_layer():
    g = _shell()
    rows = g.B * g.T
    A = [_host(rows * d_in, torch.bfloat16) for d_in, _ in g.layers]
    G = [_host(rows * d_out, torch.bfloat16) for _, d_out in g.layers]
    g._inputs(A, G, cuda=False)
    with pytest.raises(ValueError, match=r"Gout\[1\]"):
        g._inputs(A, G[:1] + [_host(rows * 48 - 1, torch.bfloat16)], cuda=False)
    with pytest.raises(ValueError, match="need 2"):
        g._inputs(A[:1], G[:1], cuda=False)
    # masked inputs carry T_full tokens per sample
    with pytest.raises(ValueError, match=r"A\[0\]"):
        g._inputs(A, G, T=g.T + 1, cuda=False)
    with pytest.raises(ValueError):   # fp32 inputs for a bf16 context
        g._inputs([_host(rows * d, torch.float32) for d, _ in g.layers], G, cuda=False)


def test_weights_are_fp32_on_the_device():
    g = _shell()
    Wh = [_host(d_in * d_out, torch.float32) for d_in, d_out in g.layers]
    with pytest.raises(ValueError, match="CUDA"):
        g._weights(Wh)
    with pytest.raises(ValueError, match="need 2"):
        g._weights([1, 2, 3])
    g._weights([1, 2])              # raw device addresses are the caller's responsibility
