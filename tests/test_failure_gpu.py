"""Failure detection on the device, without a fault or a hang (needs a B200).

Every wait of the tensor-core kernels is bounded: a wait that runs out raises the CTA's
abort flag, the CTA's other waits leave at once, an error word is written and the host
reports GRAPE_ETIMEOUT with the context still usable.  grape_selftest_wait_timeout runs
exactly that helper on two mbarriers that nothing ever arrives on.
"""
import time

import numpy as np
import pytest

import workloads as W
from harness import to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeStep, grape  # noqa: E402


def test_bounded_wait_gives_up_and_aborts_the_cta():
    t0 = time.perf_counter()
    rc, bits = grape.grape_selftest_wait_timeout(2_000_000, 5_000_000_000)   # 2 ms and 5 s
    elapsed = time.perf_counter() - t0
    assert rc == grape.GRAPE_ETIMEOUT
    assert bits == 3, bits            # warp 0 timed out; warp 1 left on the abort flag
    assert elapsed < 2.0, elapsed     # nowhere near the 5 s limit of the second wait


def test_device_is_usable_after_a_timeout():
    rc, _ = grape.grape_selftest_wait_timeout(1_000_000, 1_000_000_000)
    assert rc == grape.GRAPE_ETIMEOUT
    w = W.scaled(W.get("mlp4x1024"), n_layers=1, B=2, T=32)
    g = GrapeStep.for_workload(w, path=grape.GRAPE_PATH_TC)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    x = W.make_step_inputs(w, 0, threads=8)
    g.step([to_device(a, w.dtype) for a in x.A], [to_device(a, w.dtype) for a in x.Gout], Ws, 0)
    torch.cuda.synchronize()
    assert np.all(np.isfinite(g.norms()))
    g.close()
