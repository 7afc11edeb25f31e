"""B200-native (sm_100a) DP-GRAPE projection step behind a C ABI (include/grape.h).

``grape`` is the ctypes binding of ``libgrape.so``; the library is built
in-tree with ``python -m random_gradient_projection_b200.build``.
"""
from . import grape  # noqa: F401
from .grape import GrapeStep, GrapeError  # noqa: F401
