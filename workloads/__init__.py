"""Seeded synthetic workloads for the DP-GRAPE projection step.

This module is shared by the fp64 oracle (``oracle/``), the tests and the
benchmark. It holds the five workload shapes and the input recipe, and
nothing of the method's own arithmetic: no projection, no clipping, no
noise, no Adam. The random numbers that the *method* draws (the projection
matrix P and the privacy noise) are not made here; both the oracle and the
CUDA path derive them from the counter-based Philox generator.

Recipe (the same for every workload):

* numpy ``Generator(PCG64)`` streams keyed by ``(seed, step, tag, ...)``
  so that the inputs of any step, and of any sample, can be drawn without
  drawing the others;
* per step, per layer l and sample i: ``A_{l,i} ~ N(0, 1)`` of shape
  ``T x d_in`` from key ``(seed, step, tag, l, 0, i)`` and
  ``Z_{l,i} ~ N(0, 1)`` of shape ``T x d_out`` from key
  ``(seed, step, tag, l, 1, i)``; once per step, from key
  ``(seed, step, tag, 65535)``, the per-sample scale
  ``s_i ~ LogNormal(0, scale_sigma)`` and, where the workload has a
  loss-token mask, ``m_{i,t} ~ Bernoulli(p)``; ``s_i`` and the mask are
  shared by all layers of a sample (a per-sample loss scale and a loss mask);
* ``Gout_{i,l} = kappa * s_i * m_{i,t} * Z_{i,l}`` with
  ``kappa = C / sqrt(p * sum_l T d_in d_out)``: with P scaled to
  ``N(0, 1/r)`` the expected squared norm of a sample's projected gradient
  is ``(C s_i)^2``, so about half of the samples exceed the clipping
  threshold (the median of ``s_i`` is 1);
* inputs of ``bf16`` workloads are rounded to bf16 (round to nearest even)
  after scaling and are kept as their raw 16-bit patterns;
* initial weights ``W_l ~ N(0, 0.02^2)`` in fp32, from their own stream.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Sequence, Tuple

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "get", "kappa", "f32_to_bf16_bits",
    "bf16_bits_to_f32", "StepInputs", "make_step_inputs", "make_weights",
    "scaled",
]

_TAG_INPUTS = 0x5EED
_TAG_WEIGHTS = 0xA11CE


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: a stack of linear layers and the step's hyper-parameters."""

    name: str
    layers: Tuple[Tuple[int, int], ...]   # (d_in, d_out) per linear layer, in order
    r: int                                # projection dimension
    B: int                                # samples per batch
    T: int                                # tokens per sample
    dtype: str                            # "f32" or "bf16" (A and Gout)
    C: float                              # clipping threshold
    sigma: float                          # noise multiplier
    seed: int = 0
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    steps: int = 10
    scale_sigma: float = 1.0              # LogNormal(0, scale_sigma) per-sample scale
    mask_p: float = 1.0                   # Bernoulli keep probability of a loss token
    w_std: float = 0.02
    refresh: int = 1                      # projection-refresh period K (P keyed on step // K)

    @property
    def n_layers(self) -> int:
        return len(self.layers)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    # -- sizes ---------------------------------------------------------------
    def input_bytes(self) -> int:
        """Bytes of A and Gout for one step."""
        el = 4 if self.dtype == "f32" else 2
        return sum(self.B * self.T * (di + do) * el for di, do in self.layers)

    def state_bytes(self) -> int:
        """Bytes of W (fp32) and of the Adam moments m, v (fp32, r x d_out)."""
        return sum(4 * di * do + 8 * self.r * do for di, do in self.layers)


def _stack(blocks: int, per_block: Sequence[Tuple[int, int]]):
    return tuple(l for _ in range(blocks) for l in per_block)


WORKLOADS = {
    # one 64x32 linear layer, fp32, the size the oracle finishes instantly
    "tiny_f32": Workload("tiny_f32", ((64, 32),), r=8, B=4, T=16, dtype="f32",
                         C=1.0, sigma=1.0, steps=3, scale_sigma=1.0),
    # four 1024x1024 linears (an MLP stack)
    "mlp4x1024": Workload("mlp4x1024", _stack(4, [(1024, 1024)]), r=128, B=64,
                          T=128, dtype="bf16", C=1.0, sigma=0.8, steps=10,
                          scale_sigma=1.0),
    # ViT-B shaped: 12 blocks of QKV, out, MLP up, MLP down; 197 tokens
    "vit_b": Workload("vit_b", _stack(12, [(768, 2304), (768, 768), (768, 3072),
                                           (3072, 768)]),
                      r=256, B=32, T=197, dtype="bf16", C=1.0, sigma=1.0,
                      steps=10, scale_sigma=0.5),
    # 7B-LLM shaped slice: 4 decoder blocks of Q, K, V, O, gate, up, down
    "llm7b_slice": Workload("llm7b_slice", _stack(4, [(4096, 4096)] * 4 +
                                                  [(4096, 11008), (4096, 11008),
                                                   (11008, 4096)]),
                            r=512, B=16, T=512, dtype="bf16", C=1.0, sigma=0.6,
                            steps=10, scale_sigma=1.0),
    # long context: 2 blocks, 8192 tokens, sparse loss tokens
    "longctx": Workload("longctx", _stack(2, [(2048, 6144), (2048, 2048),
                                              (2048, 8192), (8192, 2048)]),
                        r=256, B=8, T=8192, dtype="bf16", C=0.5, sigma=1.2,
                        steps=10, scale_sigma=1.0, mask_p=0.1),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def kappa(w: Workload) -> float:
    """Scale of Gout that puts the median projected per-sample norm at C."""
    total = sum(w.T * di * do for di, do in w.layers)
    return w.C / math.sqrt(w.mask_p * total)


# -- bf16 bit patterns (input format only) -----------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the uint16 patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 patterns to fp32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# -- inputs --------------------------------------------------------------------

@dataclasses.dataclass
class StepInputs:
    """A and Gout of one step, per layer, in the workload's storage format.

    ``A[l]`` has shape ``(B, T, d_in)``, ``Gout[l]`` has shape ``(B, T, d_out)``;
    bf16 workloads hold uint16 bit patterns, fp32 workloads hold float32.
    ``scale`` (B,) and ``mask`` (B, T) are the per-sample scale and token mask
    that went into Gout; they are kept for inspection only.
    """

    A: List[np.ndarray]
    Gout: List[np.ndarray]
    scale: np.ndarray
    mask: np.ndarray
    dtype: str

    def as_f64(self, x: np.ndarray) -> np.ndarray:
        """Exact float64 values of a stored input array."""
        if self.dtype == "bf16":
            return bf16_bits_to_f32(x).astype(np.float64)
        return np.asarray(x, dtype=np.float64)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(list(key)))


def make_step_inputs(w: Workload, step: int, samples: Sequence[int] | None = None,
                     threads: int = 0) -> StepInputs:
    """Draw the A and Gout of ``step`` (0-based) following the recipe above.

    ``samples`` keeps only those samples, in that order; each sample has its
    own streams, so a sub-batch equals the matching rows of the full batch.
    ``threads`` > 1 draws the per-sample streams on a thread pool (numpy
    releases the GIL while it fills an array).
    """
    sel = list(range(w.B)) if samples is None else [int(i) for i in samples]
    head = _rng(w.seed, step, _TAG_INPUTS, 65535)
    s = head.lognormal(0.0, w.scale_sigma, size=w.B).astype(np.float32)
    if w.mask_p < 1.0:
        mask = (head.random((w.B, w.T)) < w.mask_p).astype(np.float32)
    else:
        mask = np.ones((w.B, w.T), dtype=np.float32)
    k = np.float32(kappa(w))
    store = np.uint16 if w.dtype == "bf16" else np.float32
    A = [np.empty((len(sel), w.T, di), dtype=store) for di, _ in w.layers]
    G = [np.empty((len(sel), w.T, do), dtype=store) for _, do in w.layers]

    def fill(job):
        l, j = job
        i = sel[j]
        d_in, d_out = w.layers[l]
        a = _rng(w.seed, step, _TAG_INPUTS, l, 0, i).standard_normal((w.T, d_in), dtype=np.float32)
        z = _rng(w.seed, step, _TAG_INPUTS, l, 1, i).standard_normal((w.T, d_out), dtype=np.float32)
        g = (k * s[i] * mask[i][:, None]) * z
        if w.dtype == "bf16":
            A[l][j] = f32_to_bf16_bits(a)
            G[l][j] = f32_to_bf16_bits(g)
        else:
            A[l][j] = a
            G[l][j] = g

    jobs = [(l, j) for l in range(w.n_layers) for j in range(len(sel))]
    if threads > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, jobs))
    else:
        for job in jobs:
            fill(job)
    return StepInputs(A=A, Gout=G, scale=s[sel], mask=mask[sel], dtype=w.dtype)


def make_weights(w: Workload) -> List[np.ndarray]:
    """Initial fp32 weights W_l (d_in x d_out, row-major), N(0, w_std^2)."""
    rng = _rng(w.seed, _TAG_WEIGHTS)
    return [(w.w_std * rng.standard_normal((di, do), dtype=np.float32)).astype(np.float32)
            for di, do in w.layers]


def scaled(w: Workload, **kw) -> Workload:
    """A reduced copy of a workload (fewer layers / samples / tokens) for fast tests.

    ``n_layers`` keeps the first layers; every other keyword replaces a field.
    """
    n = kw.pop("n_layers", None)
    if n is not None:
        kw["layers"] = tuple(w.layers[:n])
    return w.replace(**kw)
