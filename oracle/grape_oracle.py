"""fp64 CPU oracle of the DP-GRAPE projection step.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module. The
library (``random_gradient_projection_b200``) never imports, links or runs
it, and this module imports nothing from the library: the two share no
code. The only shared module is ``workloads`` (seeded synthetic inputs,
which holds none of the method's arithmetic).

What it computes, in the pages' order (source: "Memory-Efficient
Differentially Private Training with Gradient Random Projection",
gist.science/es/paper/2506.15588, "Resumen Técnico: DP-GRAPE",
section "Metodología: DP-GRAPE"; the same text is on the fr, it and hi
pages of the same paper):

1. random Gaussian projection matrices, one per layer, regenerated from a
   seed instead of stored (design choice 1 of "Metodología");
2. the *raw* per-sample gradients are projected first, then clipped and
   noised in the projected space (design choice 2: projection comes before
   privatization);
3. Adam's first and second moments live in the projected space
   (design choice 3: the optimizer states are kept projected);
4. the loop: per-layer projection of per-sample gradients, then
   aggregation, clipping and noise, then a projected Adam update of the
   parameters (closing paragraph of "Metodología").

The pages describe the method in prose only. The concrete operator below
is the plainest reading that the prose supports; every point the pages
leave open is marked "reading:".

This oracle materialises every per-sample gradient ``G_i = A_i^T Gout_i``
(d_in x d_out, fp64), exactly the object that DP-Adam stores and that the
method avoids; the CUDA library never forms it.

Pins (tests/test_oracle_pins.py): Philox against torch's own Philox engine
and its counter arithmetic; Box-Muller statistics; P = I reducing to
explicit per-sample DP-Adam built on autograd; the factored projection by
brute force; clipping bounds; sigma = 0; the Adam t = 1 closed form; the
no-privacy reduction to one stacked GEMM; and a mutation test showing that
plausible mistakes planted in this file fail a pin. Conventions that the
pages do not fix (the 1/sqrt(r) scale of P, re-drawing P every step, the
1/B normalisation, the Adam variant) are pinned only by internal
consistency: parity unpinned against the pages for those readings.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Optional, Sequence

import numpy as np

# --------------------------------------------------------------------------
# Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
# Easy as 1, 2, 3", SC'11, section 3.2 and table 2): a 4 x 32-bit counter, a
# 2 x 32-bit key, 10 rounds.  Each round multiplies counter words 0 and 2 by
# the two round multipliers, keeps the high and low halves of both products,
# and mixes the high halves with the other two counter words and the key;
# the key is advanced by the two Weyl constants between rounds.
# --------------------------------------------------------------------------
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
PHILOX_ROUNDS = 10
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(counter: np.ndarray, key: Sequence[int]) -> np.ndarray:
    """Philox4x32-10 of every row of ``counter`` (n x 4, uint32) under ``key`` (2 words)."""
    c = [np.asarray(counter[:, j], dtype=np.uint64) for j in range(4)]
    k0, k1 = np.uint64(int(key[0]) & 0xFFFFFFFF), np.uint64(int(key[1]) & 0xFFFFFFFF)
    m0, m1 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1)
    for rnd in range(PHILOX_ROUNDS):
        if rnd > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = c[0] * m0          # < 2^64: exact in uint64
        p1 = c[2] * m1
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return np.stack(c, axis=1).astype(np.uint32)


# Streams of the method's randomness (reading: the pages say only that P is rebuilt
# from a seed rather than stored; the key and counter layout below are this
# library's choice).
STREAM_PROJECTION = 0
STREAM_NOISE = 1


def philox_words(seed: int, layer: int, step: int, stream: int, n_blocks: int) -> np.ndarray:
    """The 4-word outputs for counters (q, layer, step, stream), q = 0..n_blocks-1.

    key = (low 32 bits of seed, high 32 bits of seed).
    """
    ctr = np.zeros((n_blocks, 4), dtype=np.uint32)
    ctr[:, 0] = np.arange(n_blocks, dtype=np.uint64).astype(np.uint32)
    ctr[:, 1] = np.uint32(layer)
    ctr[:, 2] = np.uint32(step)
    ctr[:, 3] = np.uint32(stream)
    return philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))


def box_muller(xa: np.ndarray, xb: np.ndarray):
    """Box-Muller (1958) on two uint32 words, in fp64.

    u1 = (xa + 1) / 2^32 lies in (0, 1] so the logarithm is finite;
    u2 = xb / 2^32 lies in [0, 1).  Returns (rho cos 2 pi u2, rho sin 2 pi u2)
    with rho = sqrt(-2 ln u1).
    """
    u1 = (xa.astype(np.float64) + 1.0) * 2.0 ** -32
    u2 = xb.astype(np.float64) * 2.0 ** -32
    rho = np.sqrt(-2.0 * np.log(u1))
    return rho * np.cos(2.0 * np.pi * u2), rho * np.sin(2.0 * np.pi * u2)


def gaussian_stream(seed: int, layer: int, step: int, stream: int, n: int) -> np.ndarray:
    """Standard normals z[e], e = 0..n-1, of one (seed, layer, step, stream).

    Element e comes from counter block q = e // 4: words (x0, x1) give
    elements 4q and 4q+1 (cosine, sine); words (x2, x3) give 4q+2 and 4q+3.
    """
    nb = (n + 3) // 4
    w = philox_words(seed, layer, step, stream, nb)
    z0, z1 = box_muller(w[:, 0], w[:, 1])
    z2, z3 = box_muller(w[:, 2], w[:, 3])
    return np.stack([z0, z1, z2, z3], axis=1).reshape(-1)[:n]


def projection_matrix(seed: int, layer: int, step: int, d_in: int, r: int) -> np.ndarray:
    """P_l (d_in x r), row-major element e = k*r + j, entries N(0, 1/r).

    Reading: the pages give no scale for the Gaussian matrix; 1/sqrt(r) makes
    E[P P^T] = I, so P P^T G is an unbiased estimate of G.  P is re-drawn at
    every step from (seed, layer, step) (reading of design choice 1, which has P
    rebuilt from a seed whenever it is needed).
    """
    return gaussian_stream(seed, layer, step, STREAM_PROJECTION, d_in * r).reshape(d_in, r) / np.sqrt(r)


def noise_matrix(seed: int, layer: int, step: int, r: int, d_out: int) -> np.ndarray:
    """xi_l (r x d_out), row-major element e = j*d_out + n, entries N(0, 1)."""
    return gaussian_stream(seed, layer, step, STREAM_NOISE, r * d_out).reshape(r, d_out)


# --------------------------------------------------------------------------
# The step
# --------------------------------------------------------------------------

def per_sample_gradient(A_i: np.ndarray, Gout_i: np.ndarray) -> np.ndarray:
    """G_i = A_i^T Gout_i (d_in x d_out): the gradient of a linear layer for one sample."""
    return A_i.T @ Gout_i


def project(P: np.ndarray, G: np.ndarray) -> np.ndarray:
    """R = P^T G (r x d_out): the projected per-sample gradient."""
    return P.T @ G


def clip_factor(norm: float, C: float) -> float:
    """c = C / n if n > C else 1 (reading: the threshold itself is not clipped; n = 0 gives 1)."""
    return C / norm if norm > C else 1.0


def adam(m: np.ndarray, v: np.ndarray, g: np.ndarray, t: int, beta1: float, beta2: float,
         eps: float):
    """Bias-corrected Adam (Kingma & Ba 2015, Algorithm 1) on the projected gradient.

    Reading: plain Adam, eps added after the square root, no weight decay and
    no extra scale.  Returns (m', v', step direction dR).
    """
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    return m, v, m_hat / (np.sqrt(v_hat) + eps)


@dataclasses.dataclass
class Hyper:
    r: int
    C: float
    sigma: float
    seed: int
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    refresh: int = 1     # projection-refresh period K: P of step s is drawn with key floor(s / K)

    @classmethod
    def of(cls, w) -> "Hyper":
        return cls(r=w.r, C=w.C, sigma=w.sigma, seed=w.seed, lr=w.lr, beta1=w.beta1,
                   beta2=w.beta2, eps=w.eps, refresh=getattr(w, "refresh", 1))

    def projection_key(self, step: int) -> int:
        """Step field of P's Philox counter at step s.

        Reading: design choice 1 of "Metodología" has P rebuilt from a seed and
        leaves the refresh schedule open.  K = 1 re-draws P every
        step; K > 1 keeps one random subspace for K consecutive steps (as GaLore
        keeps its SVD subspace between refreshes), with m and v carried across
        refreshes unchanged.  The noise is drawn per step whatever K is.
        """
        return step // self.refresh


@dataclasses.dataclass
class State:
    """W_l (d_in x d_out) and the projected Adam moments m_l, v_l (r x d_out), fp64."""

    W: List[np.ndarray]
    m: List[np.ndarray]
    v: List[np.ndarray]

    @classmethod
    def init(cls, W0: Sequence[np.ndarray], r: int) -> "State":
        W = [np.asarray(w, dtype=np.float64).copy() for w in W0]
        return cls(W=W, m=[np.zeros((r, w.shape[1])) for w in W],
                   v=[np.zeros((r, w.shape[1])) for w in W])

    def copy(self) -> "State":
        return State([w.copy() for w in self.W], [m.copy() for m in self.m],
                     [v.copy() for v in self.v])


ProjectionFn = Callable[[int, int, int, int], np.ndarray]   # (layer, step, d_in, r) -> P


def default_projection(h: Hyper) -> ProjectionFn:
    return lambda layer, step, d_in, r: projection_matrix(h.seed, layer, h.projection_key(step), d_in, r)


def projected_per_sample(A: Sequence[np.ndarray], Gout: Sequence[np.ndarray],
                         Ps: Sequence[np.ndarray], samples: Sequence[int]):
    """R[i][l] = P_l^T (A_{i,l}^T Gout_{i,l}) for the given samples, G materialised.

    ``A[l]`` / ``Gout[l]`` are fp64 arrays of shape (B, T, d).
    """
    return {i: [project(Ps[l], per_sample_gradient(A[l][i], Gout[l][i]))
                for l in range(len(Ps))] for i in samples}


def step(state: State, A: Sequence[np.ndarray], Gout: Sequence[np.ndarray], step_index: int,
         h: Hyper, projection: Optional[ProjectionFn] = None,
         batch_divisor: Optional[int] = None) -> Dict[str, object]:
    """One DP-GRAPE step, in place on ``state``.  Returns the intermediate values.

    ``A[l]``, ``Gout[l]``: fp64, shape (B, T, d_in) and (B, T, d_out).
    ``step_index`` s is 0-based; Adam's bias correction uses t = s + 1.
    ``projection`` replaces the Philox projection (P = I reduces the method to
    plain DP-Adam).  ``batch_divisor`` replaces B in the average (a data-parallel
    shard divides by the global batch).
    """
    proj = projection or default_projection(h)
    L = len(state.W)
    B = A[0].shape[0]
    Ps = [proj(l, step_index, state.W[l].shape[0], h.r) for l in range(L)]

    # projection before privatization: every raw per-sample gradient is projected
    R = projected_per_sample(A, Gout, Ps, range(B))

    # per-sample norm over all layers, then the clip factor
    norms = np.array([np.sqrt(sum(np.sum(R[i][l] ** 2) for l in range(L))) for i in range(B)])
    c = np.array([clip_factor(n, h.C) for n in norms])

    S, dR = [], []
    t = step_index + 1
    div = B if batch_divisor is None else batch_divisor
    for l in range(L):
        # aggregate the clipped projected gradients
        S_l = sum(c[i] * R[i][l] for i in range(B))
        # Gaussian noise in the projected space, then the batch average (reading: divide by B)
        xi = noise_matrix(h.seed, l, step_index, h.r, state.W[l].shape[1]) if h.sigma != 0 \
            else np.zeros_like(S_l)
        g = (S_l + h.sigma * h.C * xi) / div
        # projected Adam
        state.m[l], state.v[l], d = adam(state.m[l], state.v[l], g, t, h.beta1, h.beta2, h.eps)
        # back to the parameter space with the same P
        state.W[l] = state.W[l] - h.lr * (Ps[l] @ d)
        S.append(S_l)
        dR.append(d)
    # the moments after this step (copies: the state is updated again by later steps)
    return {"P": Ps, "R": R, "norms": norms, "clip": c, "S": S, "dR": dR,
            "m": [m.copy() for m in state.m], "v": [v.copy() for v in state.v]}


def sample_norms(A: Sequence[np.ndarray], Gout: Sequence[np.ndarray], step_index: int,
                 h: Hyper, d_in: Sequence[int]) -> np.ndarray:
    """Per-sample projected norms only (spot checks at full size).

    ``A[l]`` / ``Gout[l]`` hold just the samples to check, fp64.
    """
    L = len(A)
    n = A[0].shape[0]
    tot = np.zeros(n)
    for l in range(L):
        P = projection_matrix(h.seed, l, h.projection_key(step_index), d_in[l], h.r)
        for j in range(n):
            tot[j] += float(np.sum(project(P, per_sample_gradient(A[l][j], Gout[l][j])) ** 2))
    return np.sqrt(tot)


# --------------------------------------------------------------------------
# Ghost norm of a projected per-sample gradient
#
# The technical summary of "Memory-Efficient Differentially Private Training with
# Gradient Random Projection" places DP-GRAPE as orthogonal to Ghost Clipping; the
# DP-SGD-RC summary gives Ghost Clipping's cost as O(B T^2 (p + d)) for a linear
# layer.  Ghost clipping evaluates ||X^T Y||_F^2 as <X X^T, Y Y^T>_F from two T x T
# Gram matrices, never forming X^T Y.  For DP-GRAPE, X = A_i P (T x r) and
# Y = Gout_i (T x d_out).
# --------------------------------------------------------------------------

def ghost_sqnorm(AP_i: np.ndarray, Gout_i: np.ndarray) -> float:
    """<(A_i P)(A_i P)^T, Gout_i Gout_i^T>_F, from the two T x T Gram matrices."""
    X = AP_i @ AP_i.T
    Y = Gout_i @ Gout_i.T
    return float(np.sum(X * Y))


# --------------------------------------------------------------------------
# Loss-token masks
#
# The pages are silent about masking: a mask is a property of the workload
# (tokens that carry no loss).  Reading: a masked token contributes nothing to
# the sample's gradient, exactly as if its output gradient row were zero; the
# gradient of a linear layer is a sum over tokens (A_i^T Gout_i = sum_t
# a_t^T g_t), so dropping such tokens is an exact rewrite, not an approximation.
# --------------------------------------------------------------------------

def apply_token_mask(Gout: Sequence[np.ndarray], mask: np.ndarray) -> List[np.ndarray]:
    """Gout_l with the rows of masked tokens set to zero; ``mask`` has shape (B, T), nonzero = kept."""
    keep = (np.asarray(mask) != 0)[:, :, None]
    return [np.where(keep, g, 0.0) for g in Gout]


# --------------------------------------------------------------------------
# Hutchinson estimate of a per-sample gradient norm (DP-SGD-RC)
#
# Source: "DP-SGD-RC" technical summary on the same site (gist.science,
# 2605.24879), sections "Metodología: DP-SGD-RC" (the trace identity and the
# Hutchinson estimator) and "Flujo Algorítmico" step 3 (the norm-estimation
# routine, applied per sample).  ||A^T G||_F^2 = tr(O) with O = (A^T G)(A^T G)^T;
# Hutchinson's estimator sums p_j^T O p_j over the k columns p_j of a Gaussian
# matrix.  Reading: the sketch acts on the activation width (d_in), and its
# entries are N(0, 1/k), the same scale as DP-GRAPE's P, so the sum is unbiased
# with no further factor.
# --------------------------------------------------------------------------

def hutchinson_sqnorm(A_i: np.ndarray, Gout_i: np.ndarray, P: np.ndarray) -> float:
    """sum_j P[:, j]^T O P[:, j] with O = G G^T, G = A_i^T Gout_i (d_in x d_out).

    O is formed explicitly (d_in x d_in, fp64): the definition written out, not
    the factored ||(A_i P)^T Gout_i||^2 that the kernels compute."""
    G = per_sample_gradient(A_i, Gout_i)
    O = G @ G.T
    return float(sum(P[:, j] @ O @ P[:, j] for j in range(P.shape[1])))


def hutchinson_sample_sqnorms(A: Sequence[np.ndarray], Gout: Sequence[np.ndarray], step_index: int,
                              h: Hyper, d_in: Sequence[int]) -> np.ndarray:
    """Per-sample estimate of sum_l ||A_{i,l}^T Gout_{i,l}||_F^2 with k = h.r sketch
    columns per layer, P_l drawn as DP-GRAPE draws it (key floor(s / K))."""
    L = len(A)
    n = A[0].shape[0]
    tot = np.zeros(n)
    for l in range(L):
        P = projection_matrix(h.seed, l, h.projection_key(step_index), d_in[l], h.r)
        for j in range(n):
            tot[j] += hutchinson_sqnorm(A[l][j], Gout[l][j], P)
    return tot


def run(workload, steps: int, samples: Optional[Sequence[int]] = None,
        stop_after: Optional[int] = None) -> Dict[str, object]:
    """Run ``steps`` steps of a workload from its seeded inputs.  Returns the final
    state and the per-step intermediates (test helper)."""
    import workloads as W

    h = Hyper.of(workload)
    state = State.init(W.make_weights(workload), workload.r)
    trace = []
    for s in range(steps):
        x = W.make_step_inputs(workload, s, samples=samples)
        A = [x.as_f64(a) for a in x.A]
        G = [x.as_f64(g) for g in x.Gout]
        trace.append(step(state, A, G, s, h))
        if stop_after is not None and s + 1 >= stop_after:
            break
    return {"state": state, "trace": trace}
