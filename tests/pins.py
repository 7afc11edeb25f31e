"""Pins of the fp64 oracle against things other than itself.

Each ``pin_*`` takes the oracle module and raises ``AssertionError`` when the
oracle disagrees with an independent source: torch's own Philox engine
(compiled from its header), torch autograd + ``torch.optim.Adam`` (plain
DP-Adam when P = I), brute-force loops, closed forms and statistical
properties.  ``test_oracle_pins.py`` runs them on the oracle as it is;
``test_oracle_mutations.py`` plants plausible mistakes in the oracle and
checks that every mistake fails at least one pin.
"""
from __future__ import annotations

import functools
import math
import os
import subprocess
import tempfile

import numpy as np

# --------------------------------------------------------------------------
# torch's ATen Philox engine (BSD, header-only) compiled on the host
# --------------------------------------------------------------------------
_ATEN_MAIN = r"""
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
#include <cstdint>
int main() {
  unsigned long long seed, offset, subseq;
  while (std::scanf("%llu %llu %llu", &seed, &offset, &subseq) == 3) {
    at::philox_engine e(seed, subseq, offset);
    unsigned a = e(), b = e(), c = e(), d = e();
    std::printf("%u %u %u %u\n", a, b, c, d);
  }
  return 0;
}
"""


@functools.lru_cache(maxsize=1)
def aten_philox_binary() -> str:
    import torch
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    d = tempfile.mkdtemp(prefix="aten_philox_")
    src = os.path.join(d, "main.cpp")
    exe = os.path.join(d, "aten_philox")
    with open(src, "w") as f:
        f.write(_ATEN_MAIN)
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", inc, src, "-o", exe], check=True,
                   capture_output=True)
    return exe


def aten_philox(seed: int, offsets, subseqs) -> np.ndarray:
    """ATen philox_engine(seed, subsequence, offset): the four words of its first block.

    ATen's counter is (offset lo, offset hi, subsequence lo, subsequence hi) and
    its key is (seed lo, seed hi).
    """
    lines = "".join(f"{seed} {o} {s}\n" for o, s in zip(offsets, subseqs))
    out = subprocess.run([aten_philox_binary()], input=lines, capture_output=True, text=True,
                         check=True).stdout
    return np.array([[int(x) for x in ln.split()] for ln in out.strip().splitlines()],
                    dtype=np.uint64).astype(np.uint32)


def pin_philox_vs_aten(O):
    """Our counter (q, layer, step, stream) is ATen's offset q + layer*2^32 and
    subsequence step + stream*2^32; the words must agree bit for bit, both through
    the oracle's counter layout (first blocks) and for arbitrary 32-bit q."""
    rng = np.random.default_rng(1)
    for seed in (0, 1, 0x0123456789ABCDEF, 2**64 - 1):
        for layer, step, stream in ((0, 0, 0), (3, 7, 1), (27, 12345, 0), (2**32 - 1, 2**31, 1)):
            q = np.arange(6, dtype=np.uint64)
            ours = O.philox_words(seed, layer, step, stream, 6)
            theirs = aten_philox(seed, [int(x) + (layer << 32) for x in q],
                                 [step + (stream << 32)] * len(q))
            assert np.array_equal(ours, theirs), (seed, layer, step, stream)
            q = rng.integers(0, 2**32, 6, dtype=np.uint64)
            ctr = np.zeros((len(q), 4), dtype=np.uint32)
            ctr[:, 0] = q.astype(np.uint32)
            ctr[:, 1], ctr[:, 2], ctr[:, 3] = layer, step, stream
            ours = O.philox4x32_10(ctr, (seed & 0xFFFFFFFF, seed >> 32))
            theirs = aten_philox(seed, [int(x) + (layer << 32) for x in q],
                                 [step + (stream << 32)] * len(q))
            assert np.array_equal(ours, theirs), (seed, layer, step, stream, "random q")


# --------------------------------------------------------------------------
# Box-Muller normals
# --------------------------------------------------------------------------

def pin_box_muller_definition(O):
    """Elements 4q..4q+3 follow the stated pairing: (x0, x1) -> cos, sin; (x2, x3) -> cos, sin,
    with u1 = (x+1)/2^32 and u2 = x/2^32 (checked with Python's math module on ATen's words)."""
    seed, layer, step, stream = 42, 2, 5, 1
    z = O.gaussian_stream(seed, layer, step, stream, 40)
    w = aten_philox(seed, [q + (layer << 32) for q in range(10)], [step + (stream << 32)] * 10)
    for q in range(10):
        for pair in (0, 1):
            xa, xb = int(w[q, 2 * pair]), int(w[q, 2 * pair + 1])
            rho = math.sqrt(-2.0 * math.log((xa + 1) / 2**32))
            ang = 2 * math.pi * (xb / 2**32)
            assert abs(z[4 * q + 2 * pair] - rho * math.cos(ang)) < 1e-12
            assert abs(z[4 * q + 2 * pair + 1] - rho * math.sin(ang)) < 1e-12


def pin_normal_statistics(O):
    """10^6 draws: mean, variance, KS distance to the standard normal CDF, and no
    correlation between the cosine and sine halves of a pair."""
    from scipy import stats
    n = 1 << 20
    z = O.gaussian_stream(7, 1, 3, 0, n)
    assert abs(z.mean()) < 5 / math.sqrt(n)
    assert abs(z.var() - 1) < 5 * math.sqrt(2 / n)
    ks = stats.kstest(z, "norm")
    assert ks.pvalue > 1e-4, ks
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 5 / math.sqrt(n / 2)
    # different streams and layers are not the same numbers
    z2 = O.gaussian_stream(7, 1, 3, 1, 1024)
    z3 = O.gaussian_stream(7, 2, 3, 0, 1024)
    assert abs(np.corrcoef(z[:1024], z2)[0, 1]) < 0.2 and abs(np.corrcoef(z[:1024], z3)[0, 1]) < 0.2


# --------------------------------------------------------------------------
# projection
# --------------------------------------------------------------------------

def pin_projection_scale(O):
    """E ||P^T x||^2 = ||x||^2 (Johnson-Lindenstrauss scaling of an N(0, 1/r) matrix)."""
    rng = np.random.default_rng(3)
    d_in, r = 96, 16
    ratios = []
    for step in range(200):
        P = O.projection_matrix(11, 0, step, d_in, r)
        assert P.shape == (d_in, r)
        x = rng.standard_normal(d_in)
        ratios.append(np.sum((P.T @ x) ** 2) / np.sum(x ** 2))
    # each ratio ~ chi2_r / r: mean 1, sd sqrt(2/r)/sqrt(200)
    assert abs(np.mean(ratios) - 1) < 5 * math.sqrt(2 / r) / math.sqrt(200)


def pin_projection_layout(O):
    """P is the row-major reshape of the projection stream, scaled by 1/sqrt(r), and
    is regenerated bit-identically from (seed, layer, step)."""
    d_in, r = 10, 6
    P = O.projection_matrix(5, 4, 9, d_in, r)
    z = O.gaussian_stream(5, 4, 9, 0, d_in * r)
    for k in range(d_in):
        for j in range(r):
            assert P[k, j] == z[k * r + j] / math.sqrt(r)
    assert np.array_equal(P, O.projection_matrix(5, 4, 9, d_in, r))
    assert not np.array_equal(P, O.projection_matrix(5, 4, 10, d_in, r))
    xi = O.noise_matrix(5, 4, 9, r, 7)
    zn = O.gaussian_stream(5, 4, 9, 1, r * 7)
    assert xi.shape == (r, 7) and xi[2, 3] == zn[2 * 7 + 3]


def pin_factored_bruteforce(O):
    """(A_i P)^T Gout_i computed with explicit loops equals the oracle's P^T (A_i^T Gout_i)."""
    rng = np.random.default_rng(4)
    T, d_in, d_out, r = 5, 7, 4, 3
    A = rng.standard_normal((T, d_in))
    G = rng.standard_normal((T, d_out))
    P = O.projection_matrix(1, 0, 0, d_in, r)
    AP = [[sum(A[t][k] * P[k][j] for k in range(d_in)) for j in range(r)] for t in range(T)]
    R_loop = [[sum(AP[t][j] * G[t][n] for t in range(T)) for n in range(d_out)] for j in range(r)]
    R = O.project(P, O.per_sample_gradient(A, G))
    assert np.allclose(R, np.array(R_loop), rtol=1e-12, atol=1e-12)
    # and the per-sample gradient itself is sum_t a_t g_t^T
    Gi = O.per_sample_gradient(A, G)
    for k in range(d_in):
        for n in range(d_out):
            assert abs(Gi[k, n] - sum(A[t, k] * G[t, n] for t in range(T))) < 1e-12


# --------------------------------------------------------------------------
# the step
# --------------------------------------------------------------------------

def _tiny_problem(seed=0, B=5, T=6, layers=((9, 4), (5, 7)), scale=0.3):
    rng = np.random.default_rng(seed)
    A = [rng.standard_normal((B, T, di)) for di, _ in layers]
    s = np.exp(rng.standard_normal(B))
    G = [scale * s[:, None, None] * rng.standard_normal((B, T, do)) for _, do in layers]
    W0 = [0.02 * rng.standard_normal((di, do)) for di, do in layers]
    return A, G, W0


def pin_identity_projection_is_dp_adam(O):
    """With P = I (r = d_in) the step is plain DP-Adam: per-sample gradients from torch
    autograd, clipped by their norm over all layers, summed, noised with sigma*C*xi,
    averaged over B and fed to torch.optim.Adam.  Three steps, C != 1, sigma != 0."""
    import torch
    layers = ((6, 4), (6, 3))           # equal d_in so a single r = d_in works
    B, T = 4, 5
    A, G, W0 = _tiny_problem(1, B, T, layers, scale=0.6)
    h = O.Hyper(r=6, C=0.7, sigma=0.9, seed=3, lr=1e-2, beta1=0.8, beta2=0.95, eps=1e-6)
    ident = lambda layer, step, d_in, r: np.eye(d_in)
    st = O.State.init(W0, h.r)

    Wt = [torch.tensor(w, dtype=torch.float64, requires_grad=True) for w in W0]
    opt = torch.optim.Adam(Wt, lr=h.lr, betas=(h.beta1, h.beta2), eps=h.eps)
    for s in range(3):
        # fresh inputs each step
        A, G, _ = _tiny_problem(10 + s, B, T, layers, scale=0.6)
        O.step(st, A, G, s, h, projection=ident)
        # independent DP-Adam
        per_sample = []
        for i in range(B):
            loss = sum((torch.tensor(A[l][i]) @ Wt[l] * torch.tensor(G[l][i])).sum()
                       for l in range(len(layers)))
            per_sample.append(torch.autograd.grad(loss, Wt))
        flat = [torch.cat([g.reshape(-1) for g in gi]) for gi in per_sample]
        norms = torch.stack([f.norm() for f in flat])
        c = torch.clamp(h.C / norms, max=1.0)
        opt.zero_grad()
        for l, w in enumerate(Wt):
            tot = sum(c[i] * per_sample[i][l] for i in range(B))
            xi = torch.tensor(O.noise_matrix(h.seed, l, s, layers[l][0], layers[l][1]))
            w.grad = (tot + h.sigma * h.C * xi) / B
        opt.step()
    for l in range(len(layers)):
        assert np.allclose(st.W[l], Wt[l].detach().numpy(), rtol=0, atol=1e-12), l
        exp_avg = opt.state[Wt[l]]["exp_avg"].numpy()
        exp_avg_sq = opt.state[Wt[l]]["exp_avg_sq"].numpy()
        assert np.allclose(st.m[l], exp_avg, rtol=1e-12, atol=1e-15)
        assert np.allclose(st.v[l], exp_avg_sq, rtol=1e-12, atol=1e-18)


def pin_clipping_bound(O):
    """Every clipped per-sample projected gradient has norm <= C, unclipped samples
    keep factor 1, and the norm is taken over all layers together."""
    A, G, W0 = _tiny_problem(2, B=7, scale=0.5)
    probe = O.step(O.State.init(W0, 3), A, G, 0, O.Hyper(r=3, C=1e300, sigma=0.0, seed=1))
    C = float(np.median(probe["norms"]))          # splits the batch into clipped / kept
    h = O.Hyper(r=3, C=C, sigma=0.0, seed=1)
    st = O.State.init(W0, h.r)
    out = O.step(st, A, G, 0, h)
    R, c, n = out["R"], out["clip"], out["norms"]
    assert (c < 1).any() and (c == 1).any()
    for i in range(len(c)):
        tot = math.sqrt(sum(float(np.sum((c[i] * R[i][l]) ** 2)) for l in range(len(W0))))
        assert tot <= h.C * (1 + 1e-12)
        nl = math.sqrt(sum(float(np.sum(R[i][l] ** 2)) for l in range(len(W0))))
        assert abs(nl - n[i]) < 1e-12 * max(1.0, nl)
        if n[i] <= h.C:
            assert c[i] == 1.0
        else:
            assert abs(tot - h.C) < 1e-12


def pin_sigma_zero(O):
    """sigma = 0: no noise, deterministic, and the averaged gradient is (sum_i c_i R_i)/B."""
    A, G, W0 = _tiny_problem(3)
    h = O.Hyper(r=3, C=0.5, sigma=0.0, seed=2, eps=1e-30)
    s1, s2 = O.State.init(W0, h.r), O.State.init(W0, h.r)
    o1, o2 = O.step(s1, A, G, 0, h), O.step(s2, A, G, 0, h)
    B = A[0].shape[0]
    for l in range(len(W0)):
        assert np.array_equal(s1.W[l], s2.W[l])
        S = sum(o1["clip"][i] * o1["R"][i][l] for i in range(B))
        assert np.allclose(o1["S"][l], S, rtol=1e-14, atol=0)
        # t = 1: m = (1 - beta1) g with g = S / B
        assert np.allclose(s1.m[l], (1 - h.beta1) * S / B, rtol=1e-12, atol=0)


def pin_adam_first_step(O):
    """At t = 1 Adam's bias-corrected direction is g / (|g| + eps) elementwise."""
    g = np.array([[0.3, -2e-3, 5.0], [-7.0, 1e-9, 0.0]])
    m, v, d = O.adam(np.zeros_like(g), np.zeros_like(g), g, 1, 0.9, 0.999, 1e-8)
    assert np.allclose(d, g / (np.abs(g) + 1e-8), rtol=1e-12, atol=0)
    assert np.allclose(m, 0.1 * g) and np.allclose(v, 0.001 * g * g)


def pin_no_privacy_reduction(O):
    """C = infinity and sigma = 0: S_l = P_l^T (A_stacked^T Gout_stacked), one GEMM over all
    B*T stacked rows (computed here with einsum on the stacked tensors)."""
    A, G, W0 = _tiny_problem(5)
    h = O.Hyper(r=4, C=1e300, sigma=0.0, seed=8)
    st = O.State.init(W0, h.r)
    out = O.step(st, A, G, 2, h)
    for l in range(len(W0)):
        P = O.projection_matrix(h.seed, l, 2, W0[l].shape[0], h.r)
        S = np.einsum("kj,btk,btn->jn", P, A[l], G[l])
        assert np.allclose(out["S"][l], S, rtol=1e-12, atol=1e-14)


def pin_backprojection_unbiased(O):
    """With eps much larger than |g| Adam's first step is linear (d ~ g/eps), so the
    weight change is -lr/eps * P P^T (sum_i G_i)/B.  Averaged over many draws of P it
    must approach -lr/eps * (sum_i G_i)/B (E[P P^T] = I): this pins that the
    back-projection uses the same P as the projection, and the 1/r variance."""
    rng = np.random.default_rng(6)
    B, T, d_in, d_out, r = 3, 4, 6, 3, 4
    A = [rng.standard_normal((B, T, d_in))]
    G = [rng.standard_normal((B, T, d_out))]
    eps, lr = 1e6, 1.0
    full = sum(A[0][i].T @ G[0][i] for i in range(B)) / B
    acc = np.zeros((d_in, d_out))
    n = 4000
    for seed in range(n):           # a fresh P per seed, always at t = 1
        h = O.Hyper(r=r, C=1e300, sigma=0.0, seed=seed, lr=lr, eps=eps)
        st = O.State.init([np.zeros((d_in, d_out))], r)
        O.step(st, A, G, 0, h)
        acc += st.W[0]
    mean = acc / n
    # t = 1: d = g / (|g| + eps) ~ g / eps; W = -lr * P d
    target = -lr / eps * full
    err = np.linalg.norm(mean - target) / np.linalg.norm(target)
    assert err < 0.1, err


def pin_projection_before_privatization(O):
    """The pages' ordering matters: privatizing (clipping) the full gradient first and
    projecting afterwards gives a different aggregate than the oracle's order."""
    A, G, W0 = _tiny_problem(7, scale=1.0)
    h = O.Hyper(r=2, C=0.3, sigma=0.0, seed=4)
    st = O.State.init(W0, h.r)
    out = O.step(st, A, G, 0, h)
    B = A[0].shape[0]
    full = [[O.per_sample_gradient(A[l][i], G[l][i]) for l in range(len(W0))] for i in range(B)]
    nfull = [math.sqrt(sum(float(np.sum(g ** 2)) for g in full[i])) for i in range(B)]
    naive = [sum(min(1.0, h.C / nfull[i]) * O.project(out["P"][l], full[i][l]) for i in range(B))
             for l in range(len(W0))]
    assert not np.allclose(naive[0], out["S"][0], rtol=1e-3)


# --------------------------------------------------------------------------
# projection-refresh period K
# --------------------------------------------------------------------------

def _rank(M, tol=1e-9):
    sv = np.linalg.svd(M, compute_uv=False)
    return int(np.sum(sv > tol * sv[0]))


def pin_refresh_fixed_subspace(O):
    """K >= number of steps keeps one P for the whole run, so W_T - W_0 = -lr P sum_s dR_s
    has rank <= r (the GaLore-style fixed subspace); with K = 1 a fresh P every step lets
    the rank grow past r.  A property of the update, not of the key arithmetic."""
    layers = ((12, 10),)
    B, T, steps, r = 3, 4, 4, 2
    h_fixed = O.Hyper(r=r, C=1e9, sigma=0.0, seed=5, lr=1e-2, refresh=steps)
    h_fresh = O.Hyper(r=r, C=1e9, sigma=0.0, seed=5, lr=1e-2, refresh=1)
    _, _, W0 = _tiny_problem(0, B, T, layers)
    st_fixed, st_fresh = O.State.init(W0, r), O.State.init(W0, r)
    for s in range(steps):
        A, G, _ = _tiny_problem(20 + s, B, T, layers, scale=0.5)
        O.step(st_fixed, A, G, s, h_fixed)
        O.step(st_fresh, A, G, s, h_fresh)
    assert _rank(st_fixed.W[0] - W0[0]) <= r
    assert _rank(st_fresh.W[0] - W0[0]) > r


def pin_refresh_period_two(O):
    """K = 2: steps 0 and 1 project with the same P, step 2 with another, and the noise
    still changes every step."""
    A, G, W0 = _tiny_problem(3)
    h = O.Hyper(r=2, C=0.5, sigma=1.0, seed=8, refresh=2)
    st = O.State.init(W0, h.r)
    P = [O.step(st, A, G, s, h)["P"][0] for s in range(3)]
    assert np.array_equal(P[0], P[1]) and not np.allclose(P[1], P[2])
    assert not np.allclose(O.noise_matrix(h.seed, 0, 0, 2, 4), O.noise_matrix(h.seed, 0, 1, 2, 4))
    # the noise the step itself adds, recovered from a first Adam step (m = (1 - beta1) g,
    # g = (S + sigma C xi) / B): stream 1 keyed on the step, not on the refresh key, so
    # the two steps of one period draw different noise
    B = A[0].shape[0]
    xi = []
    for s in (0, 1):
        st = O.State.init(W0, h.r)
        out = O.step(st, A, G, s, h)
        for l in range(len(W0)):
            got = (B * st.m[l] / (1.0 - h.beta1) - out["S"][l]) / (h.sigma * h.C)
            assert np.allclose(got, O.noise_matrix(h.seed, l, s, h.r, W0[l].shape[1]), rtol=1e-9, atol=1e-9)
        xi.append(got)
    assert not np.allclose(xi[0], xi[1])


def pin_spot_check_norms_match_the_step(O):
    """The full-size parity tests recompute a few samples' norms with ``sample_norms`` and
    compare ``grape_sqnorms`` with ``hutchinson_sample_sqnorms``.  On a subset of samples,
    under a refresh period (step 3, K = 2, so the key differs from the step), the first
    must equal the norms the step computes, and the second, with k = r sketch columns
    drawn as DP-GRAPE draws P, their squares (sum_j p_j^T G G^T p_j = ||P^T G||_F^2)."""
    A, G, W0 = _tiny_problem(41, B=5)
    h = O.Hyper(r=3, C=0.5, sigma=0.7, seed=12, refresh=2)
    out = O.step(O.State.init(W0, h.r), A, G, 3, h)
    pick = [0, 2, 4]
    sub_A = [a[pick] for a in A]
    sub_G = [g[pick] for g in G]
    d_in = [w.shape[0] for w in W0]
    n = O.sample_norms(sub_A, sub_G, 3, h, d_in)
    assert np.allclose(n, out["norms"][pick], rtol=1e-12, atol=0)
    sq = O.hutchinson_sample_sqnorms(sub_A, sub_G, 3, h, d_in)
    assert np.allclose(sq, out["norms"][pick] ** 2, rtol=1e-10, atol=0)


# --------------------------------------------------------------------------
# ghost norm
# --------------------------------------------------------------------------

def pin_ghost_norm_equals_projected_norm(O):
    """<(AP)(AP)^T, G G^T>_F equals ||(AP)^T G||_F^2 computed with loops (the trace identity
    tr(M^T M) for M = (AP)^T G, here written out element by element)."""
    rng = np.random.default_rng(41)
    A, G, P = rng.standard_normal((5, 6)), rng.standard_normal((5, 4)), rng.standard_normal((6, 3))
    AP = A @ P
    direct = 0.0
    for j in range(3):
        for n in range(4):
            acc = sum(AP[t, j] * G[t, n] for t in range(5))
            direct += acc * acc
    assert math.isclose(O.ghost_sqnorm(AP, G), direct, rel_tol=1e-12)


def pin_ghost_norm_with_identity_is_gradient_norm(O):
    """With P = I the ghost norm is the textbook ghost-clipping norm of the full per-sample
    gradient: <A A^T, G G^T>_F = ||A^T G||_F^2 of the materialised gradient."""
    rng = np.random.default_rng(42)
    A, G = rng.standard_normal((7, 5)), rng.standard_normal((7, 3))
    full = float(np.sum(O.per_sample_gradient(A, G) ** 2))
    assert math.isclose(O.ghost_sqnorm(A @ np.eye(5), G), full, rel_tol=1e-12)


# --------------------------------------------------------------------------
# token masks
# --------------------------------------------------------------------------

def pin_masked_tokens_drop_out(O):
    """A step on masked inputs equals the step on each sample's kept tokens alone, moved
    to the front and zero-padded to a shorter T: the gradient is a sum over tokens, so
    the step may not depend on T or on where the dropped tokens were."""
    layers = ((7, 5), (6, 4))
    B, T, T_cap = 3, 9, 5
    A, G, W0 = _tiny_problem(31, B, T, layers, scale=0.8)
    rng = np.random.default_rng(32)
    mask = rng.random((B, T)) < 0.45
    mask[0, :] = False                        # a sample with no live token
    mask[1, :T_cap] = True; mask[1, T_cap:] = False   # one exactly at the capacity
    h = O.Hyper(r=3, C=0.6, sigma=0.7, seed=9)
    st_full = O.State.init(W0, h.r)
    out_full = O.step(st_full, A, O.apply_token_mask(G, mask), 0, h)
    Ac = [np.zeros((B, T_cap, a.shape[2])) for a in A]
    Gc = [np.zeros((B, T_cap, g.shape[2])) for g in G]
    for i in range(B):
        live = np.flatnonzero(mask[i])
        assert len(live) <= T_cap
        for l in range(len(layers)):
            Ac[l][i, :len(live)] = A[l][i, live]
            Gc[l][i, :len(live)] = G[l][i, live]
    st_c = O.State.init(W0, h.r)
    out_c = O.step(st_c, Ac, Gc, 0, h)
    assert np.allclose(out_full["norms"], out_c["norms"], rtol=1e-12, atol=0)
    assert out_full["norms"][0] == 0.0 and out_full["clip"][0] == 1.0
    for l in range(len(layers)):
        assert np.allclose(st_full.W[l], st_c.W[l], rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# Hutchinson norm estimate (DP-SGD-RC)
# --------------------------------------------------------------------------

def pin_hutchinson_identity_sketch(O):
    """With the identity as the sketch (k = d_in columns e_j) the estimator is the trace
    itself: exactly ||A^T G||_F^2."""
    rng = np.random.default_rng(11)
    A, G = rng.standard_normal((5, 7)), rng.standard_normal((5, 3))
    exact = float(np.sum((A.T @ G) ** 2))
    assert math.isclose(O.hutchinson_sqnorm(A, G, np.eye(7)), exact, rel_tol=1e-12)


def pin_hutchinson_unbiased(O):
    """Gaussian sketch with N(0, 1/k) entries: the mean of N independent estimates is within
    4 standard deviations of ||A^T G||_F^2, the variance of one estimate being
    2 ||O||_F^2 / k for O = (A^T G)(A^T G)^T."""
    rng = np.random.default_rng(12)
    A, G = rng.standard_normal((6, 9)), rng.standard_normal((6, 4))
    Gm = A.T @ G
    exact = float(np.sum(Gm ** 2))
    k, N = 3, 4000
    est = np.array([O.hutchinson_sqnorm(A, G, rng.standard_normal((9, k)) / math.sqrt(k)) for _ in range(N)])
    sd = math.sqrt(2.0 * float(np.sum((Gm @ Gm.T) ** 2)) / k / N)
    assert abs(est.mean() - exact) < 4 * sd, (est.mean(), exact, sd)
    # and the spread matches the closed form (within 10 %)
    assert abs(est.std() / math.sqrt(2.0 * float(np.sum((Gm @ Gm.T) ** 2)) / k) - 1) < 0.1


def pin_hutchinson_factored(O):
    """The explicit-O estimator equals ||(A P)^T G||_F^2 computed with loops, the factored
    form the per-sample norm kernels evaluate."""
    rng = np.random.default_rng(13)
    A, G, P = rng.standard_normal((4, 6)), rng.standard_normal((4, 5)), rng.standard_normal((6, 3))
    f = 0.0
    for j in range(3):
        for n in range(5):
            acc = 0.0
            for t in range(4):
                ap = sum(A[t, q] * P[q, j] for q in range(6))
                acc += ap * G[t, n]
            f += acc * acc
    assert math.isclose(O.hutchinson_sqnorm(A, G, P), f, rel_tol=1e-12)


ALL_PINS = [
    pin_philox_vs_aten, pin_box_muller_definition, pin_normal_statistics,
    pin_projection_scale, pin_projection_layout, pin_factored_bruteforce,
    pin_identity_projection_is_dp_adam, pin_clipping_bound, pin_sigma_zero,
    pin_adam_first_step, pin_no_privacy_reduction, pin_backprojection_unbiased,
    pin_projection_before_privatization, pin_refresh_fixed_subspace, pin_refresh_period_two,
    pin_spot_check_norms_match_the_step,
    pin_hutchinson_identity_sketch, pin_hutchinson_unbiased, pin_hutchinson_factored,
    pin_masked_tokens_drop_out, pin_ghost_norm_equals_projected_norm,
    pin_ghost_norm_with_identity_is_gradient_norm,
]
