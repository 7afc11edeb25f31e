"""Properties of the fp64 oracle over random small shapes and hyper-parameters (CPU only).

The pins in tests/pins.py fix the oracle on chosen tiny problems; these draw the
shapes, r, C, sigma and the step with hypothesis and check what must hold for every
draw: every clipped sample ends at norm C, unclipped ones are untouched, the projection
computed through the materialised gradient equals the factored form, the no-privacy
limit is one stacked product, and Adam's first step is g / (|g| + eps).
"""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

import oracle.grape_oracle as O  # noqa: E402

SETTINGS = dict(max_examples=25, deadline=None, derandomize=True)


@st.composite
def problems(draw):
    n_layers = draw(st.integers(1, 3))
    layers = tuple((draw(st.integers(2, 9)), draw(st.integers(1, 8))) for _ in range(n_layers))
    r = draw(st.integers(1, min(d for d, _ in layers)))
    B, T = draw(st.integers(1, 5)), draw(st.integers(1, 6))
    seed = draw(st.integers(0, 2**32 - 1))
    rng = np.random.default_rng(seed)
    A = [rng.standard_normal((B, T, di)) for di, _ in layers]
    G = [rng.standard_normal((B, T, do)) * draw(st.floats(0.05, 3.0)) for _, do in layers]
    W0 = [0.02 * rng.standard_normal((di, do)) for di, do in layers]
    return layers, r, A, G, W0, seed


@settings(**SETTINGS)
@given(problems(), st.floats(0.05, 5.0), st.floats(0.0, 2.0), st.integers(0, 1000))
def test_clip_takes_every_sample_to_at_most_C(prob, C, sigma, step):
    layers, r, A, G, W0, seed = prob
    h = O.Hyper(r=r, C=C, sigma=sigma, seed=seed)
    out = O.step(O.State.init(W0, r), A, G, step, h)
    n, c = out["norms"], out["clip"]
    clipped = np.array([np.sqrt(sum(np.sum((c[i] * out["R"][i][l]) ** 2) for l in range(len(layers))))
                        for i in range(len(n))])
    assert np.all(clipped <= C * (1 + 1e-12))
    assert np.all(c[n <= C] == 1.0)
    assert np.allclose(clipped[n > C], C, rtol=1e-12)


@settings(**SETTINGS)
@given(problems(), st.integers(0, 1000))
def test_projection_through_the_gradient_equals_the_factored_form(prob, step):
    layers, r, A, G, W0, seed = prob
    for l, (di, _) in enumerate(layers):
        P = O.projection_matrix(seed, l, step, di, r)
        for i in range(A[l].shape[0]):
            direct = O.project(P, O.per_sample_gradient(A[l][i], G[l][i]))
            factored = (A[l][i] @ P).T @ G[l][i]
            assert np.allclose(direct, factored, rtol=1e-11, atol=1e-12)


@settings(**SETTINGS)
@given(problems(), st.integers(0, 1000))
def test_no_clipping_no_noise_is_one_stacked_product(prob, step):
    layers, r, A, G, W0, seed = prob
    h = O.Hyper(r=r, C=1e300, sigma=0.0, seed=seed)
    out = O.step(O.State.init(W0, r), A, G, step, h)
    for l, (di, do) in enumerate(layers):
        P = O.projection_matrix(seed, l, step, di, r)
        stacked = P.T @ (A[l].reshape(-1, di).T @ G[l].reshape(-1, do))
        assert np.allclose(out["S"][l], stacked, rtol=1e-11, atol=1e-12)


@settings(**SETTINGS)
@given(st.integers(1, 6), st.integers(1, 6), st.integers(0, 2**31), st.floats(1e-10, 1e-3))
def test_first_adam_step_is_the_sign_like_direction(rows, cols, seed, eps):
    g = np.random.default_rng(seed).standard_normal((rows, cols))
    m, v, d = O.adam(np.zeros_like(g), np.zeros_like(g), g, 1, 0.9, 0.999, eps)
    assert np.allclose(d, g / (np.abs(g) + eps), rtol=1e-10, atol=0)
    assert np.allclose(m, 0.1 * g, rtol=1e-14) and np.allclose(v, 0.001 * g * g, rtol=1e-12)
