"""The seeded input recipe shared by the oracle, the tests and the bench (CPU only).

The full-size GPU tests recompute a few samples with the oracle from a sub-batch of the
inputs, and the clip decisions are only meaningful when about half the samples exceed
C.  These tests pin both properties, the bf16 rounding of the inputs, and determinism.
"""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W

torch = pytest.importorskip("torch")


def _small_masked():
    return W.scaled(W.get("longctx"), layers=((64, 256), (32, 512)), B=6, T=300)


def test_a_sub_batch_is_the_matching_rows_of_the_full_batch():
    w = _small_masked()
    full = W.make_step_inputs(w, 2)
    pick = [4, 1, 5]
    sub = W.make_step_inputs(w, 2, samples=pick)
    for l in range(w.n_layers):
        assert np.array_equal(sub.A[l], full.A[l][pick])
        assert np.array_equal(sub.Gout[l], full.Gout[l][pick])
    assert np.array_equal(sub.mask, full.mask[pick]) and np.array_equal(sub.scale, full.scale[pick])


def test_threads_do_not_change_the_draw_and_steps_differ():
    w = W.scaled(W.get("mlp4x1024"), layers=((128, 256),), B=5, T=24)
    a, b = W.make_step_inputs(w, 3), W.make_step_inputs(w, 3, threads=4)
    assert np.array_equal(a.A[0], b.A[0]) and np.array_equal(a.Gout[0], b.Gout[0])
    c = W.make_step_inputs(w, 4)
    assert not np.array_equal(a.A[0], c.A[0]) and not np.array_equal(a.Gout[0], c.Gout[0])
    assert all(np.array_equal(x, y) for x, y in zip(W.make_weights(w), W.make_weights(w)))


def test_bf16_rounding_is_round_to_nearest_even_like_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 20000),
        # exact ties between two bf16 neighbours: the low 16 bits are 0x8000
        (np.arange(1, 2001, dtype=np.uint32) << 16 | np.uint32(0x8000)).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40], dtype=np.float32),
    ])
    ours = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # and widening is exact
    back = W.bf16_bits_to_f32(ours)
    assert np.array_equal(torch.from_numpy(back).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16),
                          ours)


def test_kappa_puts_the_median_projected_norm_at_C_times_the_sample_scale():
    """E ||A^T Z||_F^2 = T d_in d_out for independent unit normals, and E[P P^T] = I,
    so the projected norm of sample i concentrates at C s_i; with median(s_i) = 1 about
    half of the samples are clipped."""
    w = W.Workload("kappa", ((48, 40), (24, 56)), r=16, B=240, T=12, dtype="f32", C=0.7,
                   sigma=1.0, steps=1, scale_sigma=1.0)
    x = W.make_step_inputs(w, 0)
    h = O.Hyper.of(w)
    n = O.sample_norms([x.as_f64(a) for a in x.A], [x.as_f64(g) for g in x.Gout], 0, h,
                       [di for di, _ in w.layers])
    ratio = n / (w.C * x.scale.astype(np.float64))
    assert 0.85 < np.median(ratio) < 1.1
    assert 0.3 < np.mean(n > w.C) < 0.7


def test_the_loss_mask_keeps_the_stated_fraction_and_zeroes_gout_rows():
    w = W.scaled(W.get("longctx"), layers=((8, 256),), B=8, T=8192)
    x = W.make_step_inputs(w, 1)
    assert abs(x.mask.mean() - w.mask_p) < 0.01
    g = x.as_f64(x.Gout[0])
    assert np.all(g[x.mask == 0] == 0.0)
    assert np.all(np.any(g[x.mask != 0] != 0.0, axis=-1))


def test_sizes():
    w = W.get("mlp4x1024")
    assert w.input_bytes() == 4 * 64 * 128 * 2048 * 2 == 134_217_728
    assert w.state_bytes() == 4 * (4 * 1024 * 1024 + 8 * 128 * 1024)
