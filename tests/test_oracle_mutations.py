"""Plant plausible mistakes in (a copy of) the oracle and check that a pin catches each.

Each mutation replaces one exact fragment of ``oracle/grape_oracle.py`` and
executes the result as a fresh module on the CPU; the real oracle is never
modified.  A mutation passes this test when at least one pin in
``pins.ALL_PINS`` fails (an assertion or any exception) on the mutated copy.
"""
import itertools
import os
import sys
import types

import pytest

import pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "grape_oracle.py")

MUTATIONS = {
    # Philox
    "philox_multiplier": ("PHILOX_M0 = 0xD2511F53", "PHILOX_M0 = 0xD2511F55"),
    "philox_rounds": ("PHILOX_ROUNDS = 10", "PHILOX_ROUNDS = 9"),
    "philox_weyl": ("k1 = (k1 + np.uint64(PHILOX_W1))", "k1 = (k1 + np.uint64(PHILOX_W0))"),
    "philox_round_mix": ("c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]",
                         "c = [hi0 ^ c[1] ^ k0, lo1, hi1 ^ c[3] ^ k1, lo0]"),
    "counter_layout": ("ctr[:, 1] = np.uint32(layer)\n    ctr[:, 2] = np.uint32(step)",
                       "ctr[:, 1] = np.uint32(step)\n    ctr[:, 2] = np.uint32(layer)"),
    # Box-Muller
    "bm_open_interval": ("u1 = (xa.astype(np.float64) + 1.0)", "u1 = (xa.astype(np.float64) + 0.5)"),
    "bm_sin_cos_swap": ("return rho * np.cos(2.0 * np.pi * u2), rho * np.sin(2.0 * np.pi * u2)",
                        "return rho * np.sin(2.0 * np.pi * u2), rho * np.cos(2.0 * np.pi * u2)"),
    "bm_half_angle": ("return rho * np.cos(2.0 * np.pi * u2), rho * np.sin(2.0 * np.pi * u2)",
                      "return rho * np.cos(np.pi * u2), rho * np.sin(np.pi * u2)"),
    "bm_pairing": ("z2, z3 = box_muller(w[:, 2], w[:, 3])", "z2, z3 = box_muller(w[:, 3], w[:, 2])"),
    # projection matrix
    "p_unscaled": ("STREAM_PROJECTION, d_in * r).reshape(d_in, r) / np.sqrt(r)",
                   "STREAM_PROJECTION, d_in * r).reshape(d_in, r)"),
    "p_scaled_by_r": ("STREAM_PROJECTION, d_in * r).reshape(d_in, r) / np.sqrt(r)",
                      "STREAM_PROJECTION, d_in * r).reshape(d_in, r) / r"),
    "p_column_major": ("STREAM_PROJECTION, d_in * r).reshape(d_in, r) / np.sqrt(r)",
                       "STREAM_PROJECTION, d_in * r).reshape(r, d_in).T / np.sqrt(r)"),
    "noise_stream": ("STREAM_NOISE, r * d_out)", "STREAM_PROJECTION, r * d_out)"),
    # gradient and projection
    "grad_token_misaligned": ("return A_i.T @ Gout_i", "return A_i.T @ Gout_i[::-1]"),
    "project_transposed": ("return P.T @ G", "return (G.T @ P).T[::-1]"),
    # clipping
    "clip_inverted": ("return C / norm if norm > C else 1.0", "return min(1.0, norm / C)"),
    "clip_always": ("return C / norm if norm > C else 1.0", "return C / norm if norm > 0 else 1.0"),
    "norm_first_layer_only": ("np.sqrt(sum(np.sum(R[i][l] ** 2) for l in range(L)))",
                              "np.sqrt(np.sum(R[i][0] ** 2))"),
    "norm_not_sqrt": ("np.sqrt(sum(np.sum(R[i][l] ** 2) for l in range(L)))",
                      "sum(np.sum(R[i][l] ** 2) for l in range(L))"),
    "aggregate_unclipped": ("S_l = sum(c[i] * R[i][l] for i in range(B))",
                            "S_l = sum(R[i][l] for i in range(B))"),
    # noise and average
    "noise_without_C": ("g = (S_l + h.sigma * h.C * xi) / div", "g = (S_l + h.sigma * xi) / div"),
    "no_batch_average": ("g = (S_l + h.sigma * h.C * xi) / div", "g = (S_l + h.sigma * h.C * xi)"),
    "noise_averaged_twice": ("g = (S_l + h.sigma * h.C * xi) / div",
                             "g = S_l / div + h.sigma * h.C * xi / div / div"),
    # Adam
    "adam_no_bias_correction_m": ("m_hat = m / (1.0 - beta1 ** t)", "m_hat = m"),
    "adam_no_bias_correction_v": ("v_hat = v / (1.0 - beta2 ** t)", "v_hat = v"),
    "adam_eps_inside_sqrt": ("m_hat / (np.sqrt(v_hat) + eps)", "m_hat / np.sqrt(v_hat + eps)"),
    "adam_v_not_squared": ("v = beta2 * v + (1.0 - beta2) * g * g", "v = beta2 * v + (1.0 - beta2) * g"),
    "adam_betas_swapped": ("m = beta1 * m + (1.0 - beta1) * g", "m = beta2 * m + (1.0 - beta2) * g"),
    "adam_t_zero_based": ("t = step_index + 1", "t = step_index + 2"),
    # back-projection
    "backproject_other_P": ("state.W[l] = state.W[l] - h.lr * (Ps[l] @ d)",
                            "state.W[l] = state.W[l] - h.lr * (proj(l, step_index + 1, "
                            "state.W[l].shape[0], h.r) @ d)"),
    "backproject_sign": ("state.W[l] = state.W[l] - h.lr * (Ps[l] @ d)",
                         "state.W[l] = state.W[l] + h.lr * (Ps[l] @ d)"),
    "backproject_no_lr": ("state.W[l] = state.W[l] - h.lr * (Ps[l] @ d)",
                          "state.W[l] = state.W[l] - (Ps[l] @ d)"),
    # projection-refresh period
    "refresh_ignored": ("return step // self.refresh", "return step"),
    "refresh_off_by_one": ("return step // self.refresh", "return (step + 1) // self.refresh"),
    # Hutchinson estimate
    "hutch_wrong_gram": ("O = G @ G.T", "O = G @ G.T + np.eye(G.shape[0])"),
    "hutch_first_column": ("for j in range(P.shape[1])))", "for j in range(1)))"),
    # ghost norm
    "ghost_wrong_gram_side": ("X = AP_i @ AP_i.T", "X = AP_i.T @ AP_i"),
    "ghost_half_gram": ("X = AP_i @ AP_i.T", "X = 0.5 * (AP_i @ AP_i.T)"),
    "ghost_trace_only": ("return float(np.sum(X * Y))", "return float(np.trace(X) * np.trace(Y))"),
    # token mask
    "mask_inverted": ("keep = (np.asarray(mask) != 0)[:, :, None]", "keep = (np.asarray(mask) == 0)[:, :, None]"),
    "mask_zeroes_nothing": ("return [np.where(keep, g, 0.0) for g in Gout]", "return [g for g in Gout]"),
    "token_mean_gradient": ("return A_i.T @ Gout_i", "return A_i.T @ Gout_i / A_i.shape[0]"),
    "hutch_transposed_sketch": ("return float(sum(P[:, j] @ O @ P[:, j] for j in range(P.shape[1])))",
                                "return float(sum(P[:, j] @ O.T @ O @ P[:, j] for j in range(P.shape[1])))"),
    # generator details
    "key_words_swapped": ("return philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))",
                          "return philox4x32_10(ctr, ((seed >> 32) & 0xFFFFFFFF, seed & 0xFFFFFFFF))"),
    "philox_hi_lo_swapped": ("hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32",
                             "lo0, hi0 = p0 >> np.uint64(32), p0 & _MASK32"),
    "weyl_before_first_round": ("        if rnd > 0:\n", "        if True:\n"),
    "bm_u2_offset": ("u2 = xb.astype(np.float64) * 2.0 ** -32",
                     "u2 = (xb.astype(np.float64) + 1.0) * 2.0 ** -32"),
    "bm_log2": ("rho = np.sqrt(-2.0 * np.log(u1))", "rho = np.sqrt(-2.0 * np.log2(u1))"),
    # the step
    "noise_not_averaged": ("g = (S_l + h.sigma * h.C * xi) / div", "g = S_l / div + h.sigma * h.C * xi"),
    "clip_on_sqnorm": ("c = np.array([clip_factor(n, h.C) for n in norms])",
                       "c = np.array([clip_factor(n * n, h.C) for n in norms])"),
    "noise_keyed_by_refresh": ("xi = noise_matrix(h.seed, l, step_index,",
                               "xi = noise_matrix(h.seed, l, h.projection_key(step_index),"),
    "noise_layer_zero": ("xi = noise_matrix(h.seed, l, step_index,", "xi = noise_matrix(h.seed, 0, step_index,"),
    "P_layer_zero": ("return lambda layer, step, d_in, r: projection_matrix(h.seed, layer,",
                     "return lambda layer, step, d_in, r: projection_matrix(h.seed, 0,"),
    "adam_no_sqrt": ("return m, v, m_hat / (np.sqrt(v_hat) + eps)", "return m, v, m_hat / (v_hat + eps)"),
    "hutch_divided_by_k": ("return float(sum(P[:, j] @ O @ P[:, j] for j in range(P.shape[1])))",
                           "return float(sum(P[:, j] @ O @ P[:, j] for j in range(P.shape[1]))) / P.shape[1]"),
    # the spot-check functions of the full-size tests
    "sample_norms_no_sqrt": (
        "            tot[j] += float(np.sum(project(P, per_sample_gradient(A[l][j], Gout[l][j])) ** 2))\n"
        "    return np.sqrt(tot)",
        "            tot[j] += float(np.sum(project(P, per_sample_gradient(A[l][j], Gout[l][j])) ** 2))\n"
        "    return tot"),
    "sample_norms_ignore_refresh": (
        "        P = projection_matrix(h.seed, l, h.projection_key(step_index), d_in[l], h.r)\n"
        "        for j in range(n):\n            tot[j] += float(",
        "        P = projection_matrix(h.seed, l, step_index, d_in[l], h.r)\n"
        "        for j in range(n):\n            tot[j] += float("),
    "hutch_samples_ignore_refresh": (
        "            tot[j] += hutchinson_sqnorm(A[l][j], Gout[l][j], P)",
        "            tot[j] += hutchinson_sqnorm(A[l][j], Gout[l][j], "
        "projection_matrix(h.seed, l, step_index, d_in[l], h.r))"),
    "hutch_samples_first_layer": (
        "            tot[j] += hutchinson_sqnorm(A[l][j], Gout[l][j], P)",
        "            tot[j] += hutchinson_sqnorm(A[0][j], Gout[0][j], P) if l == 0 else 0.0"),
}

# cheap pins first: a mutation stops at the first pin that fails
ORDER = sorted(pins.ALL_PINS, key=lambda p: {
    "pin_normal_statistics": 5, "pin_backprojection_unbiased": 6}.get(p.__name__, 0))


_COUNT = itertools.count()


def _mutant(old: str, new: str) -> types.ModuleType:
    src = open(SRC).read()
    assert src.count(old) == 1, f"fragment not found exactly once: {old!r}"
    name = f"grape_oracle_mutant_{next(_COUNT)}"
    mod = types.ModuleType(name)
    mod.__file__ = SRC
    sys.modules[name] = mod          # dataclasses look their module up here
    exec(compile(src.replace(old, new), SRC + "[mutant]", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name):
    mod = _mutant(*MUTATIONS[name])
    for pin in ORDER:
        try:
            pin(mod)
        except Exception:          # noqa: BLE001  any failure of a pin catches the mutation
            return
    pytest.fail(f"mutation {name!r} passed every pin")


def test_unmutated_copy_passes_every_pin():
    """The exec'd copy itself is faithful (guards the harness)."""
    mod = _mutant("PHILOX_ROUNDS = 10", "PHILOX_ROUNDS = 10")
    for pin in pins.ALL_PINS:
        pin(mod)
