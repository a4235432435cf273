"""Planted mistakes in copies of the oracle must each fail at least one pin.

Every mutant below is a plausible slip (a dropped term, a flipped sign, a wrong
or transposed index, a missing factor).  Each is applied to a copy of
oracle/lla_oracle.c in a temporary directory, compiled with gcc and loaded in
place of the real oracle while the pins of test_oracle_pins.py run.  If a
mutant survives every pin, the pins are too weak and this test fails.  All
mutants keep every array access in bounds.  CPU only.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "lla_oracle.c")

MUTANTS = {
    "encode_sign_of_mean": ("(x[i * W + k] - mu[k])", "(x[i * W + k] + mu[k])"),
    "encode_transposed_W_down": ("W_down[(int64_t)k * r + j]", "W_down[(int64_t)j * W + k]"),
    "reconstruct_drops_mean": ("double acc = mu_t[k];", "double acc = 0.0;"),
    "reconstruct_transposed_W_up": ("W_up_t[(int64_t)j * d + k]", "W_up_t[(int64_t)k * r + j]"),
    "softmax_no_max_subtraction": ("p[i] = exp(l[i] - m);", "p[i] = exp(l[i]);"),
    "softmax_lse_drops_max": ("*lse = m + log(Z);", "*lse = log(Z);"),
    "softmax_not_normalised": ("p[i] /= Z;", "p[i] /= 1.0;"),
    "softmax_min_instead_of_max": ("if (l[i] > m)", "if (l[i] < m)"),
    "reconstruct_attn_reversed_dot": ("dot += q[k] * k_hat[k];", "dot += q[k] * k_hat[d - 1 - k];"),
    "absorb_drops_scale": ("q_tilde[j] = scale * acc;", "q_tilde[j] = acc;"),
    "absorb_mean_term_sign": ("l[i] = dot + q_mu;", "l[i] = dot - q_mu;"),
    "absorb_drops_value_mean": ("double acc = mu_V_t[k];", "double acc = 0.0;"),
    "absorb_transposed_W_up_K": ("acc += q[k] * W_up_K_t[(int64_t)j * d + k];",
                                 "acc += q[k] * W_up_K_t[(int64_t)k * r_k + j];"),
    "absorb_reversed_value_latent": ("o_lat[j] += p[i] * c_V[i * r_v + j];",
                                     "o_lat[j] += p[i] * c_V[i * r_v + (r_v - 1 - j)];"),
    "absorb_wrong_key_latent_row": ("dot += q_tilde[j] * c_K[i * r_k + j];",
                                    "dot += q_tilde[j] * c_K[(n - 1 - i) * r_k + j];"),
    "hybrid_latent_key_reversed": ("dotc += q[k] * k_hat[k];", "dotc += q[k] * k_hat[d - 1 - k];"),
    "hybrid_window_drops_scale": ("l[n + m] = scale * dotw;", "l[n + m] = dotw;"),
    "hybrid_window_values_are_keys": ("o[k] += p[n + m] * v_win[m * d + k];",
                                      "o[k] += p[n + m] * k_win[m * d + k];"),
    "hybrid_window_key_reversed": ("dotw += q[k] * k_win[m * d + k];",
                                   "dotw += q[k] * k_win[m * d + (d - 1 - k)];"),
    "rope_not_a_rotation": ("x[ib] = xa * sn + xb * cs;", "x[ib] = -xa * sn + xb * cs;"),
    "rope_frequency_exponent": ("pow(base, -2.0 * i / d)", "pow(base, -1.0 * i / d)"),
    "rope_keys_ignore_offset": ("k_pos0 + (double)i", "(double)i"),
    "rope_query_not_rotated": ("rope_rotate(d, style, base, q_pos, q_rot);", ""),
    "rope_half_pairs_adjacent": ("style == 0 ? i + d / 2 : 2 * i + 1", "style == 0 ? i + 1 : 2 * i + 1"),
    "residual_mean_of_loop_zero": ("mu + (int64_t)t * Dp, x_hat", "mu, x_hat"),
    "residual_first_loop_block_only": ("W_up + (int64_t)t * r * Dp", "W_up"),
    "residual_norm_of_rebuilt": ("n2 += xi[t * Dp + k] * xi[t * Dp + k];", "n2 += x_hat[k] * x_hat[k];"),
    "residual_squared": ("err[i] = sqrt(e2);", "err[i] = e2;"),
    "residual_encodes_with_up_projection": ("oracle_encode(1, W, r, xi, mu, W_down, c);",
                                            "oracle_encode(1, W, r, xi, mu, W_up, c);"),
    "residual_up_block_stride": ("W_up + (int64_t)t * r * Dp", "W_up + (int64_t)t * Dp"),
    "decoupled_drops_rope_term": ("l[i] = scale * (dn + dr);", "l[i] = scale * dn;"),
    "decoupled_query_not_rotated": ("rope_rotate(d_r, style, base, q_pos, qr);", ""),
    "decoupled_rope_term_unscaled": ("l[i] = scale * (dn + dr);", "l[i] = scale * dn + dr;"),
    "decoupled_wrong_subkey_row": ("dr += qr[k] * k_rope[i * d_r + k];", "dr += qr[k] * k_rope[k];"),
    "bytes_drop_factor_two": ("2ull * (uint64_t)T * (uint64_t)H", "(uint64_t)T * (uint64_t)H"),
    "bytes_fold_swapped": ("fold2d ? 1u : (uint64_t)H", "fold2d ? (uint64_t)H : 1u"),
    "bytes_ratio_not_reduced": ("uint64_t g = gcd_u64(per_token_uncompressed, per_token_latent);",
                                "uint64_t g = 1;"),
}


def _pins():
    pins = [
        (P.test_rank_table_golden, {}),
        (P.test_headline_ratios_golden, {}),
        (P.test_rho_closed_forms, {}),
        (P.test_capacity_bytes_exact, {}),
        (P.test_cache_bytes_linear_and_divided_by_rho, {}),
        (P.test_full_rank_roundtrip_is_exact, {}),
        (P.test_encode_of_mean_is_zero_and_affine, {}),
        (P.test_reconstruct_orientation_one_hot, {}),
        (P.test_eckart_young_calibration_residual, {"r": 4}),
        (P.test_absorb_equals_reconstruct_low_rank, {}),
        (P.test_decode_layer_matches_masked_dense_attention, {"fold2d": True}),
        (P.test_hybrid_full_rank_equals_attention_over_all_tokens, {"n": 20, "w": 5}),
        (P.test_hybrid_window_order_is_irrelevant_and_empty_is_neutral, {}),
        (P.test_decode_layer_hybrid_matches_dense_attention_over_both_parts, {"fold2d": False}),
        (P.test_rope_matches_roformer_complex_form, {"style": 0, "q_pos": 9, "k_pos0": 0}),
        (P.test_rope_matches_roformer_complex_form, {"style": 1, "q_pos": 3000, "k_pos0": 17}),
        (P.test_rope_depends_on_relative_position_only, {}),
        (P.test_rope_pairings_are_one_permutation_apart, {}),
        (P.test_decode_layer_rope_matches_dense_rotated_attention, {"style": 0}),
        (P.test_decoupled_identity_codec_is_attention_over_concatenated_keys, {"style": 1}),
        (P.test_decoupled_rope_part_depends_on_relative_position, {}),
        (P.test_decoupled_without_rope_part_is_the_plain_read, {}),
        (P.test_residual_full_rank_codec_is_zero_and_norm_is_euclidean, {}),
        (P.test_residual_energy_on_calibration_set_is_the_svd_tail, {"r": 5}),
        (P.test_residual_of_in_span_and_orthogonal_offsets, {}),
        (P.test_residual_is_homogeneous_in_the_centred_vector, {}),
        (P.test_residual_with_differently_scaled_down_and_up_projections, {}),
    ]
    for v in P.VARIANTS:
        pins += [
            (P.test_full_rank_codec_equals_uncompressed_attention, {"variant": v, "scale": 0.125}),
            (P.test_softmax_weights_sum_to_one, {"variant": v}),
            (P.test_shift_of_key_mean_is_invisible, {"variant": v}),
            (P.test_single_token_returns_its_value, {"variant": v}),
            (P.test_identity_codec_is_textbook_attention, {"variant": v}),
            (P.test_large_logits_select_the_best_token, {"variant": v}),
            (P.test_fold2d_full_rank_reproduces_each_head, {"variant": v}),
        ]
    return pins


def test_unmutated_oracle_passes_every_pin():
    for fn, kw in _pins():
        fn(**kw)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(old, new))
    path_so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           str(path_c), "-o", str(path_so), "-lm"])
    saved = oracle._load()
    oracle._lib = oracle.configure(ctypes.CDLL(str(path_so)))
    failed = []
    try:
        for fn, kw in _pins():
            try:
                fn(**kw)
            except (AssertionError, ValueError, FloatingPointError):
                failed.append(fn.__name__)
    finally:
        oracle._lib = saved
    assert failed, f"mutant {name} survived every pin"


# Mutants of the numpy-level oracle functions (the codec fit, and the per-sequence, per-loop
# and per-head slicing of a decode layer): the function's source is edited, compiled in the
# oracle module's namespace and swapped in while that function's pins run.
PY_MUTANTS = {
    "fit_not_centred": ("codec_fit", "np.linalg.svd(x - mu[None, :], full_matrices=False)",
                        "np.linalg.svd(x, full_matrices=False)"),
    "fit_left_vectors": ("codec_fit", "W_down = Vt[:r].T.copy()", "W_down = _[:, :r].copy()"),
    "fit_no_sign_convention": ("codec_fit", "W_down *= sign[None, :]", "pass"),
    "fit_up_layout": ("codec_fit", "W_up = W_down.reshape(T, W // T, r).transpose(0, 2, 1).copy()",
                      "W_up = W_down.reshape(r, T, W // T).transpose(1, 0, 2).copy()"),
    "layer_ignores_first_loop": ("decode_layer", "wk, mk, wv, mv = slices(h, t0 + tq)",
                                 "wk, mk, wv, mv = slices(h, tq)"),
    "layer_ignores_seq_start": ("decode_layer", "cK = c_K[hp, s0:s0 + n]", "cK = c_K[hp, :n]"),
    "layer_values_ignore_seq_start": ("decode_layer", "cV = c_V[hp, s0:s0 + n]", "cV = c_V[hp, :n]"),
    "layer_always_plane_zero": ("decode_layer", "hp = 0 if fold2d else h", "hp = 0"),
    "layer_fold2d_column_slice": ("decode_layer", "cols = slice(h * d, (h + 1) * d)",
                                  "cols = slice(h, h + d)"),
    "layer_per_head_index_swapped": ("decode_layer", "return W_up_K[h][t], mu_K[h][t]",
                                     "return W_up_K[t % len(W_up_K)][h % len(W_up_K[0])], mu_K[h][t]"),
    "layer_window_loop_index": ("decode_layer", "win_k[b, h, t0 + tq, :nw]", "win_k[b, h, tq, :nw]"),
    "layer_window_values_are_keys": ("decode_layer", "win_v[b, h, t0 + tq, :nw]",
                                     "win_k[b, h, t0 + tq, :nw]"),
    "layer_subkeys_ignore_seq_start": ("decode_layer", "k_rope[hp, s0:s0 + n]", "k_rope[hp, :n]"),
    "layer_decoupled_position_of_sequence_zero": ("decode_layer", "float(q_pos[b]))\n            elif rope",
                                                  "float(q_pos[0]))\n            elif rope"),
    "layer_rope_position_of_sequence_zero": ("decode_layer", "float(q_pos[b]))\n            elif window",
                                             "float(q_pos[0]))\n            elif window"),
}

PY_PINS = {
    "codec_fit": [(P.test_codec_fit_recovers_planted_orthogonal_directions, {}),
                  (P.test_codec_fit_energy_and_orthonormality, {}),
                  (P.test_codec_fit_shift_moves_only_the_mean, {})],
    "decode_layer": [(P.test_decode_layer_matches_masked_dense_attention, {"fold2d": False}),
                     (P.test_decode_layer_matches_masked_dense_attention, {"fold2d": True}),
                     (P.test_decode_layer_hybrid_matches_dense_attention_over_both_parts, {"fold2d": False}),
                     (P.test_decode_layer_rope_matches_dense_rotated_attention, {"style": 1}),
                     (P.test_decode_layer_rope_with_folded_heads, {}),
                     (P.test_decode_layer_decoupled_matches_dense_attention, {}),
                     (P.test_fold2d_full_rank_reproduces_each_head, {"variant": "absorb"})],
}


def test_unmutated_python_oracle_passes_its_pins():
    for pins in PY_PINS.values():
        for fn, kw in pins:
            fn(**kw)


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_python_mutant_is_caught(name):
    import inspect
    import textwrap
    target, old, new = PY_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(getattr(oracle, target)))
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    saved = getattr(oracle, target)
    setattr(oracle, target, ns[target])
    failed = []
    try:
        for fn, kw in PY_PINS[target]:
            try:
                fn(**kw)
            except (AssertionError, ValueError, IndexError, FloatingPointError):
                failed.append(fn.__name__)
    finally:
        setattr(oracle, target, saved)
    assert failed, f"mutant {name} survived every pin"
