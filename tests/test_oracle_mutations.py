"""Planted mistakes in the oracle must fail at least one pin.

Each mutant replaces one oracle function (on the CPU, for the duration of
one test) with a plausible wrong variant: a sign, a dropped term, a
transposed operand, a wrong index or comparison.  The pins of
``test_oracle_pins`` are then re-run and at least one must fail.
"""
import numpy as np
import pytest

from oracle import mla_oracle as O
import tests.test_oracle_pins as P

PINS = [
    P.test_worked_absorption_example,
    P.test_worked_value_example,
    lambda: P.test_rope_matches_complex_rotation(4095),
    lambda: P.test_rope_relative_position_invariance(1000),
    P.test_relocation_offset_invariance,
    P.test_matches_torch_sdpa_with_expanded_keys,
    P.test_softmax_rows_sum_to_one_and_lse_closed_form,
    P.test_zero_query_gives_mean_of_visible_rows,
    P.test_merge_of_any_split_equals_unsplit,
    P.test_merge_with_empty_is_identity,
    P.test_out_proj_fold_identity,
    P.test_written_cache_serves_textbook_rope_attention,
    P.test_cache_rows_at_position_zero_store_the_raw_key,
    P.test_append_rows_lands_in_its_slots_only,
    lambda: P.test_qknorm_absorbed_equals_explicit(dict(s_q=2, lengths=(13, 70))),
    P.test_qknorm_matches_torch_rms_norm_and_sdpa,
    P.test_qknorm_is_scale_invariant_in_query_and_latent,
    P.test_qknorm_with_unit_rms_inputs_is_plain_attention,
    P.test_packed_code_bytes_worked_by_hand,
    lambda: P.test_pack_unpack_round_trip_every_byte(4),
    lambda: P.test_quantization_error_bound_and_saturation(4),
    P.test_quantization_ties_go_to_the_even_code,
    lambda: P.test_grid_exact_cache_passes_through_unchanged(4),
]


def _rope_sign(x, pos, base):
    x = np.asarray(x, np.float64)
    ang = np.asarray(pos, np.float64)[..., None] * O.rope_inv_freq(x.shape[-1], base)
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (x.shape[-1],)))
    out[..., 0::2] = x[..., 0::2] * np.cos(ang) + x[..., 1::2] * np.sin(ang)
    out[..., 1::2] = -x[..., 0::2] * np.sin(ang) + x[..., 1::2] * np.cos(ang)
    return out


def _rope_half(x, pos, base):
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, np.float64)[..., None] * O.rope_inv_freq(d, base)
    a, b = x[..., :d // 2], x[..., d // 2:]
    return np.concatenate([a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)], -1)


def _freq_off_by_one(d_r, base):
    i = np.arange(1, d_r // 2 + 1, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d_r)


def _direct_no_rope(q_nope, q_rope, q_pos, u_k, u_v, c, k_rope, key_pos, key_shift, scale, base):
    return _ORIG["attend_direct"](q_nope, np.zeros_like(q_rope), q_pos, u_k, u_v, c,
                                  k_rope, key_pos, key_shift, scale, base)


def _direct_shift_sign(q_nope, q_rope, q_pos, u_k, u_v, c, k_rope, key_pos, key_shift, scale, base):
    return _ORIG["attend_direct"](q_nope, q_rope, q_pos, u_k, u_v, c, k_rope, key_pos,
                                  -np.asarray(key_shift), scale, base)


def _direct_strict_mask(q_nope, q_rope, q_pos, u_k, u_v, c, k_rope, key_pos, key_shift, scale, base):
    return _ORIG["attend_direct"](q_nope, q_rope, q_pos, u_k, u_v, c, k_rope,
                                  np.asarray(key_pos) + 1, key_shift, scale, base)


def _direct_no_scale(q_nope, q_rope, q_pos, u_k, u_v, c, k_rope, key_pos, key_shift, scale, base):
    return _ORIG["attend_direct"](q_nope, q_rope, q_pos, u_k, u_v, c, k_rope, key_pos,
                                  key_shift, 1.0, base)


def _content_keys_T(u_k, c):
    return np.asarray(c, np.float64) @ np.asarray(u_k, np.float64).T[::-1]


def _absorb_T(u_k, q):
    return np.asarray(q, np.float64) @ np.asarray(u_k, np.float64)[::-1]


def _values_T(u_v, c):
    return np.asarray(c, np.float64)[:, ::-1] @ np.asarray(u_v, np.float64).T


def _merge_swapped(o_a, lse_a, o_b, lse_b):
    o, l = _ORIG["merge_lse"](o_a, lse_a, o_b, lse_b)
    la, lb = np.asarray(lse_a), np.asarray(lse_b)
    wa = np.exp(la - l)
    wb = np.exp(lb - l)
    return wb[..., None] * np.asarray(o_a) + wa[..., None] * np.asarray(o_b), l


def _softmax_no_max(s):
    a, lse = _ORIG["softmax_lse"](s)
    m = np.max(np.where(np.isfinite(s), s, -1e300), axis=-1)
    return a, lse - np.where(np.isfinite(m), m, 0.0)


def _out_proj_T(o_lat, w_uv, w_o):
    v = np.einsum("hdc,qhc->qdh", np.asarray(w_uv, np.float64), np.asarray(o_lat, np.float64))
    return v, v.reshape(v.shape[0], -1) @ np.asarray(w_o, np.float64).T


def _writer_position_plus_one(c, k_rope_raw, cache_pos, base):
    return _ORIG["cache_rows"](c, k_rope_raw, np.asarray(cache_pos) + 1, base)


def _writer_unrotated(c, k_rope_raw, cache_pos, base):
    return np.concatenate([np.asarray(c, np.float64), np.asarray(k_rope_raw, np.float64)], -1)


def _writer_request_rotation_sign(c, k_rope_raw, cache_pos, base):
    return _ORIG["cache_rows"](c, k_rope_raw, -np.asarray(cache_pos), base)


def _append_slot_shift(pool, block_table_b, row0, rows, page=64):
    out = np.array(pool, dtype=np.float64, copy=True)
    for i, row in enumerate(np.asarray(rows, np.float64)):
        r = int(row0) + i
        out[int(block_table_b[r // page]), (r + 1) % page] = row
    return out


def _append_page_of_next_row(pool, block_table_b, row0, rows, page=64):
    out = np.array(pool, dtype=np.float64, copy=True)
    for i, row in enumerate(np.asarray(rows, np.float64)):
        r = int(row0) + i
        out[int(block_table_b[(r + 1) // page]), r % page] = row
    return out


def _qk_absorbed_rope_scaled(q_nope, q_rope, q_pos, w_uk, c, k_rope, key_shift, g_q, g_k,
                             scale, base, eps=O.QK_NORM_EPS):
    # the per-token key statistic applied to the whole score, rotary term too
    s = _ORIG["qknorm_scores_absorbed"](q_nope, q_rope, q_pos, w_uk, c, k_rope, key_shift,
                                        g_q, g_k, scale, base, eps)
    inv = O.key_inv_rms(c, w_uk, eps)
    content = _ORIG["qknorm_scores_absorbed"](q_nope, np.zeros_like(q_rope), q_pos, w_uk, c,
                                              k_rope, key_shift, g_q, g_k, scale, base, eps)
    return content + (s - content) * inv[None, :]


def _qk_absorbed_key_weight_dropped(q_nope, q_rope, q_pos, w_uk, c, k_rope, key_shift, g_q,
                                    g_k, scale, base, eps=O.QK_NORM_EPS):
    return _ORIG["qknorm_scores_absorbed"](q_nope, q_rope, q_pos, w_uk, c, k_rope, key_shift,
                                           g_q, np.ones_like(np.asarray(g_k, np.float64)),
                                           scale, base, eps)


def _key_inv_rms_first_head(c, w_uk, eps=O.QK_NORM_EPS):
    return _ORIG["key_inv_rms"](c, np.asarray(w_uk)[:1], eps)


def _rms_norm_eps_outside(x, weight, eps=O.QK_NORM_EPS):
    x = np.asarray(x, np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * np.asarray(weight)


def _qk_direct_no_query_norm(q_nope, q_rope, q_pos, w_uk, c, k_rope, key_shift, g_q, g_k,
                             scale, base, eps=O.QK_NORM_EPS):
    # the query weight applied but the query never divided by its RMS
    H, d_n = np.asarray(q_nope).shape
    q_w = np.asarray(q_nope, np.float64) * np.asarray(g_q, np.float64).reshape(H, d_n)
    k = np.einsum("hnc,tc->thn", np.asarray(w_uk, np.float64), np.asarray(c, np.float64))
    k_hat = O.rms_norm(k.reshape(k.shape[0], -1), g_k, eps).reshape(k.shape)
    q_r = O.rope_rotate(q_rope, q_pos, base)
    k_r = O.rope_rotate(k_rope, key_shift, base)
    return scale * (np.einsum("hn,thn->ht", q_w, k_hat) + q_r @ k_r.T)


def _quantize_truncating(x, scale, bits):
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    q = np.trunc(np.asarray(x, np.float64) / np.asarray(scale, np.float64))
    return np.clip(q, lo, hi).astype(np.int64)


def _quantize_symmetric_range(x, scale, bits):
    hi = (1 << (bits - 1)) - 1
    q = np.round(np.asarray(x, np.float64) / np.asarray(scale, np.float64))
    return np.clip(q, -hi, hi).astype(np.int64)


def _pack_high_first(codes, bits):
    codes = np.asarray(codes, np.int64)
    per = 8 // bits
    fields = (codes & ((1 << bits) - 1)).reshape(codes.shape[:-1] + (-1, per))
    out = np.zeros(fields.shape[:-1], np.int64)
    for k in range(per):
        out |= fields[..., k] << (bits * (per - 1 - k))
    return out.astype(np.uint8)


def _unpack_unsigned(packed, bits):
    b = np.asarray(packed, np.int64)
    per = 8 // bits
    fields = np.stack([(b >> (bits * k)) & ((1 << bits) - 1) for k in range(per)], axis=-1)
    return fields.reshape(b.shape[:-1] + (b.shape[-1] * per,))


def _dequantize_divides(codes, scale):
    return np.asarray(codes, np.float64) / np.asarray(scale, np.float64)


_ORIG = {k: getattr(O, k) for k in ("attend_direct", "merge_lse", "softmax_lse", "cache_rows",
                                    "qknorm_scores_absorbed", "qknorm_scores_direct",
                                    "key_inv_rms")}

MUTANTS = {
    "rope_sign": ("rope_rotate", _rope_sign),
    "rope_rotate_half": ("rope_rotate", _rope_half),
    "rope_freq_index": ("rope_inv_freq", _freq_off_by_one),
    "drop_rotary_term": ("attend_direct", _direct_no_rope),
    "relocation_sign": ("attend_direct", _direct_shift_sign),
    "strict_mask": ("attend_direct", _direct_strict_mask),
    "scale_dropped": ("attend_direct", _direct_no_scale),
    "content_key_rows": ("content_keys", _content_keys_T),
    "absorb_rows": ("absorb_query", _absorb_T),
    "value_cols": ("values", _values_T),
    "merge_weights_swapped": ("merge_lse", _merge_swapped),
    "lse_without_max": ("softmax_lse", _softmax_no_max),
    "out_proj_transposed": ("out_proj", _out_proj_T),
    "writer_position_plus_one": ("cache_rows", _writer_position_plus_one),
    "writer_unrotated": ("cache_rows", _writer_unrotated),
    "writer_rotation_sign": ("cache_rows", _writer_request_rotation_sign),
    "append_slot_shift": ("append_rows", _append_slot_shift),
    "append_page_of_next_row": ("append_rows", _append_page_of_next_row),
    "qknorm_rope_scaled": ("qknorm_scores_absorbed", _qk_absorbed_rope_scaled),
    "qknorm_key_weight_dropped": ("qknorm_scores_absorbed", _qk_absorbed_key_weight_dropped),
    "qknorm_stat_one_head": ("key_inv_rms", _key_inv_rms_first_head),
    "qknorm_eps_outside_sqrt": ("rms_norm", _rms_norm_eps_outside),
    "qknorm_query_not_normalised": ("qknorm_scores_direct", _qk_direct_no_query_norm),
    "quantize_truncates": ("quantize_symmetric", _quantize_truncating),
    "quantize_symmetric_range": ("quantize_symmetric", _quantize_symmetric_range),
    "pack_first_code_high": ("pack_codes", _pack_high_first),
    "unpack_without_sign": ("unpack_codes", _unpack_unsigned),
    "dequantize_divides": ("dequantize", _dequantize_divides),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:            # an assertion or a shape error both count
            failed.append(pin)
    assert failed, f"mutant {name} passed every pin"
