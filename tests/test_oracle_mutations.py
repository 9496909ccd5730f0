"""Planted mistakes in the oracle (on the CPU) must each trip a pin.

Each mutant replaces one step of the oracle with a plausible slip -- a
dropped term, a wrong sign, a wrong weight slice, a transposed operand, a
missing normalisation -- and the test asserts that at least one of the pins
in test_oracle_pins.py fails under it.  This shows the pins can see such
mistakes anywhere in the oracle.
"""
import numpy as np
import pytest

import oracle
import oracle.mla_oracle as om
import test_oracle_pins as pins

DECODE_PINS = [
    lambda: pins.test_absorbed_equals_materialised_small_dims(0),
    pins.test_all_selected_equals_unmasked_dense,
    pins.test_softmax_rows_sum_to_one_and_nonnegative,
    pins.test_duplicates_padding_and_invalid_entries,
    pins.test_materialised_matches_with_duplicates,
    pins.test_empty_selection_gives_zero,
    pins.test_single_key_closed_form,
    pins.test_zero_query_gives_uniform_mean,
    pins.test_two_keys_closed_form,
    pins.test_brute_force_scalar_loops,
    pins.test_index_mask_brute_force,
]
ROPE_PINS = [
    pins.test_rope_position_zero_is_identity,
    pins.test_rope_unit_vector_closed_form,
    pins.test_rope_preserves_pair_norms_and_relative_positions,
    pins.test_rope_noninterleaved_is_permuted_interleaved,
    pins.test_cache_write_with_selection_weights,
]
NORM_PINS = [pins.test_rmsnorm_unit_rms, pins.test_cache_write_with_selection_weights]
OUT_PROJ_PINS = [
    pins.test_out_proj_one_hot_selects_a_weight_column,
    pins.test_out_proj_is_linear,
    pins.test_out_proj_mixes_heads_under_a_joint_permutation_only,
    pins.test_out_proj_brute_force,
]
QUERY_PINS = [
    pins.test_query_proj_routes_heads_and_splits_nope_before_rope,
    pins.test_query_proj_is_scale_invariant_through_the_norm,
    pins.test_query_proj_position_moves_only_the_rotary_part,
    pins.test_query_proj_brute_force,
]


def _fold_wrong_rows(q_nope, wkv_b):
    Dn = q_nope.shape[-1]
    return np.einsum("bhd,hdc->bhc", q_nope, wkv_b[:, -Dn:, :])


def _fold_wrong_head(q_nope, wkv_b):
    Dn = q_nope.shape[-1]
    return np.einsum("bhd,hdc->bhc", q_nope, np.roll(wkv_b, 1, axis=0)[:, :Dn, :])


def _scores_no_rope(qt, qpe, c, pe, scale):
    return (qt @ c.T) * scale


def _scores_rope_sign(qt, qpe, c, pe, scale):
    return (qt @ c.T - qpe @ pe.T) * scale


def _scores_no_scale(qt, qpe, c, pe, scale):
    return qt @ c.T + qpe @ pe.T


def _softmax_wrong_axis(s):
    e = np.exp(s - s.max(axis=0, keepdims=True))
    return e / e.sum(axis=0, keepdims=True)


def _softmax_unnormalised(s):
    return np.exp(s - s.max(axis=-1, keepdims=True))


def _mix_transposed(A, c):
    return (A / A.shape[1]) @ np.roll(c, 1, axis=0)


def _wuv_wrong_rows(o_t, wkv_b, Dv):
    return np.einsum("hc,hdc->hd", o_t, wkv_b[:, :Dv, :])


def _wuv_transposed_head(o_t, wkv_b, Dv):
    return np.einsum("hc,hdc->hd", o_t, np.roll(wkv_b, 1, axis=0)[:, -Dv:, :])


def _select_no_dedup(row, end_pos, T):
    keep, invalid = [], 0
    for v in np.asarray(row).tolist():
        if v == -1:
            continue
        if not (0 <= v < min(end_pos, T)):
            invalid += 1
            continue
        keep.append(int(v))
    return keep, invalid


def _select_off_by_one(row, end_pos, T):
    keep, invalid, seen = [], 0, set()
    for v in np.asarray(row).tolist():
        if v == -1:
            continue
        if not (0 <= v <= min(end_pos, T)) or v >= T:
            invalid += 1
            continue
        if v not in seen:
            seen.add(v)
            keep.append(int(v))
    return keep, invalid


def _rope_conjugate(x, R, interleaved=True):
    return _orig_rope(x, np.conj(R), interleaved)


def _rope_swapped_pairs(x, R, interleaved=True):
    x = np.asarray(x, dtype=np.float64)
    return _orig_rope(x, R, not interleaved)


def _rmsnorm_no_sqrt(x, w, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w)


def _rmsnorm_sum_not_mean(x, w, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w)


def _out_proj_dim_major(o, w_o):
    # flattens O value-dim-major instead of head-major
    o = np.asarray(o, dtype=np.float64)
    return np.swapaxes(o, 1, 2).reshape(o.shape[0], -1) @ np.asarray(w_o).T


def _out_proj_drop_last_head(o, w_o):
    o = np.array(o, dtype=np.float64)
    o[:, -1, :] = 0.0
    return o.reshape(o.shape[0], -1) @ np.asarray(w_o).T


def _out_proj_untransposed(o, w_o):
    # weight read [in, out] although it is stored [out, in]
    o = np.asarray(o, dtype=np.float64)
    w = np.asarray(w_o, dtype=np.float64)
    return o.reshape(o.shape[0], -1) @ w.reshape(w.shape[1], w.shape[0])


def _query_rope_first(x, wq_a, w, eps, wq_b, R_pos, n_heads, dn, interleaved=True):
    # rotary part taken from the front of each head's block
    qr = om.rmsnorm(np.asarray(x, dtype=np.float64) @ np.asarray(wq_a).T, w, eps)
    q = (qr @ np.asarray(wq_b).T).reshape(qr.shape[0], n_heads, -1)
    rr = q.shape[-1] - dn
    return q[..., rr:], om.rope(q[..., :rr], np.asarray(R_pos), interleaved)


def _query_norm_first(x, wq_a, w, eps, wq_b, R_pos, n_heads, dn, interleaved=True):
    # normalises the input instead of the down-projection
    xn = np.asarray(x, dtype=np.float64)
    xn = xn / np.sqrt(np.mean(xn * xn, axis=-1, keepdims=True) + eps)
    qr = (xn @ np.asarray(wq_a).T) * np.asarray(w)
    q = (qr @ np.asarray(wq_b).T).reshape(qr.shape[0], n_heads, -1)
    return q[..., :dn], om.rope(q[..., dn:], np.asarray(R_pos), interleaved)


def _query_feature_major(x, wq_a, w, eps, wq_b, R_pos, n_heads, dn, interleaved=True):
    # views the wq_b output feature-major instead of head-major
    qr = om.rmsnorm(np.asarray(x, dtype=np.float64) @ np.asarray(wq_a).T, w, eps)
    q = (qr @ np.asarray(wq_b).T).reshape(qr.shape[0], -1, n_heads).swapaxes(1, 2)
    return q[..., :dn], om.rope(q[..., dn:], np.asarray(R_pos), interleaved)


PREFILL_PINS = [
    pins.test_prefill_equals_absorbed_decode_per_token,
    pins.test_prefill_first_token_sees_only_itself,
    pins.test_prefill_ignores_future_and_unlisted_positions,
    pins.test_prefill_brute_force,
    pins.test_prefill_and_multi_query_degenerate_cases,
]
MULTI_QUERY_PINS = [pins.test_multi_query_matches_materialised_per_query,
                    pins.test_prefill_and_multi_query_degenerate_cases]


def _prefill_mask_no_causal(topk_b, S):
    # index mask only: listed positions after the token stay visible
    m = np.full((S, S), -np.inf)
    for s_ in range(S):
        for t in np.asarray(topk_b[s_]).tolist():
            if 0 <= t < S:
                m[s_, t] = 0.0
    return m


def _prefill_mask_strict(topk_b, S):
    # causal mask that also hides the token's own position
    m = _prefill_mask_no_causal(topk_b, S)
    return m + np.triu(np.full((S, S), -np.inf), 0)


def _prefill_mask_dense(topk_b, S):
    # causal mask only: the index selection is ignored
    return np.triu(np.full((S, S), -np.inf), 1)


_orig_expand = om.expand_keys_values


def _expand_values_from_key_rows(c, pe, wkv_b, Dn):
    # values taken from the first rows of each head (the key rows)
    k, v = _orig_expand(c, pe, wkv_b, Dn)
    kv = np.einsum("tc,hjc->thj", c, wkv_b)
    return k, kv[:, :, :v.shape[-1]]


def _expand_without_rotary_key(c, pe, wkv_b, Dn):
    # the shared rotary key left out of every head's key
    k, v = _orig_expand(c, pe, wkv_b, Dn)
    k = k.copy()
    k[..., Dn:] = 0.0
    return k, v


def _multi_query_modulo_rows(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale, qpr):
    # query row r read from cache row r % (cache rows) instead of r // qpr
    rows = np.arange(np.asarray(q_nope).shape[0]) % np.asarray(c_kv).shape[0]
    return om.decode_absorbed(q_nope, q_pe, wkv_b, np.asarray(c_kv)[rows], np.asarray(k_pe)[rows],
                              topk, end_pos, scale)


_orig_rope = om.rope

MUTANTS = [
    ("fold_wuk", _fold_wrong_rows, DECODE_PINS),
    ("fold_wuk", _fold_wrong_head, DECODE_PINS),
    ("scores", _scores_no_rope, DECODE_PINS),
    ("scores", _scores_rope_sign, DECODE_PINS),
    ("scores", _scores_no_scale, DECODE_PINS),
    ("softmax_rows", _softmax_wrong_axis, DECODE_PINS),
    ("softmax_rows", _softmax_unnormalised, DECODE_PINS),
    ("mix_latent", _mix_transposed, DECODE_PINS),
    ("apply_wuv", _wuv_wrong_rows, DECODE_PINS),
    ("apply_wuv", _wuv_transposed_head, DECODE_PINS),
    ("selected_positions", _select_no_dedup, DECODE_PINS),
    ("selected_positions", _select_off_by_one, DECODE_PINS),
    ("rope", _rope_conjugate, ROPE_PINS),
    ("rope", _rope_swapped_pairs, ROPE_PINS),
    ("rmsnorm", _rmsnorm_no_sqrt, NORM_PINS),
    ("rmsnorm", _rmsnorm_sum_not_mean, NORM_PINS),
    ("out_proj", _out_proj_dim_major, OUT_PROJ_PINS),
    ("out_proj", _out_proj_drop_last_head, OUT_PROJ_PINS),
    ("out_proj", _out_proj_untransposed, OUT_PROJ_PINS),
    ("query_proj", _query_rope_first, QUERY_PINS),
    ("query_proj", _query_norm_first, QUERY_PINS),
    ("query_proj", _query_feature_major, QUERY_PINS),
    ("prefill_mask", _prefill_mask_no_causal, PREFILL_PINS),
    ("prefill_mask", _prefill_mask_strict, PREFILL_PINS),
    ("prefill_mask", _prefill_mask_dense, PREFILL_PINS),
    ("expand_keys_values", _expand_values_from_key_rows, PREFILL_PINS),
    ("expand_keys_values", _expand_without_rotary_key, PREFILL_PINS),
    ("decode_multi_query", _multi_query_modulo_rows, MULTI_QUERY_PINS),
]


@pytest.mark.parametrize("name,mutant,checks", MUTANTS,
                         ids=[f"{n}:{m.__name__}" for n, m, _ in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, checks):
    monkeypatch.setattr(om, name, mutant)
    monkeypatch.setattr(oracle, name, mutant, raising=False)
    caught = 0
    for check in checks:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake in {name}"
