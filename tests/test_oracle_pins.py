"""Pins of the CPU oracle against what the pages and the mathematics fix.

No test here re-types the oracle's own formula: each compares it with an
independent route (the materialised per-head key/value path, dense masked
attention, scalar brute force, closed forms of special cases, invariants)
or with numbers printed on the pages.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle as orc

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(rng, B=2, H=4, Dn=8, Dv=6, C=16, Rr=4, T=40, k=17, scale=0.3):
    q_nope = rng.standard_normal((B, H, Dn))
    q_pe = rng.standard_normal((B, H, Rr))
    wkv_b = rng.standard_normal((H, Dn + Dv, C)) / math.sqrt(C)
    c_kv = rng.standard_normal((B, T, C))
    k_pe = rng.standard_normal((B, T, Rr))
    end_pos = np.array([T - 3 * b for b in range(B)])
    k = min(k, int(end_pos.min()))
    topk = np.stack([rng.permutation(int(end_pos[b]))[:k] for b in range(B)])
    return q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ---------------------------------------------------------------------------
# absorbed == materialised ("Key heads": folding W_UK into the queries gives
# the same scores; "Mix and project": O_i = O~_i W_UV,i)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_absorbed_equals_materialised_small_dims(seed):
    rng = np.random.default_rng(seed)
    p = _rand_problem(rng)
    a = orc.decode_absorbed(*p)
    m = orc.decode_materialised(*p)
    assert _rel(a, m) < 1e-12


def test_absorbed_equals_materialised_model_dims():
    wl = mi.make_small(B=2, T=70, k=33, seed=3, end_pos=[70, 51])
    args = (mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
            mi.f64(wl.cache[..., :mi.C]), mi.f64(wl.cache[..., mi.C:]),
            wl.topk.numpy(), wl.end_pos.numpy(), wl.scale)
    a = orc.decode_absorbed(*args)
    m = orc.decode_materialised(*args)
    assert a.shape == (2, 128, 128)
    assert _rel(a, m) < 1e-12


def test_all_selected_equals_unmasked_dense():
    """Selecting every position reproduces dense attention (no mask at all),
    computed here from per-head keys/values built from the latent."""
    rng = np.random.default_rng(7)
    q_nope, q_pe, wkv_b, c_kv, k_pe, _, _, scale = _rand_problem(rng, B=1, T=12, k=12)
    T = 12
    topk = rng.permutation(T)[None, :]
    end_pos = np.array([T])
    a = orc.decode_absorbed(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale)
    Dn = q_nope.shape[-1]
    out = np.zeros_like(a)
    for h in range(q_nope.shape[1]):
        K = np.concatenate([c_kv[0] @ wkv_b[h, :Dn].T, k_pe[0]], 1)     # [T, Dn+Rr]
        V = c_kv[0] @ wkv_b[h, Dn:].T                                   # [T, Dv]
        q = np.concatenate([q_nope[0, h], q_pe[0, h]])
        s = K @ q * scale
        w = np.exp(s - s.max())
        out[0, h] = (w / w.sum()) @ V
    assert _rel(a, out) < 1e-12


# ---------------------------------------------------------------------------
# softmax / selection invariants
# ---------------------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_nonnegative():
    rng = np.random.default_rng(11)
    p = _rand_problem(rng, k=25)
    _, ws = orc.decode_absorbed(*p, return_weights=True)
    for A, keep in ws:
        assert A.shape[1] == len(keep) == 25
        assert np.all(A >= 0)
        assert np.max(np.abs(A.sum(1) - 1.0)) < 1e-12


def test_permuting_the_selection_changes_nothing():
    rng = np.random.default_rng(12)
    p = list(_rand_problem(rng))
    a = orc.decode_absorbed(*p)
    p[5] = np.stack([row[rng.permutation(len(row))] for row in p[5]])
    b = orc.decode_absorbed(*p)
    assert _rel(b, a) < 1e-13


def test_duplicates_padding_and_invalid_entries():
    """Listed twice counts once (scatter of 0 is idempotent); -1 is padding;
    other out-of-range entries are ignored and counted."""
    rng = np.random.default_rng(13)
    p = list(_rand_problem(rng, B=2, T=30, k=10))
    base = orc.decode_absorbed(*p)
    end_pos = p[6]
    extra = np.array([[p[5][0, 0], -1, -1, int(end_pos[0]), -5],
                      [p[5][1, 3], p[5][1, 3], -1, 10_000, int(end_pos[1]) + 2]])
    p2 = list(p)
    p2[5] = np.concatenate([p[5], extra], 1)
    got = orc.decode_absorbed(*p2)
    assert _rel(got, base) < 1e-13
    mask, bad = orc.index_mask(p2[5], end_pos, 30)
    assert bad == 2 + 2
    mask0, bad0 = orc.index_mask(p[5], end_pos, 30)
    assert bad0 == 0 and np.array_equal(mask, mask0)


def test_materialised_matches_with_duplicates():
    rng = np.random.default_rng(14)
    p = list(_rand_problem(rng, B=1, T=20, k=6))
    p[5] = np.concatenate([p[5], p[5][:, :3], -np.ones((1, 2), int)], 1)
    assert _rel(orc.decode_absorbed(*p), orc.decode_materialised(*p)) < 1e-12


def test_empty_selection_gives_zero():
    rng = np.random.default_rng(15)
    p = list(_rand_problem(rng, B=2, T=20, k=4))
    p[5] = p[5].copy()
    p[5][1] = -1
    out = orc.decode_absorbed(*p)
    assert np.all(out[1] == 0)
    assert np.any(out[0] != 0)


def test_index_mask_brute_force():
    rng = np.random.default_rng(16)
    T = 50
    topk = rng.integers(-3, 60, size=(4, 30))
    end_pos = np.array([50, 10, 33, 1])
    mask, bad = orc.index_mask(topk, end_pos, T)
    exp_bad = 0
    for b in range(4):
        for t in range(T):
            listed = any(int(v) == t for v in topk[b])
            assert mask[b, t] == (1 if listed and t < end_pos[b] else 0)
        for v in topk[b]:
            if v != -1 and not (0 <= v < end_pos[b]):
                exp_bad += 1
    assert bad == exp_bad


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_single_key_closed_form():
    """One selected position: the softmax weight is 1, so O_h = W_UV,h c_t."""
    rng = np.random.default_rng(21)
    q_nope, q_pe, wkv_b, c_kv, k_pe, _, _, scale = _rand_problem(rng, B=2, T=9)
    topk = np.array([[4], [8]])
    end_pos = np.array([9, 9])
    out = orc.decode_absorbed(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale)
    Dn = q_nope.shape[-1]
    for b, t in ((0, 4), (1, 8)):
        for h in range(q_nope.shape[1]):
            assert np.allclose(out[b, h], wkv_b[h, Dn:] @ c_kv[b, t], rtol=0, atol=1e-13)


def test_zero_query_gives_uniform_mean():
    """q = 0: all scores are 0, weights are 1/n, O_h = W_UV,h mean(c_sel)."""
    rng = np.random.default_rng(22)
    q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale = _rand_problem(rng)
    q_nope[:] = 0
    q_pe[:] = 0
    out = orc.decode_absorbed(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale)
    Dn = q_nope.shape[-1]
    for b in range(out.shape[0]):
        mean = c_kv[b, topk[b]].mean(0)
        for h in range(out.shape[1]):
            assert np.allclose(out[b, h], wkv_b[h, Dn:] @ mean, atol=1e-13)


def test_shared_rotary_key_shift_invariance():
    """If every selected position has the same rotary key, the rotary term
    adds the same constant to each score of a head and cancels in the
    softmax: the result does not depend on q_pe."""
    rng = np.random.default_rng(23)
    q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale = _rand_problem(rng)
    k_pe[:] = rng.standard_normal(k_pe.shape[-1])
    a = orc.decode_absorbed(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale)
    b = orc.decode_absorbed(q_nope, 5 * rng.standard_normal(q_pe.shape), wkv_b, c_kv,
                            k_pe, topk, end_pos, scale)
    assert _rel(a, b) < 1e-12


def test_two_keys_closed_form():
    """Two positions: weight of the first is the logistic of the score gap."""
    rng = np.random.default_rng(24)
    q_nope, q_pe, wkv_b, c_kv, k_pe, _, _, scale = _rand_problem(rng, B=1, T=5)
    Dn = q_nope.shape[-1]
    topk = np.array([[1, 3]])
    out = orc.decode_absorbed(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, np.array([5]), scale)
    for h in range(q_nope.shape[1]):
        K1 = np.concatenate([wkv_b[h, :Dn] @ c_kv[0, 1], k_pe[0, 1]])
        K3 = np.concatenate([wkv_b[h, :Dn] @ c_kv[0, 3], k_pe[0, 3]])
        q = np.concatenate([q_nope[0, h], q_pe[0, h]])
        w1 = 1.0 / (1.0 + math.exp(-(q @ K1 - q @ K3) * scale))
        expect = wkv_b[h, Dn:] @ (w1 * c_kv[0, 1] + (1 - w1) * c_kv[0, 3])
        assert np.allclose(out[0, h], expect, atol=1e-13)


def test_brute_force_scalar_loops():
    """Hand-sized problem, every sum written as a scalar loop over the
    materialised definitions (K_i = [c W_UK,i^T ; k^R], V_i = c W_UV,i^T)."""
    rng = np.random.default_rng(25)
    H, Dn, Dv, C, Rr, T = 2, 2, 3, 3, 2, 4
    q_nope = rng.standard_normal((1, H, Dn))
    q_pe = rng.standard_normal((1, H, Rr))
    wkv_b = rng.standard_normal((H, Dn + Dv, C))
    c_kv = rng.standard_normal((1, T, C))
    k_pe = rng.standard_normal((1, T, Rr))
    topk = np.array([[2, 0, 3]])
    scale = 0.7
    out = orc.decode_absorbed(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, np.array([T]), scale)
    for h in range(H):
        s = {}
        for t in (2, 0, 3):
            acc = 0.0
            for d in range(Dn):
                kc = 0.0
                for c in range(C):
                    kc += c_kv[0, t, c] * wkv_b[h, d, c]
                acc += q_nope[0, h, d] * kc
            for r in range(Rr):
                acc += q_pe[0, h, r] * k_pe[0, t, r]
            s[t] = acc * scale
        mx = max(s.values())
        z = sum(math.exp(v - mx) for v in s.values())
        for d in range(Dv):
            o = 0.0
            for t in (2, 0, 3):
                v = 0.0
                for c in range(C):
                    v += c_kv[0, t, c] * wkv_b[h, Dn + d, c]
                o += math.exp(s[t] - mx) / z * v
            assert abs(out[0, h, d] - o) < 1e-12


# ---------------------------------------------------------------------------
# rotary embedding ("Rotated shared key", apply_rotary_emb)
# ---------------------------------------------------------------------------

def _angles(T, theta=1e4, Rr=64):
    j = np.arange(Rr // 2)
    return np.outer(np.arange(T), theta ** (-2.0 * j / Rr))


def test_rope_table_matches_definition():
    """R[t, j] = exp(i t theta^(-2j/64)) up to fp32 rounding of the angle."""
    T = 4096
    R = mi.rope_complex(mi.rope_table(T))
    ang = _angles(T)
    err = np.abs(R - np.exp(1j * ang))
    # the fp32 product t*freq carries up to ~T * 2^-24 rad of rounding
    assert err.max() < T * 2.0 ** -23 + 1e-6
    assert np.all(R[0] == 1.0)


def test_rope_position_zero_is_identity():
    x = np.random.default_rng(1).standard_normal((2, 1, 3, 64))
    R = np.ones((1, 32), dtype=complex)
    assert np.array_equal(orc.rope(x, R, True), x)
    assert np.array_equal(orc.rope(x, R, False), x)


def test_rope_unit_vector_closed_form():
    """Pair (1, 0) rotated by angle a becomes (cos a, sin a)."""
    ang = _angles(7)
    R = np.exp(1j * ang)
    x = np.zeros((1, 7, 1, 64))
    x[..., 0::2] = 1.0
    y = orc.rope(x, R, True)
    assert np.allclose(y[0, :, 0, 0::2], np.cos(ang), atol=1e-15)
    assert np.allclose(y[0, :, 0, 1::2], np.sin(ang), atol=1e-15)
    x2 = np.zeros((1, 7, 1, 64))
    x2[..., :32] = 1.0
    y2 = orc.rope(x2, R, False)
    assert np.allclose(y2[0, :, 0, :32], np.cos(ang), atol=1e-15)
    assert np.allclose(y2[0, :, 0, 32:], np.sin(ang), atol=1e-15)


def test_rope_preserves_pair_norms_and_relative_positions():
    rng = np.random.default_rng(3)
    T = 40
    R = np.exp(1j * _angles(T))
    q = rng.standard_normal(64)
    k = rng.standard_normal(64)
    xq = np.broadcast_to(q, (1, T, 1, 64)).copy()
    xk = np.broadcast_to(k, (1, T, 1, 64)).copy()
    rq = orc.rope(xq, R, True)[0, :, 0]
    rk = orc.rope(xk, R, True)[0, :, 0]
    pn = lambda v: v[..., 0::2] ** 2 + v[..., 1::2] ** 2  # noqa: E731
    assert np.allclose(pn(rq), pn(xq[0, :, 0]), atol=1e-12)
    # <RoPE(q, t1), RoPE(k, t2)> depends only on t1 - t2
    for d in (0, 3, 11):
        vals = [rq[t + d] @ rk[t] for t in range(0, T - d)]
        assert np.ptp(vals) < 1e-10


def test_rope_noninterleaved_is_permuted_interleaved():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 5, 3, 64))
    R = np.exp(1j * _angles(5))
    perm = np.empty(64, dtype=int)
    perm[0::2] = np.arange(32)
    perm[1::2] = np.arange(32, 64)
    inter = orc.rope(x[..., perm], R, True)
    non = orc.rope(x, R, False)
    assert np.allclose(non, inter[..., np.argsort(perm)], atol=1e-15)


# ---------------------------------------------------------------------------
# RMSNorm and cache write ("KV compression")
# ---------------------------------------------------------------------------

def test_rmsnorm_unit_rms():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 512)) * 3.0
    eps = 1e-6
    y = orc.rmsnorm(x, np.ones(512), eps)
    ms = np.mean(x * x, -1)
    assert np.allclose(np.sqrt(np.mean(y * y, -1)), np.sqrt(ms / (ms + eps)), rtol=1e-14)
    # positive homogeneity: y(a x) = y(x) when eps = 0
    assert np.allclose(orc.rmsnorm(7 * x, np.ones(512), 0.0), orc.rmsnorm(x, np.ones(512), 0.0),
                       rtol=1e-14)
    w = rng.standard_normal(512)
    assert np.allclose(orc.rmsnorm(x, w, eps), y * w, rtol=1e-14)


def test_cache_write_with_selection_weights():
    """With W_KVa a 0/1 selection matrix, kv is a column pick of x: the latent
    is RMSNorm of the picked columns, the rotary key is their rotation."""
    rng = np.random.default_rng(6)
    dim, C, Rr, rows = 40, 16, 4, 3
    x = rng.standard_normal((rows, dim))
    cols = rng.permutation(dim)[:C + Rr]
    W = np.zeros((dim, C + Rr))
    W[cols, np.arange(C + Rr)] = 1.0
    ang = rng.uniform(-3, 3, size=(rows, Rr // 2))
    Rp = np.exp(1j * ang)
    lat, pe = orc.cache_write(x, W, np.ones(C), 1e-6, Rp, C)
    pick = x[:, cols]
    ms = np.mean(pick[:, :C] ** 2, -1, keepdims=True)
    assert np.allclose(lat, pick[:, :C] / np.sqrt(ms + 1e-6), rtol=1e-14)
    a, b = pick[:, C::2], pick[:, C + 1::2]
    assert np.allclose(pe[:, 0::2], a * np.cos(ang) - b * np.sin(ang), atol=1e-14)
    assert np.allclose(pe[:, 1::2], a * np.sin(ang) + b * np.cos(ang), atol=1e-14)


# ---------------------------------------------------------------------------
# numbers printed on the pages
# ---------------------------------------------------------------------------

def _out_proj_problem(seed, B=3, H=4, Dv=5, dim=7):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, H, Dv)), rng.standard_normal((dim, H * Dv))


def test_out_proj_one_hot_selects_a_weight_column():
    """A single 1 at head h, value dim d of O picks column h*Dv + d of W_O
    ([out, in] storage, O flattened head-major as wo(x.flatten(2)) does)."""
    _, w = _out_proj_problem(0)
    B, H, Dv = 3, 4, 5
    for b, h, d in [(0, 0, 0), (1, 2, 3), (2, 3, 4), (0, 1, 0)]:
        o = np.zeros((B, H, Dv))
        o[b, h, d] = 1.0
        out = orc.out_proj(o, w)
        assert np.array_equal(out[b], w[:, h * Dv + d])
        others = [i for i in range(B) if i != b]
        assert not out[others].any()


def test_out_proj_is_linear():
    o1, w = _out_proj_problem(1)
    o2, _ = _out_proj_problem(2)
    a = -1.75
    lhs = orc.out_proj(a * o1 + o2, w)
    rhs = a * orc.out_proj(o1, w) + orc.out_proj(o2, w)
    assert np.abs(lhs - rhs).max() <= 1e-12 * (1 + np.abs(rhs).max())


def test_out_proj_mixes_heads_under_a_joint_permutation_only():
    """Renumbering the heads of O together with the matching column blocks of
    W_O leaves Delta unchanged; renumbering O alone does not (the projection
    is the step that mixes heads)."""
    o, w = _out_proj_problem(3)
    H, Dv = 4, 5
    perm = np.array([2, 0, 3, 1])
    cols = (perm[:, None] * Dv + np.arange(Dv)[None, :]).reshape(-1)
    ref = orc.out_proj(o, w)
    assert np.abs(orc.out_proj(o[:, perm, :], w[:, cols]) - ref).max() <= 1e-12 * np.abs(ref).max()
    assert np.abs(orc.out_proj(o[:, perm, :], w) - ref).max() > 1e-3


def test_out_proj_brute_force():
    o, w = _out_proj_problem(4)
    B, H, Dv = o.shape
    want = np.zeros((B, w.shape[0]))
    for b in range(B):
        for n in range(w.shape[0]):
            acc = 0.0
            for h in range(H):
                for d in range(Dv):
                    acc += o[b, h, d] * w[n, h * Dv + d]
            want[b, n] = acc
    assert np.abs(orc.out_proj(o, w) - want).max() <= 1e-12 * (1 + np.abs(want).max())


def _query_problem(seed, B=3, dim=10, ql=6, H=2, dn=4, rr=4):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, dim))
    wa = rng.standard_normal((ql, dim))
    w = 1.0 + 0.25 * rng.standard_normal(ql)
    wb = rng.standard_normal((H * (dn + rr), ql))
    R = np.exp(1j * rng.standard_normal((B, rr // 2)))
    return x, wa, w, wb, R


def test_query_proj_routes_heads_and_splits_nope_before_rope():
    """wq_a = [I 0] and w = 1, eps = 0 make qr = x[:, :ql] / rms; a one-hot
    wq_b sends qr[j] to (head h, feature e) of the head-major [H, dn + rr]
    view; at position 0 (R = 1) features e < dn land in q_nope[h, e] and the
    rest in q_pe[h, e - dn], exactly."""
    B, dim, ql, H, dn, rr = 2, 9, 5, 3, 4, 6
    rng = np.random.default_rng(5)
    x = rng.standard_normal((B, dim))
    wa = np.zeros((ql, dim))
    wa[np.arange(ql), np.arange(ql)] = 1.0
    t = x[:, :ql]
    qr = t / np.sqrt(np.mean(t * t, axis=1, keepdims=True))
    routes = [(0, 0, 0), (0, dn - 1, 1), (1, dn, 2), (2, dn + rr - 1, 4), (2, 1, 3)]
    wb = np.zeros((H * (dn + rr), ql))
    for h, e, j in routes:
        wb[h * (dn + rr) + e, j] = 1.0
    R0 = np.ones((B, rr // 2), dtype=complex)
    qn, qp = orc.query_proj(x, wa, np.ones(ql), 0.0, wb, R0, H, dn)
    assert qn.shape == (B, H, dn) and qp.shape == (B, H, rr)
    want_n, want_p = np.zeros((B, H, dn)), np.zeros((B, H, rr))
    for h, e, j in routes:
        if e < dn:
            want_n[:, h, e] = qr[:, j]
        else:
            want_p[:, h, e - dn] = qr[:, j]
    assert np.abs(qn - want_n).max() <= 1e-12
    assert np.abs(qp - want_p).max() <= 1e-12


def test_query_proj_is_scale_invariant_through_the_norm():
    """With eps = 0 the RMSNorm cancels any positive scale of x."""
    x, wa, w, wb, R = _query_problem(6)
    a = orc.query_proj(x, wa, w, 0.0, wb, R, 2, 4)
    b = orc.query_proj(3.7 * x, wa, w, 0.0, wb, R, 2, 4)
    for u, v in zip(a, b):
        assert np.abs(u - v).max() <= 1e-12 * np.abs(u).max()


def test_query_proj_position_moves_only_the_rotary_part():
    x, wa, w, wb, R = _query_problem(7)
    R2 = R * np.exp(1j * np.array([0.3, -1.1]))
    n1, p1 = orc.query_proj(x, wa, w, 1e-6, wb, R, 2, 4)
    n2, p2 = orc.query_proj(x, wa, w, 1e-6, wb, R2, 2, 4)
    assert np.array_equal(n1, n2)
    assert np.abs(p1 - p2).max() > 1e-3
    pair = lambda p: p[..., 0::2] ** 2 + p[..., 1::2] ** 2  # noqa: E731
    assert np.abs(pair(p1) - pair(p2)).max() <= 1e-12 * pair(p1).max()


def test_query_proj_brute_force():
    B, dim, ql, H, dn, rr = 2, 5, 4, 2, 3, 4
    x, wa, w, wb, _ = _query_problem(8, B, dim, ql, H, dn, rr)
    ang = np.random.default_rng(9).standard_normal((B, rr // 2))
    R = np.cos(ang) + 1j * np.sin(ang)
    eps = 1e-6
    qn_want = np.zeros((B, H, dn))
    qp_want = np.zeros((B, H, rr))
    for b in range(B):
        t = [sum(x[b, i] * wa[o, i] for i in range(dim)) for o in range(ql)]
        ms = sum(v * v for v in t) / ql
        qr = [t[o] / math.sqrt(ms + eps) * w[o] for o in range(ql)]
        for h in range(H):
            feats = [sum(qr[j] * wb[h * (dn + rr) + e, j] for j in range(ql)) for e in range(dn + rr)]
            for e in range(dn):
                qn_want[b, h, e] = feats[e]
            for p in range(rr // 2):
                x0, x1 = feats[dn + 2 * p], feats[dn + 2 * p + 1]
                c, s_ = math.cos(ang[b, p]), math.sin(ang[b, p])
                qp_want[b, h, 2 * p] = x0 * c - x1 * s_
                qp_want[b, h, 2 * p + 1] = x0 * s_ + x1 * c
    qn, qp = orc.query_proj(x, wa, w, eps, wb, R, H, dn)
    assert np.abs(qn - qn_want).max() <= 1e-12 * (1 + np.abs(qn_want).max())
    assert np.abs(qp - qp_want).max() <= 1e-12 * (1 + np.abs(qp_want).max())


def test_parameter_counts_match_the_pages():
    gold = json.load(open(os.path.join(GOLD, "param_counts.json")))
    pc = orc.parameter_counts()
    for key in ("W_UK", "W_KR", "key_heads_total", "wkv_a_latent", "kv_norm",
                "kv_compression_total", "W_O", "W_QR", "cache_per_position",
                "full_kv_per_position"):
        assert pc[key] == gold[key]["value"], key
    assert pc["key_heads_total"] * 58 == gold["key_heads_x58"]["value"]
    assert pc["W_O"] * 58 == gold["W_O_x58"]["value"]
    assert pc["W_QR"] * 58 == gold["W_QR_x58"]["value"]
    assert pc["kv_compression_total"] * 58 == gold["kv_compression_x58"]["value"]
    # wkv_a + kv_norm = 7168 x 576 + 512 = latent part + rotary part + norm
    assert pc["wkv_a_plus_norm"] == gold["wkv_a_latent"]["value"] + gold["W_KR"]["value"] \
        + gold["kv_norm"]["value"]
    # wkv_b = W_UK + W_UV, each 512 x 16,384
    assert pc["wkv_b"] == 2 * gold["W_UK"]["value"]


def test_decode_example_shape_from_the_pages():
    """'Mix and project' at position 1000: A is [B, 128 heads, 1 query, 1001
    keys] and c^KV is [B, 1001, 512].  The all-selected tiny workload has
    exactly this shape."""
    wl = mi.make_config(0)
    assert tuple(wl.cache.shape) == (1, 1001, 576)
    assert int(wl.end_pos[0]) == 1001 and wl.k == 1001
    rows = mi.f64(wl.cache)
    _, ws = orc.decode_absorbed(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                                rows[..., :512], rows[..., 512:], wl.topk.numpy(),
                                wl.end_pos.numpy(), wl.scale, return_weights=True)
    A, keep = ws[0]
    assert A.shape == (128, 1001) and sorted(keep) == list(range(1001))


def test_score_scale_is_unit_variance_for_the_workloads():
    """With the workload distributions, scaled scores have variance ~1
    (128*512*(1/512) + 64 = 192, times 1/192): a non-degenerate softmax."""
    wl = mi.make_small(B=2, T=300, k=200, seed=9)
    q_t = orc.fold_wuk(mi.f64(wl.q_nope), mi.f64(wl.wkv_b))
    rows = mi.f64(wl.cache[0, :200])
    s = orc.scores(q_t[0], mi.f64(wl.q_pe[0]), rows[:, :512], rows[:, 512:], wl.scale)
    assert 0.8 < s.var() < 1.25


def test_inputs_are_seeded_and_shapes_match():
    a = mi.make_small(seed=1)
    b = mi.make_small(seed=1)
    assert torch.equal(a.cache, b.cache) and torch.equal(a.topk, b.topk)
    for b_ in range(a.B):
        row = a.topk[b_].tolist()
        valid = [v for v in row if 0 <= v < int(a.end_pos[b_])]
        assert len(set(valid)) == len(valid)
    w3 = mi.make_config(1)
    assert tuple(w3.topk.shape) == (8, 2048)
    for b_ in range(8):
        assert len(set(w3.topk[b_].tolist())) == 2048


# ---------------------------------------------------------------------------
# sparse prefill ("Mix and project", MHA prefill branch) and multi-query decode
# ---------------------------------------------------------------------------

def _prefill_problem(seed, B=2, S=9, H=3, Dn=4, Dv=3, C=6, Rr=4, k=5, future=True):
    """Hand-sized prefill: each token lists up to k positions; with `future`
    some listed positions lie after the token (the causal mask removes them)."""
    rng = np.random.default_rng(seed)
    qn = rng.standard_normal((B, S, H, Dn))
    qp = rng.standard_normal((B, S, H, Rr))
    wkv = rng.standard_normal((H, Dn + Dv, C)) / math.sqrt(C)
    c = rng.standard_normal((B, S + 2, C))
    pe = rng.standard_normal((B, S + 2, Rr))
    topk = np.full((B, S, k), -1, dtype=np.int64)
    for b in range(B):
        for s in range(S):
            hi = S if future else s + 1
            pick = rng.choice(hi, size=min(k, hi), replace=False)
            topk[b, s, :len(pick)] = pick
    return qn, qp, wkv, c, pe, topk, 0.4


def test_prefill_equals_absorbed_decode_per_token():
    """The expanded-key prefill equals the absorbed decode of each token on its
    own ("Key heads": folding W_UK into the query gives the same scores), with
    the token's causal limit s + 1 as end_pos: listed positions after the
    token are excluded in both."""
    qn, qp, wkv, c, pe, topk, scale = _prefill_problem(31)
    got = orc.prefill_materialised(qn, qp, wkv, c, pe, topk, scale)
    B, S = qn.shape[:2]
    for b in range(B):
        want = orc.decode_absorbed(qn[b], qp[b], wkv, np.repeat(c[b:b + 1], S, 0),
                                   np.repeat(pe[b:b + 1], S, 0), topk[b], np.arange(1, S + 1),
                                   scale)
        assert np.abs(got[b] - want).max() <= 1e-12


def test_prefill_first_token_sees_only_itself():
    """Token 0 may attend only to position 0: with 0 listed its output is the
    value of position 0, W_UV[h] c[0], for every head (softmax of one key)."""
    qn, qp, wkv, c, pe, topk, scale = _prefill_problem(32)
    topk[:, 0, 0] = 0
    got = orc.prefill_materialised(qn, qp, wkv, c, pe, topk, scale)
    Dn = qn.shape[-1]
    for b in range(qn.shape[0]):
        want = np.einsum("hdc,c->hd", wkv[:, Dn:, :], c[b, 0])
        assert np.abs(got[b, 0] - want).max() <= 1e-12


def test_prefill_ignores_future_and_unlisted_positions():
    """Changing the cache rows of positions after a token, or of positions it
    does not list, leaves that token's output unchanged; changing a listed
    earlier position changes it."""
    qn, qp, wkv, c, pe, topk, scale = _prefill_problem(33)
    base = orc.prefill_materialised(qn, qp, wkv, c, pe, topk, scale)
    S = qn.shape[1]
    s = S // 2
    listed = sorted(t for t in topk[0, s].tolist() if 0 <= t <= s)
    others = [t for t in range(S) if t > s or t not in listed]
    c2, pe2 = c.copy(), pe.copy()
    c2[0, others] += 3.0
    pe2[0, others] -= 2.0
    moved = orc.prefill_materialised(qn, qp, wkv, c2, pe2, topk, scale)
    assert np.abs(moved[0, s] - base[0, s]).max() <= 1e-12
    assert listed, "the token lists an earlier position"
    c3 = c.copy()
    c3[0, listed[0]] += 1.0
    changed = orc.prefill_materialised(qn, qp, wkv, c3, pe, topk, scale)
    assert np.abs(changed[0, s] - base[0, s]).max() > 1e-6


def test_prefill_brute_force():
    """Scalar loops over tokens, heads, listed earlier positions and
    features on a tiny case."""
    qn, qp, wkv, c, pe, topk, scale = _prefill_problem(34, B=1, S=5, H=2, Dn=2, Dv=2, C=3,
                                                        Rr=2, k=4)
    got = orc.prefill_materialised(qn, qp, wkv, c, pe, topk, scale)
    S, H, Dn, Dv, C, Rr = 5, 2, 2, 2, 3, 2
    for s in range(S):
        keys = sorted(set(t for t in topk[0, s].tolist() if 0 <= t <= s))
        for h in range(H):
            if not keys:
                assert np.abs(got[0, s, h]).max() == 0.0
                continue
            sc = []
            for t in keys:
                acc = 0.0
                for d in range(Dn):
                    kd = sum(wkv[h, d, j] * c[0, t, j] for j in range(C))
                    acc += qn[0, s, h, d] * kd
                for r in range(Rr):
                    acc += qp[0, s, h, r] * pe[0, t, r]
                sc.append(acc * scale)
            m = max(sc)
            e = [math.exp(x - m) for x in sc]
            z = sum(e)
            for d in range(Dv):
                want = 0.0
                for t, w in zip(keys, e):
                    want += (w / z) * sum(wkv[h, Dn + d, j] * c[0, t, j] for j in range(C))
                assert abs(got[0, s, h, d] - want) <= 1e-12


def test_multi_query_matches_materialised_per_query():
    """Several query rows per cache row: each row equals the expanded-key path
    run on its own cache row (the cache repeated per query), with its own
    selection and limit."""
    rng = np.random.default_rng(35)
    qn, qp, wkv, c, pe, topk, end_pos, scale = _rand_problem(rng, B=6, T=30, k=11)
    q = 3
    got = orc.decode_multi_query(qn, qp, wkv, c[:2], pe[:2], topk, end_pos, scale, q)
    want = orc.decode_materialised(qn, qp, wkv, np.repeat(c[:2], q, 0), np.repeat(pe[:2], q, 0),
                                   topk, end_pos, scale)
    assert np.abs(got - want).max() <= 1e-12
    other = orc.decode_multi_query(qn, qp, wkv, c[2:4], pe[2:4], topk, end_pos, scale, q)
    assert np.abs(other - got).max() > 1e-6  # the cache rows are used


def test_prefill_and_multi_query_inputs_are_causal_and_seeded():
    """Each query row lists distinct positions inside its causal limit, as
    many as the limit allows up to k, with -1 padding only after them; the
    draws repeat under the same seed."""
    pf = mi.make_prefill(B=2, S=70, k=40, seed=3)
    again = mi.make_prefill(B=2, S=70, k=40, seed=3)
    assert torch.equal(pf.topk, again.topk) and torch.equal(pf.q_nope, again.q_nope)
    assert pf.queries_per_row == 70 and pf.B == 140 and tuple(pf.cache.shape) == (2, 70, 576)
    for r in range(pf.B):
        lim = int(pf.end_pos[r])
        assert lim == r % 70 + 1
        row = pf.topk[r].tolist()
        n = min(40, lim)
        assert all(0 <= t < lim for t in row[:n]) and len(set(row[:n])) == n
        assert all(t == -1 for t in row[n:])
    mq = mi.make_multi_query(B=3, S=2, T=9000, k=64, seed=4)
    assert mq.queries_per_row == 2 and tuple(mq.cache.shape) == (3, 9000, 576)
    for r in range(mq.B):
        lim = int(mq.end_pos[r])
        row = mq.topk[r].tolist()
        assert all(0 <= t < lim for t in row) and len(set(row)) == 64
        if r % 2 == 0:
            assert lim == int(mq.end_pos[r + 1]) - 1  # token 0 sees one position less
        recent = sum(t >= lim - 4096 for t in row)
        assert recent >= 32  # half from the last 4096 positions (T > 8192)


def test_prefill_and_multi_query_degenerate_cases():
    """A one-token prompt is that token attending to itself (the value of
    position 0); one query per cache row is plain decode; a prefill token
    whose list holds only positions after it gets O = 0."""
    qn, qp, wkv, c, pe, topk, scale = _prefill_problem(36, B=2, S=1, k=3)
    topk[:] = -1
    topk[:, 0, 0] = 0
    got = orc.prefill_materialised(qn, qp, wkv, c, pe, topk, scale)
    Dn = qn.shape[-1]
    for b in range(2):
        assert np.abs(got[b, 0] - np.einsum("hdc,c->hd", wkv[:, Dn:, :], c[b, 0])).max() <= 1e-12
    rng = np.random.default_rng(37)
    qn1, qp1, wkv1, c1, pe1, topk1, end1, scale1 = _rand_problem(rng, B=3, T=25, k=9)
    a = orc.decode_multi_query(qn1, qp1, wkv1, c1, pe1, topk1, end1, scale1, 1)
    b_ = orc.decode_materialised(qn1, qp1, wkv1, c1, pe1, topk1, end1, scale1)
    assert np.abs(a - b_).max() <= 1e-12
    qn, qp, wkv, c, pe, topk, scale = _prefill_problem(38, B=1, S=6, k=2)
    topk[0, 2] = [4, 5]  # token 2 lists only later positions
    got = orc.prefill_materialised(qn, qp, wkv, c, pe, topk, scale)
    assert np.abs(got[0, 2]).max() == 0.0


def test_workload_tensors_have_the_printed_sizes():
    """The tensors the GPU tests and the bench feed the kernels have the
    sizes the pages print: W_O 117,440,512 weights, the rotary rows of wq_b
    12,582,912, wkv_b twice W_UK (8,388,608 each), 576 cached values per
    position."""
    gold = json.load(open(os.path.join(GOLD, "param_counts.json")))
    _, w_o = mi.make_out_proj(B=1, seed=0)
    assert w_o.numel() == gold["W_O"]["value"]
    x, wq_a, qn_w, wq_b, tab, pos = mi.make_query_proj(B=1, T=8, seed=0)
    assert wq_b.view(128, 192, 1536)[:, 128:, :].numel() == gold["W_QR"]["value"]
    wl = mi.make_small(B=1, T=40, k=8, seed=0)
    assert wl.wkv_b.numel() == 2 * gold["W_UK"]["value"]
    assert wl.cache.shape[-1] == gold["cache_per_position"]["value"]
