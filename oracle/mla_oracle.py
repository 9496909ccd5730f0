"""CPU oracle for the absorbed sparse-MLA decode step (float64, numpy).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package entry point's smoke
check and the bench's CPU-baseline leg may import this module.  The CUDA
library never calls it, and it shares no code with the CUDA path.

Every function is a plain restatement of what the DeepSeek-V3.2-Exp pages
define, in float64, with no blocking, fusion or reordering beyond the stated
equations.  Library primitives (numpy matmul/einsum, exp, sqrt) serve as
single steps.  All functions are shape-generic (head count, latent width,
rotary width and head dims are taken from the arguments) so that tests can
run them on hand-sized problems.

Sources (page title, section):
  * "Mix and project" (the decode code excerpt): absorbed decode --
    fold W_UK into q_nope, score against the cached latent plus the shared
    rotary key over the indexer's selected positions, scale, softmax, mix
    the latent, apply W_UV per head.
  * "Key heads" (equations k^C = c^KV W_UK, K_i = [K^C_i ; k^R]; the
    prefill code excerpt): the materialised path used as a cross-check.
  * "KV compression" (the key-value down-projection excerpt) and "Rotated
    shared key" (the apply_rotary_emb excerpt): cache write and rotary
    embedding.
  * "Mix and project" (the output projection wo and its parameter count):
    Delta_attn = flatten(O) W_O^T.
  * "Query rotary up-projection" (the MLA init and forward excerpts): the
    query path wq_a -> q_norm -> wq_b -> split -> RoPE.
  * "Mix and project" (the MHA prefill branch of the forward excerpt): sparse
    prefill with expanded per-head keys and values under the index mask plus
    the causal mask; multi-query decode is the decode definition applied to
    several query rows that share one cache row.

Readings taken where the pages are silent:
  * index semantics follow the decode mask built by scatter of 0 into a -inf
    row over [0, end_pos): a position counts once however often it is
    listed; -1 is padding; any other index outside [0, end_pos) is ignored
    and counted as invalid;
  * a row whose selection is empty gives O = 0 (the reference softmax would
    produce NaN);
  * RMSNorm is y = x / sqrt(mean(x^2) + eps) * w;
  * end_pos is given per batch row.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(equivalences, closed forms, invariants, brute force and the pages' printed
parameter counts); there is no printed numeric output on the pages to match.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------


def selected_positions(topk_row, end_pos: int, T: int):
    """Valid distinct positions of one row, in first-occurrence order, and the
    number of invalid entries (neither -1 padding nor in [0, min(end_pos, T)))."""
    seen = set()
    keep = []
    invalid = 0
    lim = min(int(end_pos), int(T))
    for v in np.asarray(topk_row).tolist():
        v = int(v)
        if v == -1:
            continue
        if v < 0 or v >= lim:
            invalid += 1
            continue
        if v not in seen:
            seen.add(v)
            keep.append(v)
    return keep, invalid


def index_mask(topk, end_pos, T: int):
    """mask[b, t] = 1 iff t is listed in topk[b] and 0 <= t < end_pos[b].

    Mirrors the decode mask ("Mix and project", decode listing): a -inf row
    over [0, end_pos) into which the indexer's positions are scattered as 0.
    Returns (uint8 mask [B, T], total count of invalid entries)."""
    topk = np.asarray(topk)
    B = topk.shape[0]
    mask = np.zeros((B, T), dtype=np.uint8)
    bad = 0
    for b in range(B):
        keep, inv = selected_positions(topk[b], int(end_pos[b]), T)
        mask[b, keep] = 1
        bad += inv
    return mask, bad


# ---------------------------------------------------------------------------
# absorbed decode, step by step ("Mix and project", decode branch)
# ---------------------------------------------------------------------------


def fold_wuk(q_nope, wkv_b):
    """q~[b,h,c] = sum_d q_nope[b,h,d] * W_UK[h,d,c], W_UK = wkv_b[:, :Dn, :]."""
    Dn = q_nope.shape[-1]
    w_uk = wkv_b[:, :Dn, :]
    return np.einsum("bhd,hdc->bhc", q_nope, w_uk)


def scores(q_tilde_bh, q_pe_bh, c_rows, pe_rows, scale):
    """s[h,t] = (q~[h]·c_KV[t] + q_pe[h]·k_pe[t]) * softmax_scale."""
    return (q_tilde_bh @ c_rows.T + q_pe_bh @ pe_rows.T) * scale


def softmax_rows(s):
    """Row softmax with the row maximum subtracted."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def mix_latent(A, c_rows):
    """O~[h,c] = sum_t A[h,t] * c_KV[t,c]."""
    return A @ c_rows


def apply_wuv(o_tilde, wkv_b, Dv):
    """O[h,d] = sum_c O~[h,c] * W_UV[h,d,c], W_UV = wkv_b[:, -Dv:, :]."""
    w_uv = wkv_b[:, -Dv:, :]
    return np.einsum("hc,hdc->hd", o_tilde, w_uv)


def decode_absorbed(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale,
                    return_weights=False):
    """Absorbed sparse decode for one query per batch row.

    q_nope [B,H,Dn], q_pe [B,H,Rr], wkv_b [H, Dn+Dv, C], c_kv [B,T,C],
    k_pe [B,T,Rr], topk [B,k] int, end_pos [B] int -> O [B,H,Dv] float64.
    With return_weights the per-row attention weights and selected positions
    are returned as well."""
    q_nope = np.asarray(q_nope, dtype=np.float64)
    q_pe = np.asarray(q_pe, dtype=np.float64)
    wkv_b = np.asarray(wkv_b, dtype=np.float64)
    B, Hh, Dn = q_nope.shape
    Dv = wkv_b.shape[1] - Dn
    T = c_kv.shape[1]
    q_tilde = fold_wuk(q_nope, wkv_b)
    out = np.zeros((B, Hh, Dv))
    weights = []
    for b in range(B):
        keep, _ = selected_positions(topk[b], int(end_pos[b]), T)
        if not keep:
            weights.append((np.zeros((Hh, 0)), keep))
            continue
        c_rows = np.asarray(c_kv[b, keep], dtype=np.float64)
        pe_rows = np.asarray(k_pe[b, keep], dtype=np.float64)
        s = scores(q_tilde[b], q_pe[b], c_rows, pe_rows, scale)
        A = softmax_rows(s)
        out[b] = apply_wuv(mix_latent(A, c_rows), wkv_b, Dv)
        weights.append((A, keep))
    if return_weights:
        return out, weights
    return out


# ---------------------------------------------------------------------------
# materialised path ("Key heads": K_i = [c^KV W_UK,i ; k^R], V_i = c^KV W_UV,i)
# ---------------------------------------------------------------------------


def decode_materialised(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale):
    """Per-head keys and values are expanded from the latent, every position
    in [0, end_pos) is scored, the index mask (-inf everywhere, 0 at the
    listed positions) is added, then softmax and the value mix -- the shape
    of the prefill branch, specialised to one query."""
    q_nope = np.asarray(q_nope, dtype=np.float64)
    q_pe = np.asarray(q_pe, dtype=np.float64)
    wkv_b = np.asarray(wkv_b, dtype=np.float64)
    B, Hh, Dn = q_nope.shape
    Dv = wkv_b.shape[1] - Dn
    T = c_kv.shape[1]
    out = np.zeros((B, Hh, Dv))
    for b in range(B):
        e = min(int(end_pos[b]), T)
        c = np.asarray(c_kv[b, :e], dtype=np.float64)          # [e, C]
        kv = np.einsum("tc,hjc->thj", c, wkv_b)                # [e, H, Dn+Dv]
        k_nope, v = kv[:, :, :Dn], kv[:, :, Dn:]
        pe = np.asarray(k_pe[b, :e], dtype=np.float64)         # [e, Rr]
        k = np.concatenate([k_nope, np.broadcast_to(pe[:, None, :], (e, Hh, pe.shape[1]))], -1)
        q = np.concatenate([q_nope[b], q_pe[b]], -1)           # [H, Dn+Rr]
        s = np.einsum("hd,thd->ht", q, k) * scale
        mask = np.full(e, -np.inf)
        for v_idx in np.asarray(topk[b]).tolist():
            if 0 <= v_idx < e:
                mask[v_idx] = 0.0
        s = s + mask[None, :]
        if not np.isfinite(mask).any():
            continue
        m = s.max(-1, keepdims=True)
        p = np.exp(s - m)
        p = p / p.sum(-1, keepdims=True)
        out[b] = np.einsum("ht,thd->hd", p, v)
    return out


# ---------------------------------------------------------------------------
# sparse prefill ("Mix and project", the MHA prefill branch of the forward
# excerpt) and multi-query decode
# ---------------------------------------------------------------------------


def prefill_mask(topk_b, S):
    """The prefill branch's mask for one sequence of S tokens: the index mask
    (-inf everywhere, 0 at each token's listed positions inside [0, S)) plus
    the causal mask (-inf where the key position is after the token) -> [S, S]."""
    index_mask = np.full((S, S), -np.inf)
    for s_ in range(S):
        for t in np.asarray(topk_b[s_]).tolist():
            if 0 <= t < S:
                index_mask[s_, t] = 0.0
    return index_mask + np.triu(np.full((S, S), -np.inf), 1)


def expand_keys_values(c, pe, wkv_b, Dn):
    """Per-head keys and values of the prefill branch from latent rows c [S, C]
    and rotary keys pe [S, Rr]: kv = wkv_b(c) split into k_nope (first Dn
    rows of each head) and v (the rest); k = [k_nope ; pe broadcast to every
    head] -> (k [S, H, Dn+Rr], v [S, H, Dv])."""
    kv = np.einsum("tc,hjc->thj", c, wkv_b)                    # [S, H, Dn+Dv]
    k_nope, v = kv[:, :, :Dn], kv[:, :, Dn:]
    Hh = wkv_b.shape[0]
    k = np.concatenate([k_nope, np.broadcast_to(pe[:, None, :], (c.shape[0], Hh, pe.shape[1]))],
                       -1)
    return k, v


def prefill_materialised(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, scale):
    """Prefill of a prompt of S tokens per sequence, cached at positions
    0 .. S-1, following the prefill branch step by step:

      q      = [q_nope ; q_pe]                              per token and head
      k, v   = expand_keys_values(c_KV, k_pe)               expanded per head
      scores = q . k * scale                                [S, H, S]
      O      = softmax_t(scores + prefill_mask) . v

    q_nope [B,S,H,Dn], q_pe [B,S,H,Rr], wkv_b [H, Dn+Dv, C], c_kv [B,T,C],
    k_pe [B,T,Rr] with T >= S, topk [B,S,k] int (-1 = padding) ->
    O [B,S,H,Dv] float64.  A token whose masked row has no finite entry
    gets O = 0 (the reading taken for an empty selection in decode)."""
    q_nope = np.asarray(q_nope, dtype=np.float64)
    q_pe = np.asarray(q_pe, dtype=np.float64)
    wkv_b = np.asarray(wkv_b, dtype=np.float64)
    B, S, Hh, Dn = q_nope.shape
    Dv = wkv_b.shape[1] - Dn
    out = np.zeros((B, S, Hh, Dv))
    for b in range(B):
        c = np.asarray(c_kv[b, :S], dtype=np.float64)          # [S, C]
        pe = np.asarray(k_pe[b, :S], dtype=np.float64)         # [S, Rr]
        k, v = expand_keys_values(c, pe, wkv_b, Dn)
        q = np.concatenate([q_nope[b], q_pe[b]], -1)           # [S, H, Dn+Rr]
        mask = prefill_mask(topk[b], S)
        sc = np.einsum("shd,thd->sht", q, k) * scale + mask[:, None, :]
        for s_ in range(S):
            if not np.isfinite(mask[s_]).any():
                continue
            row = sc[s_]                                        # [H, S]
            p = np.exp(row - row.max(-1, keepdims=True))
            p = p / p.sum(-1, keepdims=True)
            out[b, s_] = np.einsum("ht,thd->hd", p, v)
    return out


def decode_multi_query(q_nope, q_pe, wkv_b, c_kv, k_pe, topk, end_pos, scale, queries_per_row):
    """Absorbed decode of B query rows over B / queries_per_row cache rows:
    query row r is scored against cache row r // queries_per_row with its own
    selection topk[r] and limit end_pos[r] -- the decode definition applied to
    each query row."""
    rows = np.arange(np.asarray(q_nope).shape[0]) // int(queries_per_row)
    return decode_absorbed(q_nope, q_pe, wkv_b, np.asarray(c_kv)[rows], np.asarray(k_pe)[rows],
                           topk, end_pos, scale)


# ---------------------------------------------------------------------------
# rotary embedding ("Rotated shared key", apply_rotary_emb)
# ---------------------------------------------------------------------------


def rope(x, R, interleaved=True):
    """Rotate feature pairs of x [..., S, Hx, Rr] by R [S, Rr/2] (complex).

    interleaved: pair j is (x[2j], x[2j+1]) and the result goes back to
    (2j, 2j+1).  Otherwise pair j is (x[j], x[j+Rr/2]) and the result is laid
    out as all real parts, then all imaginary parts."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    if interleaved:
        z = x[..., 0::2] + 1j * x[..., 1::2]
    else:
        z = x[..., :half] + 1j * x[..., half:]
    y = z * R[:, None, :]
    out = np.empty_like(x)
    if interleaved:
        out[..., 0::2] = y.real
        out[..., 1::2] = y.imag
    else:
        out[..., :half] = y.real
        out[..., half:] = y.imag
    return out


# ---------------------------------------------------------------------------
# cache write ("KV compression", key-value down-projection excerpt)
# ---------------------------------------------------------------------------


def rmsnorm(x, w, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, dtype=np.float64)


def cache_write(x, w_kva, norm_w, eps, R_pos, C, interleaved=True):
    """kv = x W_KVa, split [C latent, rotary]; latent -> RMSNorm; rotary ->
    RoPE at the row's position.  x [rows, dim], w_kva [dim, C+Rr] (x·W form),
    R_pos complex [rows, Rr/2] (the rotary coefficients of each row's
    position).  Returns (latent [rows, C], rotary key [rows, Rr]) in float64."""
    kv = np.asarray(x, dtype=np.float64) @ np.asarray(w_kva, dtype=np.float64)
    lat, pe = kv[:, :C], kv[:, C:]
    lat = rmsnorm(lat, norm_w, eps)
    pe = rope(pe[:, None, :], R_pos, interleaved)[:, 0, :]
    return lat, pe


# ---------------------------------------------------------------------------
# query path ("Query rotary up-projection": the MLA init and forward excerpts;
# W_QR is output features Dn..Dn+Rr of each head's block in wq_b)
# ---------------------------------------------------------------------------


def query_proj(x, wq_a, q_norm_w, eps, wq_b, R_pos, n_heads, dn, interleaved=True):
    """qr = RMSNorm(x wq_a^T) * w;  q = qr wq_b^T viewed [B, n_heads, dn + rr];
    q_nope = q[..., :dn];  q_pe = RoPE(q[..., dn:]) at each row's position.

    x [B, dim], wq_a [q_lora, dim] and wq_b [n_heads*(dn+rr), q_lora] stored
    [out, in]; R_pos complex [B, rr/2] (the rotary coefficients of each row's
    query position).  Returns (q_nope [B, n_heads, dn], q_pe [B, n_heads, rr])."""
    t = np.asarray(x, dtype=np.float64) @ np.asarray(wq_a, dtype=np.float64).T
    qr = rmsnorm(t, q_norm_w, eps)
    q = qr @ np.asarray(wq_b, dtype=np.float64).T
    B = q.shape[0]
    q = q.reshape(B, n_heads, -1)
    q_nope, q_pe = q[..., :dn], q[..., dn:]
    # rope takes [..., S, Hx, Rr] with R [S, Rr/2]: treat the batch as positions
    q_pe = rope(q_pe, np.asarray(R_pos), interleaved)
    return q_nope, q_pe


# ---------------------------------------------------------------------------
# output projection ("Mix and project": the output projection wo, the only
# step that mixes heads; Delta_attn [B, dim])
# ---------------------------------------------------------------------------


def out_proj(o, w_o):
    """Delta[b, n] = sum over heads h and value dims d of O[b,h,d] * W_O[n, h*Dv + d].

    O [B, H, Dv] is flattened over (head, value dim) in that order, as the
    decode excerpt's wo(x.flatten(2)) does; W_O is stored [out, in] =
    [dim, H*Dv] and applied as x W_O^T."""
    o = np.asarray(o, dtype=np.float64)
    x = o.reshape(o.shape[0], -1)
    return x @ np.asarray(w_o, dtype=np.float64).T


# ---------------------------------------------------------------------------
# parameter counts (printed on the "Key heads", "KV compression", "Mix and
# project" and "Query rotary up-projection" pages)
# ---------------------------------------------------------------------------


def parameter_counts(n_heads=128, kv_lora_rank=512, qk_nope=128, qk_rope=64,
                     v_head=128, dim=7168, q_lora_rank=1536):
    return {
        "W_UK": kv_lora_rank * n_heads * qk_nope,
        "W_KR": dim * qk_rope,
        "key_heads_total": kv_lora_rank * n_heads * qk_nope + dim * qk_rope,
        "wkv_a_latent": dim * kv_lora_rank,
        "kv_norm": kv_lora_rank,
        "kv_compression_total": dim * kv_lora_rank + kv_lora_rank,
        "wkv_a_plus_norm": dim * (kv_lora_rank + qk_rope) + kv_lora_rank,
        "W_O": n_heads * v_head * dim,
        "W_QR": q_lora_rank * n_heads * qk_rope,
        "wkv_b": kv_lora_rank * n_heads * (qk_nope + v_head),
        "cache_per_position": kv_lora_rank + qk_rope,
        "full_kv_per_position": n_heads * ((qk_nope + qk_rope) + v_head),
    }
