"""Seeded synthetic workloads for the absorbed sparse-MLA decode step.

This module is shared by the CUDA-path tests, the bench and the oracle-side
tests.  It holds no arithmetic of the method itself: it only draws random
tensors with the shapes and distributions of the workloads, draws the top-k
index sets, builds the fp32 rotary table that the model precomputes once at
start-up (it is an *input* of the rope and cache-write calls), and converts
bf16 tensors to float64 numpy arrays (an exact widening).

Dimensions follow the DeepSeek-V3.2-Exp MLA block ("Key heads" page, MLA
init listing): 128 heads, a 512-wide key/value latent, a 64-wide shared rotary
key, 128-wide non-rotary query/key parts and 128-wide values; the model width
is 7168 ("KV compression" page, parameter table).

Distribution notation N(0, v) is read as variance v.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

H = 128          # query heads
C = 512          # kv latent width (kv_lora_rank)
R = 64           # shared rotary key width (qk_rope_head_dim)
DN = 128         # non-rotary query/key part per head (qk_nope_head_dim)
DV = 128         # value width per head (v_head_dim)
KROW = C + R     # 576 cached values per position
DIM = 7168       # model width
QL = 1536        # query latent width (q_lora_rank)
THETA = 1.0e4    # rope_theta


def softmax_scale(m: float = 1.0) -> float:
    """qk_head_dim**-0.5 times mscale**2 (MLA init listing); m=1 leaves it."""
    return (DN + R) ** -0.5 * m * m


@dataclasses.dataclass
class Workload:
    """One decode workload.  Tensors live on ``device``.

    cache    bf16 [B, T, 576]   fused row: latent c_KV in 0..511, k_pe in 512..575
    q_nope   bf16 [B, 128, 128]
    q_pe     bf16 [B, 128, 64]
    wkv_b    bf16 [128, 256, 512] (rows 0..127 = W_UK, 128..255 = W_UV per head)
    topk     int32 [B, k]
    end_pos  int32 [B]
    scale    float
    For the cache-write workload additionally:
    x        bf16 [B, 7168], w_kva bf16 [7168, 576], norm_w bf16 [512],
    rope     fp32 [T, 32, 2] (cos, sin), write_pos int, eps float
    """
    name: str
    B: int
    T: int
    k: int
    cache: torch.Tensor
    q_nope: torch.Tensor
    q_pe: torch.Tensor
    wkv_b: torch.Tensor
    topk: torch.Tensor
    end_pos: torch.Tensor
    scale: float
    x: Optional[torch.Tensor] = None
    w_kva: Optional[torch.Tensor] = None
    norm_w: Optional[torch.Tensor] = None
    rope: Optional[torch.Tensor] = None
    write_pos: Optional[int] = None
    eps: float = 1e-6


# --------------------------------------------------------------------------
# random draws
# --------------------------------------------------------------------------

def _normal_bf16(shape, std, gen, device):
    """Draw N(0, std^2) in fp32 and round to bf16 (round-to-nearest-even)."""
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def rope_table(T: int, theta: float = THETA) -> torch.Tensor:
    """fp32 rotary coefficients [T, 32, 2] = (cos, sin) of t * theta^(-2j/64).

    Built like the model's precomputed table ("Rotated shared key" page,
    precompute_freqs_cis): fp32 frequencies, the fp32 outer product with an
    integer position range, then unit-modulus polar form.  YaRN blending is
    not applied (its helpers are not given on the pages).  Returned on CPU.
    """
    j = torch.arange(0, R, 2, dtype=torch.float32)
    freqs = 1.0 / (theta ** (j / R))
    t = torch.arange(T)
    ang = torch.outer(t, freqs)
    cis = torch.polar(torch.ones_like(ang), ang)
    return torch.view_as_real(cis).contiguous()  # [T, 32, 2] fp32


def _draw_indices_uniform(B, lo, hi, k, gen):
    """k distinct positions per row drawn uniformly from [lo[b], hi[b])."""
    out = torch.empty(B, k, dtype=torch.int64)
    for b in range(B):
        n = int(hi[b] - lo[b])
        out[b] = torch.randperm(n, generator=gen)[:k] + int(lo[b])
    return out


def _shuffle_rows(idx, gen):
    """Indexers emit positions in score order, not position order."""
    out = idx.clone()
    for b in range(idx.shape[0]):
        out[b] = idx[b, torch.randperm(idx.shape[1], generator=gen)]
    return out


CONFIG_NAMES = {
    0: "tiny-dense B=1 end_pos=1001 all-selected",
    1: "B=8 end_pos=4096 top-k=2048",
    2: "B=64 end_pos=32768 top-k=2048",
    3: "B=128 end_pos~U[4096,131072] top-k=2048 (50% recent)",
    4: "B=32 cache-write@65535 + top-k=2048 over 65536",
}


# the five headline workloads: batch rows, cache rows per batch row, top-k
CONFIG_SPECS = {
    0: dict(B=1, T=1001, k=1001),
    1: dict(B=8, T=4096, k=2048),
    2: dict(B=64, T=32768, k=2048),
    3: dict(B=128, T=131072, k=2048),
    4: dict(B=32, T=65536, k=2048),
}


def make_config(cid: int, device="cpu", batch: Optional[slice] = None) -> Workload:
    """Build one of the five headline workloads.

    ``batch`` optionally restricts to a slice of the batch (used to shard the
    batch across processes); the draws of the selected rows are identical to
    those of the full workload because every per-row draw is seeded by the
    row's own batch index.
    """
    s = CONFIG_SPECS[cid]
    B, T, k = s["B"], s["T"], s["k"]
    rows = range(B) if batch is None else range(B)[batch]
    return _make_rows(cid, list(rows), B, T, k, device)


def _make_rows(cid, rows, B_full, T, k, device) -> Workload:
    scale = softmax_scale(1.0)
    Bs = len(rows)
    cache = torch.empty(Bs, T, KROW, dtype=torch.bfloat16, device=device)
    q_nope = torch.empty(Bs, H, DN, dtype=torch.bfloat16, device=device)
    q_pe = torch.empty(Bs, H, R, dtype=torch.bfloat16, device=device)
    # weights are shared by the whole batch: one seed
    gw = _gen(1000 + cid, device)
    wkv_b = _normal_bf16((H, DN + DV, C), 1.0 / math.sqrt(C), gw, device)
    rows_per_chunk = max(1, (1 << 22) // KROW)
    for i, b in enumerate(rows):
        g = _gen(1000 + cid * 100003 + 7919 * (b + 1), device)
        for t0 in range(0, T, rows_per_chunk):
            t1 = min(T, t0 + rows_per_chunk)
            cache[i, t0:t1] = _normal_bf16((t1 - t0, KROW), 1.0, g, device)
        q_nope[i] = _normal_bf16((H, DN), 1.0, g, device)
        q_pe[i] = _normal_bf16((H, R), 1.0, g, device)

    gi = torch.Generator()
    gi.manual_seed(2000 + cid)
    # per-row end positions and index sets (drawn for the full batch, then sliced)
    if cid == 0:
        end_pos = torch.full((B_full,), T, dtype=torch.int64)
        idx = torch.arange(T).repeat(B_full, 1)
    elif cid in (1, 2):
        end_pos = torch.full((B_full,), T, dtype=torch.int64)
        idx = _draw_indices_uniform(B_full, [0] * B_full, end_pos, k, gi)
    elif cid == 3:
        end_pos = torch.randint(4096, T + 1, (B_full,), generator=gi)
        recent = _draw_indices_uniform(B_full, end_pos - 4096, end_pos, k // 2, gi)
        older = _draw_indices_uniform(B_full, torch.zeros(B_full, dtype=torch.int64),
                                      end_pos - 4096, k - k // 2, gi)
        idx = torch.cat([recent, older], dim=1)
    elif cid == 4:
        end_pos = torch.full((B_full,), T, dtype=torch.int64)
        wp = T - 1
        older = _draw_indices_uniform(B_full, [0] * B_full, [wp] * B_full, k - 1, gi)
        idx = torch.cat([torch.full((B_full, 1), wp, dtype=torch.int64), older], dim=1)
    else:
        raise ValueError(cid)
    idx = _shuffle_rows(idx, gi)
    rows_t = torch.tensor(rows, dtype=torch.int64)
    topk = idx[rows_t].to(torch.int32).to(device)
    ep = end_pos[rows_t].to(torch.int32).to(device)

    wl = Workload(name=CONFIG_NAMES[cid], B=Bs, T=T, k=k, cache=cache,
                  q_nope=q_nope, q_pe=q_pe, wkv_b=wkv_b, topk=topk,
                  end_pos=ep, scale=scale)
    if cid == 4:
        gx = _gen(3000 + cid, device)
        x_full = _normal_bf16((B_full, DIM), 1.0, gx, device)
        wl.x = x_full[rows_t.to(x_full.device)].contiguous()
        wl.w_kva = _normal_bf16((DIM, KROW), 1.0 / math.sqrt(DIM), gx, device)
        wl.norm_w = torch.ones(C, dtype=torch.bfloat16, device=device)
        wl.rope = rope_table(T).to(device)
        wl.write_pos = T - 1
        wl.eps = 1e-6
    return wl


def make_small(B=3, T=300, k=130, seed=0, device="cpu", end_pos=None,
               n_pad=0, n_invalid=0, q_zero=False, dup=0) -> Workload:
    """Small ragged workload for parity tests: full head/latent dims, small
    B/T/k, per-row end_pos, optional -1 padding, out-of-range entries and
    duplicated indices at the end of each row (the row keeps ``k`` entries)."""
    g = _gen(50_000 + seed, device)
    cache = _normal_bf16((B, T, KROW), 1.0, g, device)
    q_nope = _normal_bf16((B, H, DN), 1.0, g, device)
    q_pe = _normal_bf16((B, H, R), 1.0, g, device)
    if q_zero:
        q_nope.zero_()
        q_pe.zero_()
    wkv_b = _normal_bf16((H, DN + DV, C), 1.0 / math.sqrt(C), g, device)
    gi = torch.Generator()
    gi.manual_seed(60_000 + seed)
    if end_pos is None:
        end_pos = [T - (b * 37) % max(1, T // 3) for b in range(B)]
    end_pos = torch.tensor(end_pos, dtype=torch.int64)
    n_real = k - n_pad - n_invalid - dup
    assert n_real >= 0 and all(int(e) >= n_real for e in end_pos)
    real = _draw_indices_uniform(B, [0] * B, end_pos, n_real, gi)
    parts = [real]
    if dup:
        parts.append(real[:, :dup])
    if n_invalid:
        bad = torch.stack([end_pos + 3 * j + 1 for j in range(n_invalid)], 1)
        bad[:, 0::2] = -7  # negative entries other than -1 are invalid too
        parts.append(bad)
    if n_pad:
        parts.append(torch.full((B, n_pad), -1, dtype=torch.int64))
    idx = torch.cat(parts, 1)
    idx = _shuffle_rows(idx, gi)
    return Workload(name=f"small B={B} T={T} k={k}", B=B, T=T, k=k,
                    cache=cache, q_nope=q_nope, q_pe=q_pe, wkv_b=wkv_b,
                    topk=idx.to(torch.int32).to(device),
                    end_pos=end_pos.to(torch.int32).to(device),
                    scale=softmax_scale(1.0))


def make_cache_write(rows=32, T=64, write_pos=None, seed=0, device="cpu",
                     norm_w_ones=True):
    """Inputs of one cache write: x [rows,7168], W_KVa [7168,576], norm weight,
    rope table [T,32,2]; rows are written at position ``write_pos``."""
    g = _gen(70_000 + seed, device)
    x = _normal_bf16((rows, DIM), 1.0, g, device)
    w_kva = _normal_bf16((DIM, KROW), 1.0 / math.sqrt(DIM), g, device)
    if norm_w_ones:
        norm_w = torch.ones(C, dtype=torch.bfloat16, device=device)
    else:
        norm_w = (1.0 + 0.25 * torch.randn(C, generator=g, device=device)).to(torch.bfloat16)
    if write_pos is None:
        write_pos = T - 1
    return x, w_kva, norm_w, rope_table(T).to(device), write_pos


def make_out_proj(B=8, seed=0, device="cpu", o_std=0.035):
    """Inputs of the output projection: O [B,128,128] with the spread of the
    decode outputs of the workloads (std ~0.035) and W_O [7168, 16384]
    ([out, in]) with variance 1/16384."""
    g = _gen(90_000 + seed, device)
    o = _normal_bf16((B, H, DV), o_std, g, device)
    w_o = _normal_bf16((DIM, H * DV), 1.0 / math.sqrt(H * DV), g, device)
    return o, w_o


def make_query_proj(B=8, T=4096, seed=0, device="cpu"):
    """Inputs of the query path: x [B, 7168] ~ N(0,1), wq_a [1536, 7168] with
    variance 1/7168, q_norm weight 1, wq_b [24576, 1536] with variance 1/1536
    (so qr and q are ~N(0,1)), the rope table [T, 32, 2] and one query
    position per row drawn uniformly from [0, T)."""
    g = _gen(95_000 + seed, device)
    x = _normal_bf16((B, DIM), 1.0, g, device)
    wq_a = _normal_bf16((QL, DIM), 1.0 / math.sqrt(DIM), g, device)
    q_norm_w = torch.ones(QL, dtype=torch.bfloat16, device=device)
    wq_b = _normal_bf16((H * (DN + R), QL), 1.0 / math.sqrt(QL), g, device)
    gi = torch.Generator()
    gi.manual_seed(96_000 + seed)
    pos = torch.randint(0, T, (B,), generator=gi, dtype=torch.int32).to(device)
    return x, wq_a, q_norm_w, wq_b, rope_table(T).to(device), pos


def _causal_topk(limits, k, gen, recent=None):
    """One selection row per query row with causal limit L: min(k, L) distinct
    positions from [0, L), shuffled, padded with -1 to k.  With `recent`
    set and L >= recent + k, half of them come from the last `recent`
    positions and half from the earlier ones (the long-context decode mix)."""
    out = torch.full((len(limits), k), -1, dtype=torch.int64)
    for i, L in enumerate(limits):
        L = int(L)
        if L <= k:
            sel = torch.randperm(L, generator=gen)
        elif recent and L >= recent + k:
            r = torch.randperm(recent, generator=gen)[:k // 2] + (L - recent)
            o = torch.randperm(L - recent, generator=gen)[:k - k // 2]
            sel = torch.cat([r, o])
            sel = sel[torch.randperm(k, generator=gen)]
        else:
            sel = torch.randperm(L, generator=gen)[:k]
        out[i, :len(sel)] = sel
    return out


def make_prefill(B=1, S=256, k=64, seed=0, device="cpu") -> Workload:
    """Sparse prefill of B prompts of S tokens, cached at positions 0 .. S-1:
    query row b * S + s is token s of prompt b, with causal limit s + 1 and
    min(k, s + 1) distinct listed positions from [0, s] (an indexer lists
    only visible positions), padded with -1.  Cache rows, q_nope and q_pe
    ~ N(0,1), wkv_b variance 1/512, as in the decode workloads.  The returned
    workload has B * S query rows and `queries_per_row` = S."""
    g = _gen(70_000 + seed, device)
    cache = _normal_bf16((B, S, KROW), 1.0, g, device)
    q_nope = _normal_bf16((B * S, H, DN), 1.0, g, device)
    q_pe = _normal_bf16((B * S, H, R), 1.0, g, device)
    wkv_b = _normal_bf16((H, DN + DV, C), 1.0 / math.sqrt(C), g, device)
    gi = torch.Generator()
    gi.manual_seed(71_000 + seed)
    limits = [s + 1 for _ in range(B) for s in range(S)]
    topk = _causal_topk(limits, k, gi).to(torch.int32).to(device)
    end_pos = torch.tensor(limits, dtype=torch.int32).to(device)
    wl = Workload(name=f"sparse prefill B={B} S={S} top-k={k}", B=B * S, T=S, k=k, cache=cache,
                  q_nope=q_nope, q_pe=q_pe, wkv_b=wkv_b, topk=topk, end_pos=end_pos,
                  scale=softmax_scale(1.0))
    wl.queries_per_row = S
    return wl


def make_multi_query(B=4, S=2, T=2048, k=256, seed=0, device="cpu", cache=None, end_pos=None,
                     wkv_b=None) -> Workload:
    """Multi-query decode: S new tokens per sequence (speculative or
    multi-token-prediction tokens) whose rows are the last S cached
    positions.  With e_b the sequence's cached length, token s sees
    positions [0, e_b - (S - 1 - s)); its selection follows _causal_topk
    (the recent/older mix when T > 8192).  `cache`, `end_pos` (e_b per
    sequence) and `wkv_b` may be passed in to reuse a decode workload's;
    otherwise they are drawn as in the decode workloads with e_b ~ U[T/2, T].
    The returned workload has B * S query rows and `queries_per_row` = S."""
    g = _gen(72_000 + seed, device)
    if cache is None:
        cache = _normal_bf16((B, T, KROW), 1.0, g, device)
    if wkv_b is None:
        wkv_b = _normal_bf16((H, DN + DV, C), 1.0 / math.sqrt(C), g, device)
    gi = torch.Generator()
    gi.manual_seed(73_000 + seed)
    if end_pos is None:
        e = torch.randint(T // 2, T + 1, (B,), generator=gi)
    else:
        e = end_pos.to("cpu").to(torch.int64)
    q_nope = _normal_bf16((B * S, H, DN), 1.0, g, device)
    q_pe = _normal_bf16((B * S, H, R), 1.0, g, device)
    limits = [int(e[b]) - (S - 1 - s) for b in range(B) for s in range(S)]
    topk = _causal_topk(limits, k, gi, recent=4096 if T > 8192 else None)
    wl = Workload(name=f"multi-query decode B={B} S={S} T={T} top-k={k}", B=B * S, T=T, k=k,
                  cache=cache, q_nope=q_nope, q_pe=q_pe, wkv_b=wkv_b,
                  topk=topk.to(torch.int32).to(device),
                  end_pos=torch.tensor(limits, dtype=torch.int32).to(device),
                  scale=softmax_scale(1.0))
    wl.queries_per_row = S
    return wl


def make_rope_input(B=2, S=5, Hx=128, seed=0, device="cpu"):
    g = _gen(80_000 + seed, device)
    return _normal_bf16((B, S, Hx, R), 1.0, g, device)


# --------------------------------------------------------------------------
# conversions (exact)
# --------------------------------------------------------------------------

def f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (bf16/fp32/int) tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def rope_complex(rope: torch.Tensor) -> np.ndarray:
    """[T,32,2] fp32 (cos, sin) -> complex128 [T,32] with the same fp32 values."""
    r = rope.detach().to("cpu").to(torch.float64).numpy()
    return r[..., 0] + 1j * r[..., 1]


def compact_rows(wl: Workload, b: int):
    """Selected cache rows of batch row ``b`` in topk order, plus the
    re-indexed selection (0..n-1) for a compacted single-row workload.
    Only valid, first-occurrence indices are kept."""
    idx = wl.topk[b].to("cpu").to(torch.int64)
    ep = int(wl.end_pos[b])
    seen, keep = set(), []
    for v in idx.tolist():
        if 0 <= v < ep and v < wl.T and v not in seen:
            seen.add(v)
            keep.append(v)
    sel = torch.tensor(keep, dtype=torch.int64)
    rows = wl.cache[b].index_select(0, sel.to(wl.cache.device))
    return rows, keep
