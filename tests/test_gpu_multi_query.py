"""Several query rows per cache row on the GPU (mla_decode_mq) against the
oracle: sparse prefill ("Mix and project" page, the MHA prefill branch with
the index mask plus the causal mask) and multi-query decode."""
import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle as orc

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS = 2e-2


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _run(wl):
    import sparse_head_latent_absorbed_b200 as shla
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos,
                             wl.scale, wl.queries_per_row, status=status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    return out.float().cpu().numpy().astype(np.float64)


def test_prefill_matches_oracle():
    """Two prompts of 96 tokens, 80 listed positions per token (a full 64-key
    tile and a ragged one of 16; tokens before position 79 list fewer and pad
    with -1).  Early tokens see few keys, so their outputs are of order 1,
    not 0.04: the max-abs bound scales with max|O| as in the decode stress
    case (one bf16 rounding of an order-1 value is ~4e-3)."""
    B, S, k = 2, 96, 80
    wl = mi.make_prefill(B=B, S=S, k=k, seed=1, device="cuda")
    got = _run(wl).reshape(B, S, 128, 128)
    cache = mi.f64(wl.cache)
    want = orc.prefill_materialised(mi.f64(wl.q_nope).reshape(B, S, 128, 128),
                                    mi.f64(wl.q_pe).reshape(B, S, 128, 64), mi.f64(wl.wkv_b),
                                    cache[..., :512], cache[..., 512:],
                                    wl.topk.cpu().numpy().reshape(B, S, k), wl.scale)
    assert np.isfinite(got).all()
    assert _rel(got, want) <= REL_L2
    assert np.abs(got - want).max() <= MAX_ABS * max(1.0, float(np.abs(want).max()))


def test_multi_query_matches_oracle():
    """Three sequences with two new tokens each; token s of sequence b reads
    cache row b with its own selection and causal limit."""
    wl = mi.make_multi_query(B=3, S=2, T=700, k=200, seed=2, device="cuda")
    got = _run(wl)
    cache = mi.f64(wl.cache)
    want = orc.decode_multi_query(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                                  cache[..., :512], cache[..., 512:], wl.topk.cpu().numpy(),
                                  wl.end_pos.cpu().numpy(), wl.scale, 2)
    assert _rel(got, want) <= REL_L2
    assert np.abs(got - want).max() <= MAX_ABS


def test_shared_cache_rows_equal_decode_on_a_repeated_cache():
    """Reading cache row r // S gives bit for bit what mla_decode gives on a
    cache with each row repeated S times (same rows, same schedule)."""
    import sparse_head_latent_absorbed_b200 as shla
    wl = mi.make_multi_query(B=4, S=3, T=500, k=150, seed=3, device="cuda")
    a = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale,
                           3)
    rep = wl.cache.repeat_interleave(3, dim=0).contiguous()
    b = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, rep, wl.topk, wl.end_pos, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_one_query_per_row_is_mla_decode():
    import sparse_head_latent_absorbed_b200 as shla
    wl = mi.make_small(B=3, T=300, k=130, seed=4, device="cuda")
    a = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale,
                           1)
    b = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
