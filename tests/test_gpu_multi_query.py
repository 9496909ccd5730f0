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


def test_shared_cache_rows_equal_one_query_per_row_on_a_repeated_cache():
    """Reading cache row r // S gives bit for bit what one query per row
    gives on a cache with each row repeated S times (same rows, same lists,
    so the same schedule)."""
    import sparse_head_latent_absorbed_b200 as shla
    wl = mi.make_multi_query(B=4, S=3, T=500, k=150, seed=3, device="cuda")
    a = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale,
                           3)
    rep = wl.cache.repeat_interleave(3, dim=0).contiguous()
    b = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, rep, wl.topk, wl.end_pos, wl.scale, 1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_one_query_per_row_matches_mla_decode():
    """One query per row is mla_decode's operation; the two may cut the rows
    at different tiles (mla_decode_mq balances a per-row cost as well), so
    they agree within the workload tolerance, and each with the oracle."""
    import sparse_head_latent_absorbed_b200 as shla
    wl = mi.make_small(B=3, T=300, k=130, seed=4, device="cuda")
    a = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale,
                           1)
    b = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale)
    torch.cuda.synchronize()
    a64 = a.double().cpu().numpy()
    b64 = b.double().cpu().numpy()
    cache = mi.f64(wl.cache)
    want = orc.decode_absorbed(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                               cache[..., :512], cache[..., 512:], wl.topk.cpu().numpy(),
                               wl.end_pos.cpu().numpy(), wl.scale)
    assert _rel(a64, b64) <= REL_L2
    assert _rel(a64, want) <= REL_L2
    assert np.abs(a64 - want).max() <= MAX_ABS


def test_prefill_1024_token_prompt_sampled_tokens():
    """One prompt of 1024 tokens, top-k 256 (four 64-key tiles per token).
    Tokens before position 255 list fewer positions and pad with -1; the
    tiles that hold only padding are not scheduled, so the rows have 1 to 4
    tiles and the cluster ranges cut them unevenly.  The whole prompt runs on
    the GPU; 40 tokens (the tile edges, both ends and a seeded draw) are
    checked against the oracle's absorbed decode at their causal limits
    (pinned equal to the prefill branch on the CPU)."""
    S, k = 1024, 256
    wl = mi.make_prefill(B=1, S=S, k=k, seed=5, device="cuda")
    got = _run(wl)
    rng = np.random.default_rng(11)
    fixed = [0, 1, 2, 62, 63, 64, 65, 127, 128, 191, 192, 254, 255, 256, 257, 511, 512, 1022, 1023]
    rows = sorted(set(fixed) | set(rng.choice(S, 40 - len(fixed), replace=False).tolist()))
    sel = torch.tensor(rows, device="cuda")
    cache = mi.f64(wl.cache)
    c = np.broadcast_to(cache, (len(rows),) + cache.shape[1:])
    want = orc.decode_absorbed(mi.f64(wl.q_nope[sel]), mi.f64(wl.q_pe[sel]), mi.f64(wl.wkv_b),
                               c[..., :512], c[..., 512:], wl.topk[sel].cpu().numpy(),
                               wl.end_pos[sel].cpu().numpy(), wl.scale)
    g = got[rows]
    assert np.isfinite(got).all()
    assert _rel(g, want) <= REL_L2
    assert np.abs(g - want).max() <= MAX_ABS * max(1.0, float(np.abs(want).max()))


def test_trailing_padding_tiles_are_skipped():
    """Four query rows with room for 640 entries (10 tiles each) but at most
    40 listed: each row needs one tile, so the 4 tiles in all fall to 4 of
    the clusters and the others get an empty range; one row lists nothing.
    The result is bit for bit mla_decode on the same lists cut to 40 entries
    (one tile per row, each row held whole by one cluster in both), which
    also shows that the padding tiles were not run: a padding tile changes
    no value, but a row cut in two would be merged in another order."""
    import sparse_head_latent_absorbed_b200 as shla
    wl = mi.make_small(B=4, T=300, k=40, seed=6, device="cuda")
    wl.topk[2] = -1
    padded = torch.full((4, 640), -1, dtype=torch.int32, device="cuda")
    padded[:, :40] = wl.topk
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    a = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, padded, wl.end_pos, wl.scale,
                           1, status=status)
    b = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    assert torch.equal(a, b)
    assert float(a[2].abs().max()) == 0.0
    cache = mi.f64(wl.cache)
    want = orc.decode_absorbed(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                               cache[..., :512], cache[..., 512:], padded.cpu().numpy(),
                               wl.end_pos.cpu().numpy(), wl.scale)
    assert _rel(a.double().cpu().numpy(), want) <= REL_L2


def test_ragged_rows_split_across_clusters():
    """Multi-query rows whose lists end in padding of different lengths, with
    enough tiles in all that rows are split across clusters at uneven
    points: every split row is merged from the right clusters' slots."""
    wl = mi.make_multi_query(B=24, S=2, T=3000, k=1024, seed=7, device="cuda")
    # cut each row's list to a different length (padding at the end)
    g = torch.Generator().manual_seed(8)
    keep = torch.randint(1, 1025, (wl.B,), generator=g)
    keep[::5] = 1024
    for r in range(wl.B):
        wl.topk[r, int(keep[r]):] = -1
    got = _run(wl)
    cache = mi.f64(wl.cache)
    want = orc.decode_multi_query(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                                  cache[..., :512], cache[..., 512:], wl.topk.cpu().numpy(),
                                  wl.end_pos.cpu().numpy(), wl.scale, 2)
    assert _rel(got, want) <= REL_L2
    assert np.abs(got - want).max() <= MAX_ABS * max(1.0, float(np.abs(want).max()))


def test_ragged_row_split_across_many_clusters():
    """Two query rows of 32 tiles each: with so few tiles the ranges are one
    tile or none, so each row is merged from about 30 clusters' segments
    (the merge's general path), with trailing padding on one row."""
    wl = mi.make_multi_query(B=2, S=1, T=3000, k=2048, seed=9, device="cuda")
    wl.topk[1, 1500:] = -1
    got = _run(wl)
    cache = mi.f64(wl.cache)
    want = orc.decode_multi_query(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                                  cache[..., :512], cache[..., 512:], wl.topk.cpu().numpy(),
                                  wl.end_pos.cpu().numpy(), wl.scale, 1)
    assert _rel(got, want) <= REL_L2
    assert np.abs(got - want).max() <= MAX_ABS * max(1.0, float(np.abs(want).max()))


@pytest.mark.parametrize("case", range(6))
def test_ragged_seeded_sweep(case):
    """Seeded random shapes for the ragged schedule: sequences, new tokens
    per sequence (1, 2 or 4), list length, trailing padding per row (from
    none to all of it), and a few invalid entries; each checked against the
    oracle, with the invalid entries counted in status[1]."""
    import sparse_head_latent_absorbed_b200 as shla
    rng = np.random.default_rng(1000 + case)
    S = int(rng.choice([1, 2, 4]))
    B = int(rng.integers(1, 12))
    k = int(rng.choice([40, 64, 130, 700, 1500]))
    T = int(rng.integers(k + 10, 3 * k + 100))
    wl = mi.make_multi_query(B=B, S=S, T=T, k=k, seed=500 + case, device="cuda")
    topk = wl.topk.cpu()
    ep = wl.end_pos.cpu()
    n_bad = 0
    for r in range(wl.B):
        keep = int(rng.integers(0, k + 1))
        topk[r, keep:] = -1
        if keep > 2 and rng.random() < 0.5:
            topk[r, 1] = int(ep[r]) + 5  # out of range: masked and counted
            n_bad += 1
    wl.topk.copy_(topk)
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = shla.mla_decode_mq(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos,
                             wl.scale, S, status=status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, n_bad]
    got = out.double().cpu().numpy()
    cache = mi.f64(wl.cache)
    want = orc.decode_multi_query(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                                  cache[..., :512], cache[..., 512:], topk.numpy(),
                                  ep.numpy(), wl.scale, S)
    assert np.isfinite(got).all()
    if np.linalg.norm(want) > 0:
        assert _rel(got, want) <= REL_L2
    assert np.abs(got - want).max() <= MAX_ABS * max(1.0, float(np.abs(want).max()))
