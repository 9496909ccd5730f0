"""The full decode call launches the attend, merge and W_UV kernels with
programmatic dependent launch (each may start while the previous one
drains); launching the three phases one by one keeps plain stream order.
Both orders must give the same bits."""
import pytest
import torch

import mla_inputs as mi

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,k", [(8, 2500, 2048), (1000, 200, 64), (130, 900, 300)])
def test_full_call_equals_phases_launched_one_by_one(B, T, k):
    import sparse_head_latent_absorbed_b200 as shla
    wl = mi.make_small(B=B, T=T, k=k, seed=B, device="cuda")
    ws = torch.empty(shla.mla_decode_workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    full = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos,
                           wl.scale, ws=ws, status=status)
    ws2 = torch.empty_like(ws)
    split = torch.empty_like(full)
    for phase in (1, 2, 3):
        shla.mla_decode_phase(phase, wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk,
                              wl.end_pos, wl.scale, split, ws2, status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    assert torch.equal(full, split)


def test_both_merge_paths_are_covered():
    """The cases above include rows split across clusters (merge kernel runs)
    and rows held whole by one cluster (the attend kernel writes them)."""
    import sparse_head_latent_absorbed_b200 as shla
    assert shla.mla_decode_num_splits(8, 2048) > 1
    assert shla.mla_decode_num_splits(1000, 64) == 1
