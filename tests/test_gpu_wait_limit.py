"""The expiry path of the bounded waits, on the GPU, without a fault.

Every wait in the library's kernels gives up after 1 s and reports
MLA_STATUS_TIMEOUT in the caller's status word, so that a lost arrival ends
as an error the host reads.  `mla_wait_limit_check` makes two warps wait,
through that code, on an mbarrier that nothing arrives on: both must give
up, the status word must carry the flag, and the context must stay usable
(a decode right after matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle as orc

pytestmark = pytest.mark.gpu

MLA_STATUS_TIMEOUT = 1


def test_wait_gives_up_and_reports():
    import sparse_head_latent_absorbed_b200 as shla
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    shla.mla_wait_limit_check(status, gave_up)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status[0]) & MLA_STATUS_TIMEOUT
    assert int(status[1]) == 0
    assert int(gave_up[0]) == 2
    # the limit is 1 s; the second warp may leave through the first one's abort
    assert 0.9 < dt < 30.0

    # the context is still usable
    wl = mi.make_small(B=3, T=300, k=130, seed=9, device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale,
                          status=st)
    torch.cuda.synchronize()
    assert st.tolist() == [0, 0]
    cache = mi.f64(wl.cache)
    want = orc.decode_absorbed(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                               cache[..., :512], cache[..., 512:], wl.topk.cpu().numpy(),
                               wl.end_pos.cpu().numpy(), wl.scale)
    got = out.double().cpu().numpy()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-2
