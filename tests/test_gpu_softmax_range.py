"""Softmax arithmetic of the attend kernel at large and peaked scores, through
the C ABI, against the float64 oracle.

The decode softmax of the "Mix and project" page's decode excerpt is invariant
to adding one constant to every score of a head.  These workloads give every
cache row the same value in two rotary columns (one in each half of the
rotary part), so that q_pe in those columns adds one constant per head to all
of its scores: +16, +64, +256 and +2048 log2 units.  The kernel must give the
oracle's result -- which is also the result without the offset -- within the
workload tolerance.  A second family makes one selected key stand 40 log2
units above the rest, at the start, the middle or the end of the row's list,
so that the running maximum jumps by 40 and the accumulator is rescaled by
2^-40 (or never, when the peak comes first).
"""
import math

import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle as orc

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS = 2e-2
LOG2E = 1.0 / math.log(2.0)


@pytest.fixture(scope="module")
def shla():
    import sparse_head_latent_absorbed_b200 as m
    return m


def _oracle(wl):
    cache = mi.f64(wl.cache)
    return orc.decode_absorbed(mi.f64(wl.q_nope), mi.f64(wl.q_pe), mi.f64(wl.wkv_b),
                               cache[..., :512], cache[..., 512:], wl.topk.cpu().numpy(),
                               wl.end_pos.cpu().numpy(), wl.scale)


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _check(out, ref, what):
    g = out.double().cpu().numpy()
    assert np.isfinite(g).all(), what
    rel = _rel(g, ref)
    mx = float(np.abs(g - ref).max())
    # outputs are of order 1 when the softmax is peaked (as in the stress
    # case of the parity tests), so the absolute bound scales with max|O|
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e}"
    assert mx <= MAX_ABS * max(1.0, float(np.abs(ref).max())), f"{what}: max-abs {mx:.3e}"


def _workload(seed, B=3, T=3000, k=2048):
    return mi.make_small(B=B, T=T, k=k, seed=seed, device="cuda")


@pytest.mark.parametrize("offset", [16.0, 64.0, 256.0, 2048.0])
def test_common_offset_on_every_score(shla, offset):
    wl = _workload(seed=100 + int(offset))
    base = wl.q_pe.clone()
    base[:, :, 0] = 0
    base[:, :, 32] = 0
    # the same rotary value in column 0 and 32 of every cache row
    wl.cache[:, :, 512] = 1.0
    wl.cache[:, :, 512 + 32] = 1.0
    # q_pe in those columns: half of the offset each (in log2 units of the
    # scaled score), rounded to bf16 -- whatever the rounding, it is one
    # constant per head
    a = offset / (2.0 * wl.scale * LOG2E)
    wl.q_pe.copy_(base)
    wl.q_pe[:, :, 0] = a
    wl.q_pe[:, :, 32] = a
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos,
                          wl.scale, status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    ref = _oracle(wl)
    _check(out, ref, f"offset {offset}")
    # shift invariance: the same output as without the offset
    wl.q_pe.copy_(base)
    ref0 = _oracle(wl)
    assert _rel(ref, ref0) < 1e-9
    _check(out, ref0, f"offset {offset} vs no offset")


@pytest.mark.parametrize("where", ["first", "middle", "last"])
def test_one_key_far_above_the_rest(shla, where):
    wl = _workload(seed=200 + len(where))
    B, k = wl.B, wl.k
    wl.cache[:, :, 512 + 1] = 0.0
    topk = wl.topk.cpu()
    ep = wl.end_pos.cpu()
    for b in range(B):
        valid = [j for j in range(k) if 0 <= int(topk[b, j]) < int(ep[b])]
        j = {"first": valid[0], "middle": valid[len(valid) // 2], "last": valid[-1]}[where]
        wl.cache[b, int(topk[b, j]), 512 + 1] = 1.0
    wl.q_pe[:, :, 1] = 40.0 / (wl.scale * LOG2E)
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos,
                          wl.scale, status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    _check(out, _oracle(wl), f"peak {where}")


def test_offset_and_peak_together(shla):
    """A +256 offset on every score plus one key 40 units above the rest."""
    wl = _workload(seed=300)
    wl.cache[:, :, 512] = 1.0
    wl.cache[:, :, 512 + 32] = 1.0
    wl.cache[:, :, 512 + 1] = 0.0
    topk = wl.topk.cpu()
    for b in range(wl.B):
        wl.cache[b, int(topk[b, 700]), 512 + 1] = 1.0
    a = 256.0 / (2.0 * wl.scale * LOG2E)
    wl.q_pe[:, :, 0] = a
    wl.q_pe[:, :, 32] = a
    wl.q_pe[:, :, 1] = 40.0 / (wl.scale * LOG2E)
    out = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale)
    _check(out, _oracle(wl), "offset 256 + peak")


def test_negative_offset(shla):
    """Scores far below zero (-2048 log2 units): nothing underflows to an
    all-zero row, because the maximum is subtracted before the exponential."""
    wl = _workload(seed=400)
    wl.cache[:, :, 512] = 1.0
    wl.cache[:, :, 512 + 32] = 1.0
    a = -2048.0 / (2.0 * wl.scale * LOG2E)
    wl.q_pe[:, :, 0] = a
    wl.q_pe[:, :, 32] = a
    out = shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale)
    _check(out, _oracle(wl), "offset -2048")
