"""Query path on the GPU against the oracle ("Query rotary up-projection"
page: wq_a, q_norm, wq_b viewed head-major, split, RoPE of the rotary part)."""
import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle as orc

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _oracle(x, wa, w, wb, rope, pos):
    R = mi.rope_complex(rope)[pos.cpu().numpy().clip(0, rope.shape[0] - 1)]
    return orc.query_proj(mi.f64(x), mi.f64(wa), mi.f64(w), EPS, mi.f64(wb), R, 128, 128)


def _close(got, want):
    """q ~ N(0,1): fp32 sums of bf16 products, qr and q each rounded once to
    bf16, so |err| <= 2^-7 |q| + 1e-2 element-wise and rel-L2 <= 1e-2."""
    got = mi.f64(got)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel <= 1e-2, rel
    assert (np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 1e-2).all()


@pytest.mark.parametrize("B", [1, 8, 130])
def test_query_proj_matches_oracle(B):
    import sparse_head_latent_absorbed_b200 as shla
    x, wa, w, wb, rope, pos = mi.make_query_proj(B=B, seed=B, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    q_nope, q_pe = shla.mla_query_proj(x, wa, w, EPS, wb, rope, pos, status=status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    want_n, want_p = _oracle(x, wa, w, wb, rope, pos)
    _close(q_nope, want_n)
    _close(q_pe, want_p)


def test_query_proj_invalid_positions_give_zero_rotary_part():
    import sparse_head_latent_absorbed_b200 as shla
    x, wa, w, wb, rope, pos = mi.make_query_proj(B=4, T=64, seed=11, device="cuda")
    pos[1] = -1
    pos[3] = 64
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    q_nope, q_pe = shla.mla_query_proj(x, wa, w, EPS, wb, rope, pos, status=status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 2]
    assert not q_pe[1].any() and not q_pe[3].any()
    want_n, want_p = _oracle(x, wa, w, wb, rope, pos)
    _close(q_nope, want_n)
    _close(q_pe[[0, 2]], want_p[[0, 2]])


def test_query_proj_is_deterministic():
    import sparse_head_latent_absorbed_b200 as shla
    x, wa, w, wb, rope, pos = mi.make_query_proj(B=16, seed=3, device="cuda")
    a = shla.mla_query_proj(x, wa, w, EPS, wb, rope, pos)
    b = shla.mla_query_proj(x, wa, w, EPS, wb, rope, pos)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
