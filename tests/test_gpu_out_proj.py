"""Output projection on the GPU against the oracle ("Mix and project" page:
the output projection wo, Delta = flatten(O) W_O^T)."""
import numpy as np
import pytest
import torch

import mla_inputs as mi
import oracle as orc

pytestmark = pytest.mark.gpu


def _run(B, seed):
    import sparse_head_latent_absorbed_b200 as shla
    o, w_o = mi.make_out_proj(B=B, seed=seed, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    out = shla.mla_out_proj(o, w_o, status=status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    return o, w_o, out


@pytest.mark.parametrize("B", [1, 5, 128, 130])
def test_out_proj_matches_oracle(B):
    """Tolerance of the decode output (rel-L2 <= 1e-2, max-abs <= 2e-2);
    the kernel accumulates in fp32 and rounds once to bf16 (~2e-3 rel-L2).
    B = 130 takes two batch blocks, the second with 2 rows."""
    o, w_o, out = _run(B, seed=B)
    want = orc.out_proj(mi.f64(o), mi.f64(w_o))
    got = mi.f64(out)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel <= 1e-2, rel
    assert np.abs(got - want).max() <= 2e-2


def test_out_proj_one_hot_rows():
    """Exact column selection through the kernel: O with a single 1 at
    (h, d) in row b gives W_O[:, h*128 + d] in row b (bf16 in, one product,
    fp32 sums of zeros: exact) and zeros elsewhere."""
    import sparse_head_latent_absorbed_b200 as shla
    _, w_o = mi.make_out_proj(B=1, seed=7, device="cuda")
    B = 4
    o = torch.zeros(B, 128, 128, dtype=torch.bfloat16, device="cuda")
    picks = [(0, 0, 0), (1, 127, 127), (2, 64, 3), (3, 1, 100)]
    for b, h, d in picks:
        o[b, h, d] = 1.0
    out = shla.mla_out_proj(o, w_o)
    torch.cuda.synchronize()
    for b, h, d in picks:
        assert torch.equal(out[b], w_o[:, h * 128 + d]), (b, h, d)


def test_out_proj_is_deterministic():
    import sparse_head_latent_absorbed_b200 as shla
    o, w_o = mi.make_out_proj(B=64, seed=3, device="cuda")
    a = shla.mla_out_proj(o, w_o)
    b = shla.mla_out_proj(o, w_o)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
