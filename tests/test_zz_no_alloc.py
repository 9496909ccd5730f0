"""The allocation-free cache write (fixed library-owned scratch instead of a
caller workspace) gives the same rows as the ordinary cache write.

It exists for callers that cannot allocate device memory when they call the
library (allocation-free decode loops, callbacks inside other runtimes,
device memory owned by a foreign allocator).  This file is collected last so
that a failure here does not hide the results of the other tests; it must
pass both on its own in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_inputs as mi

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p


def _ptr(t):
    return _vp(t.data_ptr())


def _call_noalloc(L, x, w, nw, tab, start, cache):
    B, S, _ = x.shape
    return L.mla_cache_write_noalloc(_ptr(x), _ptr(w), _ptr(nw), 1e-6, _ptr(tab), B, S, start,
                                     _ptr(cache), cache.stride(0), cache.stride(1),
                                     _vp(cache.data_ptr() + 1024), cache.stride(0),
                                     cache.stride(1), cache.shape[1],
                                     _vp(torch.cuda.current_stream().cuda_stream))


def _call_ws(L, x, w, nw, tab, start, cache):
    B, S, _ = x.shape
    ws = torch.empty(L.mla_cache_write_workspace_bytes(B * S), dtype=torch.uint8, device="cuda")
    rc = L.mla_cache_write(_ptr(x), _ptr(w), _ptr(nw), 1e-6, _ptr(tab), B, S, start,
                           _ptr(cache), cache.stride(0), cache.stride(1),
                           _vp(cache.data_ptr() + 1024), cache.stride(0), cache.stride(1),
                           cache.shape[1], _ptr(ws), ws.numel(),
                           _vp(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc


def test_noalloc_cache_write_matches_workspace_version_twice():
    from sparse_head_latent_absorbed_b200 import _lib
    L = _lib.LIB
    T, start = 48, 31
    # two calls in a row with different sizes and inputs: the second must not
    # see anything the first left in the shared scratch array
    for rows, S, seed in ((64, 1, 1), (5, 3, 2)):
        B = rows // S if rows % S == 0 else rows
        x, w, nw, tab, _ = mi.make_cache_write(rows=B * S, T=T, seed=seed, device="cuda",
                                               norm_w_ones=(seed == 1))
        x = x.view(B, S, -1).contiguous()
        tab_s = tab[start:start + S].contiguous()
        ref = torch.full((B, T, 576), 5.0, dtype=torch.bfloat16, device="cuda")
        got = ref.clone()
        assert _call_ws(L, x, w, nw, tab_s, start, ref) == 0
        assert _call_noalloc(L, x, w, nw, tab_s, start, got) == 0
        torch.cuda.synchronize()
        a = ref.double().cpu().numpy()
        b = got.double().cpu().numpy()
        # the cache-write tolerance of the parity tests: one bf16 rounding
        assert np.all(np.abs(b - a) <= np.abs(a) * 2.0 ** -7 + 1e-4)
        assert torch.equal(got, ref)  # same kernels, same order: identical bits
        assert torch.all(got[:, :start] == 5.0) and torch.all(got[:, start + S:] == 5.0)


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    from sparse_head_latent_absorbed_b200 import _lib
    L = _lib.LIB
    x, w, nw, tab, _ = mi.make_cache_write(rows=65, T=8, device="cuda")
    cache = torch.zeros(65, 8, 576, dtype=torch.bfloat16, device="cuda")
    rc = _call_noalloc(L, x.view(65, 1, -1), w, nw, tab[3:4].contiguous(), 3, cache)
    assert rc == -2  # MLA_ERR_SHAPE: more than MLA_NOALLOC_MAX_ROWS rows
    torch.cuda.synchronize()
    assert torch.all(cache == 0)
