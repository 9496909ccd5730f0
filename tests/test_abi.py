"""The C-ABI library loads and exports every entry point its header declares;
host-side argument checks return their error codes before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "shla.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from sparse_head_latent_absorbed_b200 import build
    build.build()
    import sparse_head_latent_absorbed_b200._lib as L
    return L.LIB


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("mla_rope", "mla_cache_write", "mla_decode", "mla_decode_mq",
                 "mla_decode_workspace_bytes",
                 "mla_index_mask", "mla_gather_rows", "mla_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(0, -7, -1):
        s = lib.mla_status_string(code).decode()
        assert s and s != "unknown status code"
    assert lib.mla_status_string(-99).decode() == "unknown status code"


def test_null_and_shape_checks_before_any_cuda_call(lib):
    from sparse_head_latent_absorbed_b200 import _lib as L
    vp = ctypes.c_void_p
    dummy = vp(4096)
    # NULL pointers
    assert lib.mla_rope(None, dummy, 1, 1, 1, 1, dummy, None) == -1
    assert lib.mla_decode(None, dummy, dummy, dummy, 0, 576, dummy, 0, 576, 10, dummy, 4,
                          dummy, 1, 1.0, dummy, dummy, 1 << 20, None, None) == -1
    assert lib.mla_index_mask(None, 1, 1, dummy, 1, dummy, None, None) == -1
    # shapes
    assert lib.mla_rope(dummy, dummy, 0, 1, 1, 1, dummy, None) == -2
    assert lib.mla_decode(dummy, dummy, dummy, dummy, 0, 576, dummy, 0, 576, 10, dummy, 0,
                          dummy, 1, 1.0, dummy, dummy, 1 << 20, None, None) == -2
    assert lib.mla_decode(dummy, dummy, dummy, dummy, 0, 500, dummy, 0, 576, 10, dummy, 4,
                          dummy, 1, 1.0, dummy, dummy, 1 << 20, None, None) == -2
    assert lib.mla_cache_write(dummy, dummy, dummy, 1e-6, dummy, 1, 1, 10, dummy, 0, 576,
                               dummy, 0, 576, 10, dummy, 1 << 24, None) == -2
    # alignment
    odd = vp(4096 + 2)
    assert lib.mla_rope(odd, dummy, 1, 1, 1, 1, dummy, None) == -3
    assert lib.mla_decode(dummy, dummy, dummy, odd, 0, 576, dummy, 0, 576, 10, dummy, 4,
                          dummy, 1, 1.0, dummy, dummy, 1 << 20, None, None) == -3
    # workspace
    assert lib.mla_decode(dummy, dummy, dummy, dummy, 0, 576, dummy, 0, 576, 10, dummy, 4,
                          dummy, 1, 1.0, dummy, None, 0, None, None) == -4
    assert lib.mla_cache_write(dummy, dummy, dummy, 1e-6, dummy, 1, 1, 0, dummy, 0, 576,
                               dummy, 0, 576, 10, None, 0, None) == -4
    assert L.mla_cache_write_workspace_bytes(32) == 28 * 32 * 576 * 4
    # output projection
    assert lib.mla_out_proj(None, dummy, 1, dummy, dummy, 1 << 30, None, None) == -1
    assert lib.mla_out_proj(dummy, dummy, 0, dummy, dummy, 1 << 30, None, None) == -2
    assert lib.mla_out_proj(dummy, odd, 1, dummy, dummy, 1 << 30, None, None) == -3
    assert lib.mla_out_proj(dummy, dummy, 4, dummy, dummy, 16, None, None) == -4
    assert lib.mla_out_proj(dummy, dummy, 4, dummy, vp(4096 + 16), 1 << 30, None, None) == -4
    assert L.mla_out_proj_workspace_bytes(0) == 0
    # query path
    args = lambda **kw: [kw.get(n, dummy) for n in ("x", "wa", "w")] + [kw.get("eps", 1e-6)] + \
        [kw.get(n, dummy) for n in ("wb", "rope")] + [kw.get("T", 16), kw.get("pos", dummy),
                                                      kw.get("B", 2), dummy, dummy,
                                                      kw.get("ws", dummy), kw.get("wsb", 1 << 30),
                                                      None, None]  # noqa: E731
    assert lib.mla_query_proj(*args(x=None)) == -1
    assert lib.mla_query_proj(*args(pos=None)) == -1
    assert lib.mla_query_proj(*args(B=0)) == -2
    assert lib.mla_query_proj(*args(T=0)) == -2
    assert lib.mla_query_proj(*args(eps=-1.0)) == -2
    assert lib.mla_query_proj(*args(wb=odd)) == -3
    assert lib.mla_query_proj(*args(wsb=64)) == -4
    assert L.mla_query_proj_workspace_bytes(0) == 0
    assert L.mla_query_proj_workspace_bytes(8) >= 8 * 1536 * 2
    assert L.mla_out_proj_workspace_bytes(128) >= 56 * 4 * 128 * 128 * 4
    # several query rows per cache row: queries_per_row must divide B, and the
    # cache rows in use must be addressable with 32-bit row indices
    mq = lambda B, q, bstride=0: lib.mla_decode_mq(  # noqa: E731
        dummy, dummy, dummy, dummy, bstride, 576, dummy, bstride, 576, 10, dummy, 4, dummy, B, q,
        1.0, dummy, dummy, 1 << 30, None, None)
    assert mq(4, 0) == -2
    assert mq(3, 2) == -2
    assert mq(2, 1, 576 << 31) == -2


def test_workspace_and_split_choice(lib):
    from sparse_head_latent_absorbed_b200 import _lib as L
    for B, k in ((1, 1001), (8, 2048), (64, 2048), (128, 2048), (32, 2048), (3, 130)):
        s = L.mla_decode_num_splits(B, k)
        assert 1 <= s <= min(32, k)
        ws = L.mla_decode_workspace_bytes(B, k)
        # q~ and the merged O~ per row, plus a partial-output slot (O~ and its
        # log-sum-exps) in each of the s clusters that meet one row
        assert ws >= 2 * B * 128 * 512 * 2 + s * 128 * (512 * 2 + 4)
