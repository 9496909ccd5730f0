"""Work split of the weight-streaming GEMM behind the output projection and
the query path (host logic, no GPU): every (row tile, K chunk) unit belongs to
exactly one CTA, the CTAs' shares differ by at most one unit, and the first
and last CTA of each row tile -- which place each partial in its slot -- match
a brute-force assignment, with the slot count covering every tile."""
import ctypes

import numpy as np
import pytest


@pytest.fixture(scope="module")
def lib():
    from sparse_head_latent_absorbed_b200 import build
    build.build()
    import sparse_head_latent_absorbed_b200._lib as L
    return L.LIB


def _plan(lib, n_out, k_in):
    tiles = n_out // 128
    p = (ctypes.c_int32 * 4)()
    fl = (ctypes.c_int32 * (2 * tiles))()
    assert lib.mla_xwt_plan(n_out, k_in, ctypes.cast(p, ctypes.c_void_p),
                            ctypes.cast(fl, ctypes.c_void_p)) == 0
    return list(p), np.array(fl, dtype=np.int64).reshape(tiles, 2)


SHAPES = [(7168, 16384), (1536, 7168), (24576, 1536)] + [
    (n, k) for n in (128, 256, 384, 1280, 7168) for k in (128, 256, 640, 1536, 9984)]


@pytest.mark.parametrize("n_out,k_in", SHAPES)
def test_units_are_split_once_and_tiles_map_to_slots(lib, n_out, k_in):
    (tot, nc, nch, slots), fl = _plan(lib, n_out, k_in)
    tiles = n_out // 128
    assert nch == k_in // 128 and tot == tiles * nch and nc == min(148, tot)
    owner = np.full(tot, -1)
    sizes = []
    for c in range(nc):
        lo, hi = c * tot // nc, (c + 1) * tot // nc
        assert (owner[lo:hi] == -1).all()
        owner[lo:hi] = c
        sizes.append(hi - lo)
    assert (owner >= 0).all()
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    widest = 0
    for m in range(tiles):
        ctas = sorted(set(owner[m * nch:(m + 1) * nch].tolist()))
        assert ctas == list(range(ctas[0], ctas[-1] + 1))
        assert tuple(fl[m]) == (ctas[0], ctas[-1]), m
        widest = max(widest, len(ctas))
    assert slots == widest


def test_plan_argument_checks(lib):
    p = ctypes.cast((ctypes.c_int32 * 4)(), ctypes.c_void_p)
    assert lib.mla_xwt_plan(7168, 16384, None, None) == -1
    assert lib.mla_xwt_plan(100, 16384, p, None) == -2
    assert lib.mla_xwt_plan(7168, 64, p, None) == -2
    assert lib.mla_xwt_plan(0, 128, p, None) == -2
    assert lib.mla_xwt_plan(7168, 16384, p, None) == 0
