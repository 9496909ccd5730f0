"""ctypes binding of libshla.so.

Argument marshalling only: tensors are passed as raw device pointers plus
sizes and strides, with the current torch CUDA stream.  Every step of the
decode path runs in the library's CUDA kernels; if the library cannot be
loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libshla.so")

_c_int, _c_float, _c_i64, _c_size, _vp = (ctypes.c_int, ctypes.c_float, ctypes.c_int64,
                                          ctypes.c_size_t, ctypes.c_void_p)

_SIGS = {
    "mla_status_string": (ctypes.c_char_p, [_c_int]),
    "mla_rope": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp]),
    "mla_cache_write_workspace_bytes": (_c_size, [_c_int]),
    "mla_cache_write": (_c_int, [_vp, _vp, _vp, _c_float, _vp, _c_int, _c_int, _c_int,
                                 _vp, _c_i64, _c_int, _vp, _c_i64, _c_int, _c_int,
                                 _vp, _c_size, _vp]),
    "mla_cache_write_noalloc": (_c_int, [_vp, _vp, _vp, _c_float, _vp, _c_int, _c_int, _c_int,
                                         _vp, _c_i64, _c_int, _vp, _c_i64, _c_int, _c_int, _vp]),
    "mla_decode_workspace_bytes": (_c_size, [_c_int, _c_int]),
    "mla_decode_num_splits": (_c_int, [_c_int, _c_int]),
    "mla_wait_limit_check": (_c_int, [_vp, _vp, _vp]),
    "mla_decode": (_c_int, [_vp, _vp, _vp, _vp, _c_i64, _c_int, _vp, _c_i64, _c_int, _c_int,
                            _vp, _c_int, _vp, _c_int, _c_float, _vp, _vp, _c_size, _vp, _vp]),
    "mla_decode_mq": (_c_int, [_vp, _vp, _vp, _vp, _c_i64, _c_int, _vp, _c_i64, _c_int, _c_int,
                               _vp, _c_int, _vp, _c_int, _c_int, _c_float, _vp, _vp, _c_size,
                               _vp, _vp]),
    "mla_decode_phase": (_c_int, [_c_int, _vp, _vp, _vp, _vp, _c_i64, _c_int, _vp, _c_i64,
                                  _c_int, _c_int, _vp, _c_int, _vp, _c_int, _c_float, _vp, _vp,
                                  _c_size, _vp, _vp]),
    "mla_fold_wuk": (_c_int, [_vp, _vp, _c_int, _vp, _vp]),
    "mla_out_proj_workspace_bytes": (_c_size, [_c_int]),
    "mla_out_proj": (_c_int, [_vp, _vp, _c_int, _vp, _vp, _c_size, _vp, _vp]),
    "mla_query_proj_workspace_bytes": (_c_size, [_c_int]),
    "mla_query_proj": (_c_int, [_vp, _vp, _vp, _c_float, _vp, _vp, _c_int, _vp, _c_int, _vp,
                                _vp, _vp, _c_size, _vp, _vp]),
    "mla_xwt_plan": (_c_int, [_c_int, _c_int, _vp, _vp]),
    "mla_index_mask": (_c_int, [_vp, _c_int, _c_int, _vp, _c_int, _vp, _vp, _vp]),
    "mla_gather_rows": (_c_int, [_vp, _c_i64, _c_int, _vp, _c_i64, _c_int, _c_int, _vp,
                                 _c_int, _c_int, _vp, _vp, _vp, _vp]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libshla.so is not built ({LIB_PATH}); run "
                          "`python -m sparse_head_latent_absorbed_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


class MLAError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise MLAError(f"{what}: {LIB.mla_status_string(rc).decode()} (code {rc})")


def status_string(code: int) -> str:
    return LIB.mla_status_string(code).decode()


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise MLAError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise MLAError(f"{name} must be {dtype}, got {t.dtype}")


def _split_cache(cache: torch.Tensor):
    """Fused cache [B, T, 576] -> (c_kv ptr tensor, k_pe view, strides)."""
    if cache.dim() != 3 or cache.shape[-1] != 576 or cache.stride(-1) != 1:
        raise MLAError("cache must be [B, T, 576] with unit inner stride")
    _need(cache, torch.bfloat16, "cache")
    return (cache, cache.stride(0), cache.stride(1),
            cache[..., 512:], cache.stride(0), cache.stride(1))


# ---------------------------------------------------------------------------
# public calls (same names as the C ABI)
# ---------------------------------------------------------------------------

def mla_rope(x: torch.Tensor, rope: torch.Tensor, interleaved: bool = True,
             out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x bf16 [B, S, Hx, 64], rope fp32 [S, 32, 2] -> rotated bf16 (``out`` may be x)."""
    _need(x, torch.bfloat16, "x")
    _need(rope, torch.float32, "rope")
    if x.dim() != 4 or x.shape[-1] != 64 or not x.is_contiguous():
        raise MLAError("x must be contiguous [B, S, Hx, 64]")
    B, S, Hx, _ = x.shape
    if tuple(rope.shape) != (S, 32, 2) or not rope.is_contiguous():
        raise MLAError("rope must be contiguous [S, 32, 2]")
    y = torch.empty_like(x) if out is None else out
    _check(LIB.mla_rope(_p(x), _p(rope), B, S, Hx, int(bool(interleaved)), _p(y),
                        _stream(x.device)), "mla_rope")
    return y


def mla_cache_write_workspace_bytes(rows: int) -> int:
    return int(LIB.mla_cache_write_workspace_bytes(rows))


def mla_cache_write(x: torch.Tensor, w_kva: torch.Tensor, norm_w: torch.Tensor, eps: float,
                    rope: torch.Tensor, start_pos: int, cache: torch.Tensor,
                    ws: Optional[torch.Tensor] = None) -> None:
    """x bf16 [B, S, 7168] (or [B, 7168] for S = 1); writes rows
    [start_pos, start_pos + S) of the fused cache [B, T, 576]."""
    _need(x, torch.bfloat16, "x")
    if x.dim() == 2:
        x = x.unsqueeze(1)
    B, S, _ = x.shape
    c_kv, cbs, crs, k_pe, kbs, krs = _split_cache(cache)
    rows = B * S
    need = mla_cache_write_workspace_bytes(rows)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(LIB.mla_cache_write(_p(x.contiguous()), _p(w_kva), _p(norm_w), float(eps), _p(rope),
                               B, S, int(start_pos), _p(c_kv), cbs, crs, _p(k_pe), kbs, krs,
                               cache.shape[1], _p(ws), ws.numel(), _stream(x.device)),
           "mla_cache_write")


def mla_out_proj_workspace_bytes(B: int) -> int:
    return int(LIB.mla_out_proj_workspace_bytes(int(B)))


def mla_out_proj(O: torch.Tensor, w_o: torch.Tensor, out: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None,
                 status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Delta = flatten(O) W_O^T: O bf16 [B, 128, 128], w_o bf16 [7168, 16384]
    ([out, in]) -> bf16 [B, 7168]."""
    _need(O, torch.bfloat16, "O")
    _need(w_o, torch.bfloat16, "w_o")
    B = O.shape[0]
    if out is None:
        out = torch.empty(B, w_o.shape[0], dtype=torch.bfloat16, device=O.device)
    need = mla_out_proj_workspace_bytes(B)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=O.device)
    _check(LIB.mla_out_proj(_p(O.contiguous()), _p(w_o.contiguous()), B, _p(out), _p(ws),
                            ws.numel(), _p(status) if status is not None else None,
                            _stream(O.device)),
           "mla_out_proj")
    return out


def mla_query_proj_workspace_bytes(B: int) -> int:
    return int(LIB.mla_query_proj_workspace_bytes(int(B)))


def mla_query_proj(x: torch.Tensor, wq_a: torch.Tensor, q_norm_w: torch.Tensor, eps: float,
                   wq_b: torch.Tensor, rope: torch.Tensor, pos: torch.Tensor,
                   ws: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None):
    """x bf16 [B, 7168] -> (q_nope bf16 [B, 128, 128], q_pe bf16 [B, 128, 64])
    with the rotation at pos (int32 [B]) from the fp32 table rope [T, 32, 2]."""
    _need(x, torch.bfloat16, "x")
    _need(pos, torch.int32, "pos")
    _need(rope, torch.float32, "rope")
    B = x.shape[0]
    q_nope = torch.empty(B, 128, 128, dtype=torch.bfloat16, device=x.device)
    q_pe = torch.empty(B, 128, 64, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = torch.empty(mla_query_proj_workspace_bytes(B), dtype=torch.uint8, device=x.device)
    _check(LIB.mla_query_proj(_p(x.contiguous()), _p(wq_a.contiguous()), _p(q_norm_w),
                              float(eps), _p(wq_b.contiguous()), _p(rope.contiguous()),
                              rope.shape[0], _p(pos.contiguous()), B, _p(q_nope), _p(q_pe),
                              _p(ws), ws.numel(), _p(status) if status is not None else None,
                              _stream(x.device)),
           "mla_query_proj")
    return q_nope, q_pe


NOALLOC_MAX_ROWS = 64


def mla_cache_write_noalloc(x: torch.Tensor, w_kva: torch.Tensor, norm_w: torch.Tensor,
                            eps: float, rope: torch.Tensor, start_pos: int,
                            cache: torch.Tensor) -> None:
    """mla_cache_write without a workspace: for callers that cannot allocate
    device memory at call time.  Uses the library's fixed scratch array
    (at most NOALLOC_MAX_ROWS = B*S rows); calls that overlap on the GPU race
    on that array."""
    _need(x, torch.bfloat16, "x")
    if x.dim() == 2:
        x = x.unsqueeze(1)
    B, S, _ = x.shape
    c_kv, cbs, crs, k_pe, kbs, krs = _split_cache(cache)
    _check(LIB.mla_cache_write_noalloc(_p(x.contiguous()), _p(w_kva), _p(norm_w), float(eps),
                                       _p(rope), B, S, int(start_pos), _p(c_kv), cbs, crs,
                                       _p(k_pe), kbs, krs, cache.shape[1], _stream(x.device)),
           "mla_cache_write_noalloc")


def mla_decode_workspace_bytes(B: int, k: int) -> int:
    return int(LIB.mla_decode_workspace_bytes(B, k))


def mla_decode_num_splits(B: int, k: int) -> int:
    return int(LIB.mla_decode_num_splits(B, k))


def mla_decode(q_nope: torch.Tensor, q_pe: torch.Tensor, wkv_b: torch.Tensor,
               cache: torch.Tensor, topk: torch.Tensor, end_pos: torch.Tensor, scale: float,
               out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
               status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Absorbed sparse decode.  q_nope [B,128,128], q_pe [B,128,64], wkv_b
    [128,256,512] (bf16), cache [B,T,576] bf16, topk int32 [B,k], end_pos
    int32 [B] -> O bf16 [B,128,128]."""
    for t, n in ((q_nope, "q_nope"), (q_pe, "q_pe"), (wkv_b, "wkv_b")):
        _need(t, torch.bfloat16, n)
        if not t.is_contiguous():
            raise MLAError(f"{n} must be contiguous")
    _need(topk, torch.int32, "topk")
    _need(end_pos, torch.int32, "end_pos")
    B = q_nope.shape[0]
    k = topk.shape[1]
    c_kv, cbs, crs, k_pe, kbs, krs = _split_cache(cache)
    if out is None:
        out = torch.empty(B, 128, 128, dtype=torch.bfloat16, device=q_nope.device)
    if ws is None:
        ws = torch.empty(mla_decode_workspace_bytes(B, k), dtype=torch.uint8,
                         device=q_nope.device)
    _check(LIB.mla_decode(_p(q_nope), _p(q_pe), _p(wkv_b), _p(c_kv), cbs, crs, _p(k_pe), kbs,
                          krs, cache.shape[1], _p(topk.contiguous()), k, _p(end_pos), B,
                          float(scale), _p(out), _p(ws), ws.numel(), _p(status),
                          _stream(q_nope.device)), "mla_decode")
    return out


def mla_decode_mq(q_nope: torch.Tensor, q_pe: torch.Tensor, wkv_b: torch.Tensor,
                  cache: torch.Tensor, topk: torch.Tensor, end_pos: torch.Tensor, scale: float,
                  queries_per_row: int, out: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None,
                  status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Sparse decode of several query rows per cache row (multi-query decode,
    sparse prefill).  q_nope [B,128,128], q_pe [B,128,64], topk int32 [B,k],
    end_pos int32 [B] for B query rows; cache [B / queries_per_row, T, 576];
    query row r reads cache row r // queries_per_row -> O bf16 [B,128,128]."""
    for t, n in ((q_nope, "q_nope"), (q_pe, "q_pe"), (wkv_b, "wkv_b")):
        _need(t, torch.bfloat16, n)
        if not t.is_contiguous():
            raise MLAError(f"{n} must be contiguous")
    _need(topk, torch.int32, "topk")
    _need(end_pos, torch.int32, "end_pos")
    B = q_nope.shape[0]
    k = topk.shape[1]
    if queries_per_row < 1 or B % queries_per_row or cache.shape[0] != B // queries_per_row:
        raise MLAError("cache must hold B / queries_per_row batch rows")
    c_kv, cbs, crs, k_pe, kbs, krs = _split_cache(cache)
    if out is None:
        out = torch.empty(B, 128, 128, dtype=torch.bfloat16, device=q_nope.device)
    if ws is None:
        ws = torch.empty(mla_decode_workspace_bytes(B, k), dtype=torch.uint8,
                         device=q_nope.device)
    _check(LIB.mla_decode_mq(_p(q_nope), _p(q_pe), _p(wkv_b), _p(c_kv), cbs, crs, _p(k_pe), kbs,
                             krs, cache.shape[1], _p(topk.contiguous()), k, _p(end_pos), B,
                             int(queries_per_row), float(scale), _p(out), _p(ws), ws.numel(),
                             _p(status), _stream(q_nope.device)), "mla_decode_mq")
    return out


def mla_decode_phase(phase: int, q_nope, q_pe, wkv_b, cache, topk, end_pos, scale, out, ws,
                     status=None) -> None:
    """One of the three launches of mla_decode (1 fold, 2 attend, 3 merge+W_UV)."""
    c_kv, cbs, crs, k_pe, kbs, krs = _split_cache(cache)
    _check(LIB.mla_decode_phase(int(phase), _p(q_nope), _p(q_pe), _p(wkv_b), _p(c_kv), cbs, crs,
                                _p(k_pe), kbs, krs, cache.shape[1], _p(topk), topk.shape[1],
                                _p(end_pos), q_nope.shape[0], float(scale), _p(out), _p(ws),
                                ws.numel(), _p(status), _stream(q_nope.device)),
           "mla_decode_phase")


def mla_fold_wuk(q_nope: torch.Tensor, wkv_b: torch.Tensor,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(q_nope, torch.bfloat16, "q_nope")
    _need(wkv_b, torch.bfloat16, "wkv_b")
    B = q_nope.shape[0]
    if out is None:
        out = torch.empty(B, 128, 512, dtype=torch.bfloat16, device=q_nope.device)
    _check(LIB.mla_fold_wuk(_p(q_nope), _p(wkv_b), B, _p(out), _stream(q_nope.device)),
           "mla_fold_wuk")
    return out


def mla_wait_limit_check(status: torch.Tensor, gave_up: torch.Tensor) -> None:
    """Launches the bounded-wait expiry check (see include/shla.h)."""
    _need(status, torch.int32, "status")
    _need(gave_up, torch.int32, "gave_up")
    _check(LIB.mla_wait_limit_check(_p(status), _p(gave_up), _stream(status.device)),
           "mla_wait_limit_check")


def mla_index_mask(topk: torch.Tensor, end_pos: torch.Tensor, T: int,
                   status: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(topk, torch.int32, "topk")
    _need(end_pos, torch.int32, "end_pos")
    B, k = topk.shape
    mask = torch.empty(B, T, dtype=torch.uint8, device=topk.device)
    _check(LIB.mla_index_mask(_p(topk.contiguous()), B, k, _p(end_pos), T, _p(mask),
                              _p(status), _stream(topk.device)), "mla_index_mask")
    return mask


def mla_gather_rows(cache: torch.Tensor, topk: torch.Tensor, end_pos: torch.Tensor,
                    status: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(topk, torch.int32, "topk")
    c_kv, cbs, crs, k_pe, kbs, krs = _split_cache(cache)
    B, k = topk.shape
    rows = torch.empty(B, k, 576, dtype=torch.bfloat16, device=cache.device)
    _check(LIB.mla_gather_rows(_p(c_kv), cbs, crs, _p(k_pe), kbs, krs, cache.shape[1],
                               _p(topk.contiguous()), B, k, _p(end_pos), _p(rows), _p(status),
                               _stream(cache.device)), "mla_gather_rows")
    return rows
