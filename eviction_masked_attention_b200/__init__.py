"""eviction_masked_attention_b200 -- the KV-streams hot path on NVIDIA B200.

Thin Python binding over the C ABI in ``include/kvs.h`` (``libkvs.so``, built
in-tree by ``eviction_masked_attention_b200.build``). Every function here only
marshals arguments: it checks shapes, allocates outputs and scratch with torch
when the caller gives none, and calls the C entry point of the same name on
torch's current CUDA stream. All arithmetic runs in the library's kernels.

There is no fallback: importing succeeds without the library, but the first
call raises if ``libkvs.so`` is missing or CUDA is unavailable.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvs.so")

KVS_OK, KVS_ERR_INVALID_ARG, KVS_ERR_UNALIGNED, KVS_ERR_EVENT_ORDER = 0, 1, 2, 3
KVS_ERR_CAPACITY, KVS_ERR_UNSUPPORTED, KVS_ERR_TIMEOUT, KVS_ERR_CUDA = 4, 5, 6, 7
KVS_F32, KVS_BF16 = 0, 1
KVS_BWD_PREP, KVS_BWD_DKDV, KVS_BWD_DQ, KVS_BWD_ALL = 1, 2, 4, 7
TILE_EMPTY, TILE_FULL, TILE_PARTIAL = 0, 1, 2
INT32_MAX = 2**31 - 1

EXPORTED = (
    "kvs_build_tile_mask_ws_bytes", "kvs_build_tile_mask", "kvs_compact_block_table",
    "kvs_rope_logical", "kvs_paged_decode_ws_bytes", "kvs_paged_decode_attn",
    "kvs_masked_attn_fwd", "kvs_masked_attn_bwd_ws_bytes", "kvs_masked_attn_bwd",
    "kvs_status_str", "kvs_version", "kvs_last_cuda_error", "kvs_paged_decode_attn_static",
    "kvs_build_tile_mask_async",
)


class KvsError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        extra = f" [{lib().kvs_last_cuda_error().decode()}]" if code == KVS_ERR_CUDA else ""
        super().__init__(f"{where}: {status_str(code)} (status {code}){extra}")


class _TileMaskC(C.Structure):
    _fields_ = [
        ("kappa", C.c_void_p), ("cls", C.c_void_p),
        ("row_ptr", C.c_void_p), ("row_col", C.c_void_p), ("row_pidx", C.c_void_p),
        ("col_ptr", C.c_void_p), ("col_row", C.c_void_p), ("col_pidx", C.c_void_p),
        ("bits", C.c_void_p), ("nnz_cap", C.c_int64), ("partial_cap", C.c_int64),
        ("B", C.c_int32), ("N", C.c_int32), ("T", C.c_int32),
    ]


class _SizesC(C.Structure):
    _fields_ = [("nnz", C.c_int64), ("n_partial", C.c_int64), ("visible_pairs", C.c_int64)]


_lib = None


def lib() -> C.CDLL:
    """Load ``libkvs.so`` (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m eviction_masked_attention_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, i64, f32, f64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_double, C.c_size_t
        L.kvs_build_tile_mask_ws_bytes.argtypes = [i32, i32]
        L.kvs_build_tile_mask_ws_bytes.restype = sz
        L.kvs_build_tile_mask.argtypes = [vp, i32, i32, i32, C.POINTER(_TileMaskC), C.POINTER(_SizesC),
                                          vp, sz, vp]
        L.kvs_build_tile_mask_async.argtypes = [vp, i32, i32, i32, C.POINTER(_TileMaskC), vp, vp, sz, vp, vp]
        L.kvs_compact_block_table.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, vp, vp]
        L.kvs_rope_logical.argtypes = [vp, i64, vp, vp, i32, i32, i32, f64, i32, vp, i32, i32, vp, i64,
                                       vp, i32, vp, vp]
        L.kvs_paged_decode_ws_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
        L.kvs_paged_decode_ws_bytes.restype = sz
        L.kvs_paged_decode_attn.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32,
                                            i32, vp, vp, sz, vp, vp]
        L.kvs_paged_decode_attn_static.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                                   f32, i32, vp, vp, vp]
        L.kvs_masked_attn_fwd.argtypes = [vp, vp, vp, C.POINTER(_TileMaskC), i32, i32, i32, i32, i32,
                                          f32, i32, vp, vp, vp, vp, vp]
        L.kvs_masked_attn_bwd_ws_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
        L.kvs_masked_attn_bwd_ws_bytes.restype = sz
        L.kvs_masked_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, C.POINTER(_TileMaskC), i32, i32,
                                          i32, i32, i32, f32, i32, vp, vp, vp, vp, sz, i32, vp, vp]
        L.kvs_status_str.argtypes = [i32]
        L.kvs_status_str.restype = C.c_char_p
        L.kvs_version.restype = i32
        L.kvs_last_cuda_error.restype = C.c_char_p
        for r in ("kvs_build_tile_mask", "kvs_build_tile_mask_async", "kvs_compact_block_table", "kvs_rope_logical",
                  "kvs_paged_decode_attn", "kvs_paged_decode_attn_static", "kvs_masked_attn_fwd",
                  "kvs_masked_attn_bwd"):
            getattr(L, r).restype = i32
        _lib = L
    return _lib


def status_str(code: int) -> str:
    return lib().kvs_status_str(int(code)).decode()


def _check(code: int, where: str):
    if code != KVS_OK:
        raise KvsError(code, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KVS_BF16
    if t.dtype == torch.float32:
        return KVS_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------------------ mask

@dataclass
class TileMask:
    """Device buffers of a compiled eviction mask (see ``kvs_tile_mask`` in kvs.h)."""

    B: int
    N: int
    T: int
    kappa: torch.Tensor
    cls: torch.Tensor
    row_ptr: torch.Tensor
    row_col: torch.Tensor
    row_pidx: torch.Tensor
    col_ptr: torch.Tensor
    col_row: torch.Tensor
    col_pidx: torch.Tensor
    bits: torch.Tensor
    nnz: int
    n_partial: int
    visible_pairs: int

    def c_struct(self) -> _TileMaskC:
        s = _TileMaskC()
        for f in ("kappa", "cls", "row_ptr", "row_col", "row_pidx", "col_ptr", "col_row", "col_pidx",
                  "bits"):
            setattr(s, f, getattr(self, f).data_ptr())
        s.nnz_cap, s.partial_cap = self.row_col.numel(), self.bits.shape[0]
        s.B, s.N, s.T = self.B, self.N, self.T
        return s


def kvs_build_tile_mask(events: torch.Tensor, B: int, N: int, ws: Optional[torch.Tensor] = None) -> TileMask:
    """Compile an event log (int32 [E, 4] rows (seq, tau, start, end), CUDA, sorted by
    (seq, tau, start)) into the tile mask. Two library calls: count, then fill."""
    if events.numel() == 0:
        events = torch.zeros((0, 4), dtype=torch.int32, device="cuda")
    _dev(events)
    assert events.dtype == torch.int32 and events.shape[-1] == 4
    L, dev = lib(), events.device
    T = (N + 127) // 128
    wsb = L.kvs_build_tile_mask_ws_bytes(B, N)
    if ws is None or ws.numel() < wsb:
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)
    kappa = torch.empty((B, N), **i32)
    cls = torch.empty((B, T, T), dtype=torch.uint8, device=dev)
    row_ptr, col_ptr = torch.empty(B * T + 1, **i32), torch.empty(B * T + 1, **i32)
    m = _TileMaskC()
    m.kappa, m.cls, m.row_ptr, m.col_ptr = kappa.data_ptr(), cls.data_ptr(), row_ptr.data_ptr(), col_ptr.data_ptr()
    m.B, m.N = B, N
    sizes = _SizesC()
    n_ev = events.shape[0]
    evp = _p(events) if n_ev else None
    _check(L.kvs_build_tile_mask(evp, n_ev, B, N, C.byref(m), C.byref(sizes), _p(ws), wsb, _stream()),
           "kvs_build_tile_mask(count)")
    nnz, npart = sizes.nnz, sizes.n_partial
    row_col, row_pidx = torch.empty(max(nnz, 1), **i32), torch.empty(max(nnz, 1), **i32)
    col_row, col_pidx = torch.empty(max(nnz, 1), **i32), torch.empty(max(nnz, 1), **i32)
    bits = torch.empty((max(npart, 1), 128, 4), dtype=torch.int32, device=dev)
    out = TileMask(B, N, T, kappa, cls, row_ptr, row_col, row_pidx, col_ptr, col_row, col_pidx, bits,
                   nnz, npart, sizes.visible_pairs)
    m2 = out.c_struct()
    _check(L.kvs_build_tile_mask(evp, n_ev, B, N, C.byref(m2), C.byref(sizes), _p(ws), wsb, _stream()),
           "kvs_build_tile_mask(fill)")
    return out


def kvs_build_tile_mask_async(events: torch.Tensor, mask: TileMask, ws: Optional[torch.Tensor] = None,
                              sizes: Optional[torch.Tensor] = None,
                              status: Optional[torch.Tensor] = None) -> TileMask:
    """Recompile an event log into the buffers of ``mask`` (same B and N; list
    capacities are the buffers' sizes) with one asynchronous library call: no
    host round trip. ``sizes`` (int64 [3]: nnz, n_partial, visible pairs) and
    ``status`` (int32 [1], first error wins) are device tensors or None; on an
    event-log error or lists over capacity the status is set and the mask reads
    as empty. ``mask.nnz`` etc. keep the values of the build that made it."""
    if events.numel() == 0:
        events = torch.zeros((0, 4), dtype=torch.int32, device=mask.kappa.device)
    _dev(events)
    assert events.dtype == torch.int32 and events.shape[-1] == 4
    L = lib()
    wsb = L.kvs_build_tile_mask_ws_bytes(mask.B, mask.N)
    if ws is None or ws.numel() < wsb:
        ws = torch.empty(wsb, dtype=torch.uint8, device=mask.kappa.device)
    if sizes is not None:
        assert sizes.dtype == torch.int64 and sizes.numel() >= 3
    m = mask.c_struct()
    n_ev = events.shape[0]
    _check(L.kvs_build_tile_mask_async(_p(events) if n_ev else None, n_ev, mask.B, mask.N, C.byref(m),
                                       _p(sizes) if sizes is not None else None, _p(ws), wsb,
                                       _p(status) if status is not None else None, _stream()),
           "kvs_build_tile_mask_async")
    return mask


# ------------------------------------------------------------------------------ compaction

def kvs_compact_block_table(block_table, block_lpos, num_blocks, num_tokens, block_size: int,
                            pool_blocks: int, events, freed=None, n_freed=None, status=None):
    """In-place compaction (all int32 CUDA tensors). Returns (freed, n_freed, status)."""
    _dev(block_table, block_lpos, num_blocks, num_tokens, events)
    B, M = block_table.shape
    if freed is None:
        freed = torch.full((B, M), -1, dtype=torch.int32, device=block_table.device)
    if n_freed is None:
        n_freed = torch.zeros(B, dtype=torch.int32, device=block_table.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=block_table.device)
    n_ev = events.shape[0] if events is not None else 0
    _check(lib().kvs_compact_block_table(_p(block_table), _p(block_lpos), _p(num_blocks), _p(num_tokens),
                                         B, M, block_size, pool_blocks, _p(events) if n_ev else None,
                                         n_ev, _p(freed), _p(n_freed), _p(status), _stream()),
           "kvs_compact_block_table")
    return freed, n_freed, status


# ------------------------------------------------------------------------------ rope

def kvs_rope_logical(x, lpos, theta: float, inverse: bool = False, out=None, out_slot=None,
                     block_size: int = 1, v=None, v_out=None, status=None):
    """Rotate x[n, H, d] (or a row-strided 2-D view [n, stride] holding H*d) at logical
    positions lpos[n]. With out_slot, write rotated rows into the paged cache ``out``
    [pool, H, bs, d] and copy v rows into ``v_out`` at the same slots; the cache's
    first dimension is passed as the pool size the slots are checked against."""
    n = lpos.numel()
    H, d = x.shape[-2], x.shape[-1]
    if x.stride(-1) != 1 or x.stride(-2) != d:
        raise ValueError("heads must be contiguous within a row")
    if out is None:
        if out_slot is not None:
            raise ValueError("out (the cache) is required with out_slot")
        out = torch.empty((n, H, d), dtype=x.dtype, device=x.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=x.device)
    vs = v.stride(0) if v is not None else 0
    pool = out.shape[0] if out_slot is not None else 0
    _check(lib().kvs_rope_logical(_p(x), x.stride(0), _p(out), _p(lpos), n, H, d, float(theta),
                                  int(inverse), _p(out_slot), block_size, pool, _p(v), vs, _p(v_out),
                                  _dtype_code(x), _p(status), _stream()), "kvs_rope_logical")
    return out


# ------------------------------------------------------------------------------ decode

def kvs_paged_decode_attn(q, k_cache, v_cache, block_table, num_tokens, block_size: int, scale: float,
                          out=None, ws=None, status=None):
    """q [B, Hq, d]; caches [pool, Hkv, bs, d]; returns o [B, Hq, d]. Block ids are
    checked against the caches' pool size."""
    _dev(q, k_cache, v_cache, block_table, num_tokens)
    B, Hq, d = q.shape
    Hkv = k_cache.shape[1]
    M = block_table.shape[1]
    L = lib()
    wsb = L.kvs_paged_decode_ws_bytes(B, Hq, Hkv, d, block_size, M)
    if ws is None:
        ws = torch.empty(wsb, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=q.device)
    _check(L.kvs_paged_decode_attn(_p(q), _p(k_cache), _p(v_cache), _p(block_table), _p(num_tokens), B,
                                   Hq, Hkv, d, block_size, M, k_cache.shape[0], float(scale),
                                   _dtype_code(q), _p(out), _p(ws), ws.numel(), _p(status), _stream()),
           "kvs_paged_decode_attn")
    return out


# ------------------------------------------------------------------------------ attention

def kvs_masked_attn_fwd(q, k, v, mask: TileMask, scale: float, out=None, lse=None, status=None,
                        out_lo=None, residual: bool = True):
    """q [B, N, Hq, d], k/v [B, N, Hkv, d] -> (o [B, N, Hq, d], lse fp32 [B, Hq, N], o_lo).
    For bf16 with ``residual`` the rounding residual o_lo of the output is also
    returned (pass it to the backward); otherwise o_lo is None."""
    _dev(q, k, v)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if q.dtype == torch.bfloat16 and residual and out_lo is None:
        out_lo = torch.empty_like(q)
    if q.dtype != torch.bfloat16:
        out_lo = None
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=q.device)
    m = mask.c_struct()
    _check(lib().kvs_masked_attn_fwd(_p(q), _p(k), _p(v), C.byref(m), B, N, Hq, Hkv, d, float(scale),
                                     _dtype_code(q), _p(out), _p(out_lo), _p(lse), _p(status), _stream()),
           "kvs_masked_attn_fwd")
    return out, lse, out_lo


def kvs_masked_attn_bwd(q, k, v, o, do, lse, mask: TileMask, scale: float, dq=None, dk=None, dv=None,
                        ws=None, status=None, stages: int = KVS_BWD_ALL, o_lo=None):
    """Gradients (dq, dk, dv) of kvs_masked_attn_fwd (``stages`` selects the kernels;
    ``o_lo`` is the forward's output residual, improving D = <dO, O>)."""
    _dev(q, k, v, o, do, lse, o_lo)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    L = lib()
    dt = _dtype_code(q)
    wsb = L.kvs_masked_attn_bwd_ws_bytes(B, N, Hq, Hkv, d, dt)
    if ws is None or ws.numel() < wsb:
        ws = torch.empty(wsb, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=q.device)
    m = mask.c_struct()
    _check(L.kvs_masked_attn_bwd(_p(q), _p(k), _p(v), _p(o), _p(o_lo), _p(do), _p(lse), C.byref(m), B, N,
                                 Hq, Hkv, d, float(scale), dt, _p(dq), _p(dk), _p(dv), _p(ws), ws.numel(),
                                 int(stages), _p(status), _stream()), "kvs_masked_attn_bwd")
    return dq, dk, dv
