"""CPU oracle for the KV-streams hot path -- TEST INFRASTRUCTURE ONLY.

A plain, slow fp64 implementation (``oracle.c``, built with gcc) of what the
library computes: compaction-event log -> kill times, the 128x128 tile mask,
block-table compaction, rotary embedding at logical positions, paged decode,
the eviction-masked attention forward and backward, and a toy multi-layer
model that literally simulates generation with physical eviction (and the
re-prefill alternative). It shares no code with the CUDA library and must only
be used by the tests, the package smoke check and the benchmark's CPU-baseline
leg; the library's product path never imports it.

All functions take and return numpy arrays; the C side does the arithmetic.
Parity pins for every function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

EMPTY, FULL, PARTIAL = 0, 1, 2
INT32_MAX = 2**31 - 1


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                               "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _L():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = C.CDLL(_LIB)
            _lib.orc_visible_pairs.restype = C.c_int64
            _lib.orc_tile_lists.restype = C.c_int
            _lib.orc_compact.restype = C.c_int
            _lib.orc_toy_generate.restype = C.c_int
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _events(ev):
    ev = _i32(ev).reshape(-1, 4)
    return ev, C.c_int64(ev.shape[0])


# ------------------------------------------------------------------ events, masks

def kappa(events, B: int, N: int) -> np.ndarray:
    """int32 [B, N]: the first event time that removes each logical position."""
    ev, n = _events(events)
    out = np.empty((B, N), dtype=np.int32)
    _L().orc_kappa(_p(ev), n, C.c_int32(B), C.c_int32(N), _p(out))
    return out


def visible_pairs(kap: np.ndarray) -> int:
    """Number of visible (query, key) pairs: sum_j (min(kappa_j, N) - j)."""
    kap = _i32(kap)
    B, N = kap.shape
    return int(_L().orc_visible_pairs(_p(kap), C.c_int32(B), C.c_int32(N)))


def tile_mask(kap: np.ndarray) -> dict:
    """Brute-force tile classes, row/col CSR lists and partial-tile bits."""
    kap = _i32(kap)
    B, N = kap.shape
    T = (N + 127) // 128
    L = _L()
    cls = np.empty((B, T, T), dtype=np.uint8)
    L.orc_tile_classes(_p(kap), C.c_int32(B), C.c_int32(N), _p(cls))
    nnz, npart = C.c_int64(), C.c_int64()
    rp = np.empty(B * T + 1, dtype=np.int32)
    cp = np.empty(B * T + 1, dtype=np.int32)
    L.orc_tile_lists(_p(kap), _p(cls), C.c_int32(B), C.c_int32(N), _p(rp), None, None, _p(cp),
                     None, None, None, C.c_int64(0), C.c_int64(0), C.byref(nnz), C.byref(npart))
    rc_, rpx = np.empty(nnz.value, np.int32), np.empty(nnz.value, np.int32)
    cr_, cpx = np.empty(nnz.value, np.int32), np.empty(nnz.value, np.int32)
    bits = np.empty((npart.value, 128, 4), dtype=np.uint32)
    rc = L.orc_tile_lists(_p(kap), _p(cls), C.c_int32(B), C.c_int32(N), _p(rp), _p(rc_), _p(rpx),
                          _p(cp), _p(cr_), _p(cpx), _p(bits), C.c_int64(nnz.value),
                          C.c_int64(npart.value), C.byref(nnz), C.byref(npart))
    assert rc == 0
    return dict(cls=cls, row_ptr=rp, row_col=rc_, row_pidx=rpx, col_ptr=cp, col_row=cr_,
                col_pidx=cpx, bits=bits, nnz=nnz.value, n_partial=npart.value, T=T)


def tile_bits(kap: np.ndarray, b: int, qi: int, kj: int) -> np.ndarray:
    kap = _i32(kap)
    out = np.empty((128, 4), dtype=np.uint32)
    _L().orc_tile_bits(_p(kap), C.c_int32(kap.shape[1]), C.c_int32(b), C.c_int32(qi),
                       C.c_int32(kj), _p(out))
    return out


# ------------------------------------------------------------------ rotary

def rope(x, lpos, theta: float, inverse: bool = False) -> np.ndarray:
    """fp64 rotate-half rotary embedding of x[n, H, d] at logical positions lpos[n]."""
    x = _f64(x)
    n, H, d = x.shape
    lp = _i32(lpos)
    y = np.empty_like(x)
    _L().orc_rope(_p(x), _p(y), _p(lp), C.c_int64(n), C.c_int32(H), C.c_int32(d),
                  C.c_double(theta), C.c_int32(int(inverse)))
    return y


# ------------------------------------------------------------------ attention

def attn_rows(qrows, trows, k, v, kap_b, scale: float):
    """Masked attention for given query rows of one (sequence, kv head).
    qrows [n, d], trows [n] logical positions, k/v [N, d], kap_b [N]."""
    qrows, k, v = _f64(qrows), _f64(k), _f64(v)
    tr, kb = _i32(trows), _i32(kap_b)
    n, d = qrows.shape
    o = np.empty((n, d)), np.empty(n)
    _L().orc_attn_rows(_p(qrows), _p(tr), C.c_int64(n), _p(k), _p(v), _p(kb),
                       C.c_int32(k.shape[0]), C.c_int32(d), C.c_double(scale), _p(o[0]), _p(o[1]))
    return o


def attn_fwd(q, k, v, kap, scale: float):
    """Full masked forward: q [B,N,Hq,d], k/v [B,N,Hkv,d] -> o [B,N,Hq,d], lse [B,Hq,N]."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    o = np.empty((B, N, Hq, d))
    lse = np.empty((B, Hq, N))
    t = np.arange(N, dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            oo, ll = attn_rows(q[b, :, h], t, k[b, :, h // G], v[b, :, h // G], kap[b], scale)
            o[b, :, h] = oo
            lse[b, h] = ll
    return o, lse


def attn_bwd(q, k, v, do, kap, scale: float):
    """Full masked backward; returns o, lse, dq, dk, dv (fp64)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    o = np.empty((B, N, Hq, d)); lse = np.empty((B, Hq, N))
    dq = np.empty((B, N, Hq, d)); dk = np.empty((B, N, Hkv, d)); dv = np.empty((B, N, Hkv, d))
    L = _L()
    for b in range(B):
        kb = _i32(kap[b])
        for kvh in range(Hkv):
            hs = slice(kvh * G, (kvh + 1) * G)
            qg = _f64(np.transpose(q[b, :, hs], (1, 0, 2)))
            dog = _f64(np.transpose(do[b, :, hs], (1, 0, 2)))
            kk, vv = _f64(k[b, :, kvh]), _f64(v[b, :, kvh])
            og, lg = np.empty((G, N, d)), np.empty((G, N))
            dqg, dkk, dvv = np.empty((G, N, d)), np.empty((N, d)), np.empty((N, d))
            L.orc_attn_bwd_group(_p(qg), _p(kk), _p(vv), _p(dog), _p(kb), C.c_int32(N), C.c_int32(G),
                                 C.c_int32(d), C.c_double(scale), _p(og), _p(lg), _p(dqg), _p(dkk),
                                 _p(dvv))
            o[b, :, hs] = np.transpose(og, (1, 0, 2)); lse[b, hs] = lg
            dq[b, :, hs] = np.transpose(dqg, (1, 0, 2)); dk[b, :, kvh] = dkk; dv[b, :, kvh] = dvv
    return o, lse, dq, dk, dv


def dq_rows(qg, k, v, dog, kap_b, scale: float, grow, trow):
    """dQ for rows (g, t) of one group. qg/dog [G,N,d], k/v [N,d]."""
    qg, dog, k, v = _f64(qg), _f64(dog), _f64(k), _f64(v)
    gr, tr, kb = _i32(grow), _i32(trow), _i32(kap_b)
    G, N, d = qg.shape
    out = np.empty((len(tr), d))
    _L().orc_attn_dq_rows(_p(qg), _p(k), _p(v), _p(dog), _p(kb), C.c_int32(N), C.c_int32(d),
                          C.c_double(scale), _p(gr), _p(tr), C.c_int64(len(tr)), _p(out))
    return out


def dkdv_cols(qg, k, v, dog, kap_b, scale: float, cols):
    """dK, dV for key positions ``cols`` of one group. qg/dog [G,N,d], k/v [N,d]."""
    qg, dog, k, v = _f64(qg), _f64(dog), _f64(k), _f64(v)
    cs, kb = _i32(cols), _i32(kap_b)
    G, N, d = qg.shape
    dk, dv = np.empty((len(cs), d)), np.empty((len(cs), d))
    _L().orc_attn_dkdv_cols(_p(qg), _p(k), _p(v), _p(dog), _p(kb), C.c_int32(N), C.c_int32(G),
                            C.c_int32(d), C.c_double(scale), _p(cs), C.c_int64(len(cs)), _p(dk),
                            _p(dv))
    return dk, dv


def dkdv_cols_fwd(qg, k, v, dog, og, lseg, kap_b, scale: float, cols):
    """dK, dV for key positions ``cols`` of one group from the forward's per-row
    O and LSE (qg/dog/og [G,N,d], lseg [G,N], k/v [N,d]). Rows with dO = 0 add
    nothing; their og/lseg may be 0/+inf."""
    qg, dog, og, lseg, k, v = _f64(qg), _f64(dog), _f64(og), _f64(lseg), _f64(k), _f64(v)
    cs, kb = _i32(cols), _i32(kap_b)
    G, N, d = qg.shape
    dk, dv = np.empty((len(cs), d)), np.empty((len(cs), d))
    _L().orc_attn_dkdv_cols_fwd(_p(qg), _p(k), _p(v), _p(dog), _p(og), _p(lseg), _p(kb),
                                C.c_int32(N), C.c_int32(G), C.c_int32(d), C.c_double(scale),
                                _p(cs), C.c_int64(len(cs)), _p(dk), _p(dv))
    return dk, dv


# ------------------------------------------------------------------ paged cache

def compact(block_table, block_lpos, num_blocks, num_tokens, block_size: int, events):
    """List-filter compaction; returns (rc, table, lpos, nblk, ntok, freed[B,max_blocks], n_freed)."""
    bt, bl = _i32(block_table).copy(), _i32(block_lpos).copy()
    nb, nt = _i32(num_blocks).copy(), _i32(num_tokens).copy()
    B, M = bt.shape
    ev, n = _events(events)
    freed = np.full((B, M), -1, dtype=np.int32)
    nf = np.zeros(B, dtype=np.int32)
    rc = _L().orc_compact(_p(bt), _p(bl), _p(nb), _p(nt), C.c_int32(B), C.c_int32(M),
                          C.c_int32(block_size), _p(ev), n, _p(freed), _p(nf))
    return rc, bt, bl, nb, nt, freed, nf


def paged_decode(q, k_cache, v_cache, block_table, num_tokens, block_size: int, scale: float):
    """q [B,Hq,d]; caches [pool,Hkv,bs,d]; returns o [B,Hq,d] (fp64)."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    bt, nt = _i32(block_table), _i32(num_tokens)
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    o = np.empty((B, Hq, d))
    _L().orc_paged_decode(_p(q), _p(kc), _p(vc), _p(bt), _p(nt), C.c_int32(B), C.c_int32(Hq),
                          C.c_int32(Hkv), C.c_int32(d), C.c_int32(block_size),
                          C.c_int32(bt.shape[1]), C.c_double(scale), _p(o))
    return o


# ------------------------------------------------------------------ toy model

def toy_project(x, W) -> np.ndarray:
    """The toy model's projection, row by row: y[n] = x[n] W (x [n, Din], W [Din, Dout])."""
    x, W = _f64(x), _f64(W)
    n, Din = x.shape
    Dout = W.shape[1]
    y = np.empty((n, Dout))
    _L().orc_toy_project(_p(x), _p(W), C.c_int64(n), C.c_int32(Din), C.c_int32(Dout), _p(y))
    return y


def toy_rotate(x, lpos, theta: float) -> np.ndarray:
    """The toy model's rotation of x [n, H, d] at positions lpos[n] (returns a copy)."""
    y = _f64(x).copy()
    n, H, d = y.shape
    assert d % 2 == 0 and d <= 512
    _L().orc_toy_rotate(_p(y), _p(_i32(lpos)), C.c_int64(n), C.c_int32(H), C.c_int32(d),
                        C.c_double(theta))
    return y


class Toy:
    """Random-weight L-layer attention stack used to check that the replay
    reproduces generation with physical eviction at every layer."""

    def __init__(self, L, Dm, Hq, Hkv, d, theta, seed):
        assert d % 2 == 0 and d <= 512 and Hq % Hkv == 0
        rng = np.random.default_rng(seed)
        self.L, self.Dm, self.Hq, self.Hkv, self.d, self.theta = L, Dm, Hq, Hkv, d, theta
        self.scale = 1.0 / np.sqrt(d)
        s = 1.0 / np.sqrt(Dm)
        self.Wq = rng.standard_normal((L, Dm, Hq * d)) * s
        self.Wk = rng.standard_normal((L, Dm, Hkv * d)) * s
        self.Wv = rng.standard_normal((L, Dm, Hkv * d)) * s
        self.Wo = rng.standard_normal((L, Hq * d, Dm)) / np.sqrt(Hq * d)

    def _w(self):
        return (C.c_int32(self.L), C.c_int32(self.Dm), C.c_int32(self.Hq), C.c_int32(self.Hkv),
                C.c_int32(self.d), _p(self.Wq), _p(self.Wk), _p(self.Wv), _p(self.Wo),
                C.c_double(self.theta), C.c_double(self.scale))

    def generate(self, x0, events3, block_size: int, pool: int, reprefill: bool = False):
        """events3: int32 [E, 3] of (tau, start, end), sorted by tau."""
        x0 = _f64(x0)
        N = x0.shape[0]
        ev = _i32(events3).reshape(-1, 3)
        xo = np.empty_like(x0)
        attn = np.empty((N, self.L, self.Hq * self.d))
        tab, lp = np.empty(pool, np.int32), np.empty(pool, np.int32)
        nb, nt = C.c_int32(), C.c_int32()
        rc = _L().orc_toy_generate(*self._w(), _p(x0), C.c_int32(N), _p(ev), C.c_int64(ev.shape[0]),
                                   C.c_int32(block_size), C.c_int32(pool), C.c_int32(int(reprefill)),
                                   _p(xo), _p(attn), _p(tab), _p(lp), C.byref(nb), C.byref(nt))
        return rc, xo, attn, tab[: nb.value].copy(), lp[: nb.value].copy(), nt.value

    def replay(self, x0, kap_b):
        x0 = _f64(x0)
        N = x0.shape[0]
        xo = np.empty_like(x0)
        attn = np.empty((N, self.L, self.Hq * self.d))
        _L().orc_toy_replay(*self._w(), _p(x0), C.c_int32(N), _p(_i32(kap_b)), _p(xo), _p(attn))
        return xo, attn
