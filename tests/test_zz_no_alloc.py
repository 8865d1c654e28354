"""The allocation-free paged decode (kvs_paged_decode_attn_static).

It serves callers that cannot allocate device memory on their decode path
(CUDA-graph replay of generation steps, engines whose own pool owns all device
memory, embedders that only hold input/output pointers). It must give the same
result as the regular entry point, call after call, and refuse requests larger
than its fixed scratch. This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import workloads as W
from gpu_util import BF16_TOL, assert_close, dev, host

pytestmark = pytest.mark.gpu
STATIC_MAX = 16 << 20


def _lib():
    L = kvs.lib()
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    L.kvs_paged_decode_attn_static.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                               ctypes.c_float, i32, vp, vp, vp]
    L.kvs_paged_decode_attn_static.restype = i32
    return L


def _static_call(q, kc, vc, bt, nt, bs, scale, out, status):
    L = _lib()
    B, Hq, d = q.shape
    return L.kvs_paged_decode_attn_static(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), bt.data_ptr(), nt.data_ptr(), B, Hq, kc.shape[1], d,
        bs, bt.shape[1], kc.shape[0], float(scale), kvs.KVS_BF16, out.data_ptr(), status.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("bs", [16, 1])
def test_static_decode_matches_regular_entry_point(bs):
    rng = np.random.default_rng(7 + bs)
    B, Hq, Hkv, d = 6, 32, 8, 128
    M = 2048 // bs
    pool = B * M + 3
    kc = dev(W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32)), torch.bfloat16)
    vc = dev(W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32)), torch.bfloat16)
    bt = dev(rng.permutation(pool)[: B * M].reshape(B, M).astype(np.int32))
    assert kvs.lib().kvs_paged_decode_ws_bytes(B, Hq, Hkv, d, bs, M) <= STATIC_MAX
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):  # two calls in a row share (and reuse) the fixed scratch
        nt = dev(rng.integers(0, M * bs + 1, B).astype(np.int32))
        q = dev(W.round_bf16(rng.standard_normal((B, Hq, d)).astype(np.float32)), torch.bfloat16)
        want = kvs.kvs_paged_decode_attn(q, kc, vc, bt, nt, bs, 1 / np.sqrt(d))
        got = torch.full_like(q, float("nan"))
        rc = _static_call(q, kc, vc, bt, nt, bs, 1 / np.sqrt(d), got, status)
        torch.cuda.synchronize()
        assert rc == kvs.KVS_OK, kvs.status_str(rc)
        assert status.item() == 0
        assert_close(host(got), host(want), BF16_TOL, f"static decode call {call}")


def test_static_decode_rejects_oversized_requests():
    B, Hq, Hkv, d, bs, M = 4096, 64, 8, 128, 16, 64
    assert kvs.lib().kvs_paged_decode_ws_bytes(B, Hq, Hkv, d, bs, M) > STATIC_MAX
    t = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = _lib().kvs_paged_decode_attn_static(t.data_ptr(), t.data_ptr(), t.data_ptr(), i.data_ptr(),
                                            i.data_ptr(), B, Hq, Hkv, d, bs, M, 1, 0.1, kvs.KVS_BF16,
                                            t.data_ptr(), i.data_ptr(), None)
    assert rc == kvs.KVS_ERR_CAPACITY
