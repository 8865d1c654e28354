"""The C-ABI library builds, loads without a GPU, and exports every entry point
that include/kvs.h declares (no compute calls here)."""
import ctypes
import os
import re

import pytest

import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvs.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvs_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def built():
    kbuild.build()
    return ctypes.CDLL(kbuild.LIB)


def test_header_and_library_agree(built):
    decl = _declared()
    assert len(decl) >= 11
    for name in decl:
        assert hasattr(built, name), name
    assert sorted(kvs.EXPORTED) == decl


def test_host_only_calls(built):
    assert kvs.lib().kvs_version() == 100
    assert kvs.status_str(kvs.KVS_ERR_UNALIGNED) == "eviction range covers part of a block"
    # workspace queries are pure host arithmetic
    assert kvs.lib().kvs_build_tile_mask_ws_bytes(2, 131072) > 2 * 1024 * 1024 * 4
    assert kvs.lib().kvs_paged_decode_ws_bytes(64, 32, 8, 128, 16, 2049) > 0
    assert kvs.lib().kvs_masked_attn_bwd_ws_bytes(2, 300, 4, 1, 128, kvs.KVS_BF16) == 2 * 2 * 4 * 384 * 4


def test_host_side_argument_errors(built):
    L = kvs.lib()
    # invalid sizes / NULL pointers are rejected before any launch
    assert L.kvs_compact_block_table(None, None, None, None, 1, 0, 16, 1, None, 0, None, None, None,
                                     None) == kvs.KVS_ERR_INVALID_ARG
    assert L.kvs_rope_logical(None, 0, None, None, 1, 1, 96, 1e4, 0, None, 1, 1, None, 0, None,
                              kvs.KVS_F32, None, None) in (kvs.KVS_ERR_INVALID_ARG, kvs.KVS_ERR_UNSUPPORTED)
    assert L.kvs_paged_decode_attn(None, None, None, None, None, 1, 3, 2, 128, 16, 4, 8, 1.0, kvs.KVS_BF16,
                                   None, None, 0, None, None) == kvs.KVS_ERR_INVALID_ARG
    # the pool size must be positive, and max_blocks * block_size must fit in int32 (the
    # kernels index live entries with int32)
    assert L.kvs_paged_decode_attn(None, None, None, None, None, 1, 8, 1, 128, 16, 4, 0, 1.0, kvs.KVS_BF16,
                                   None, None, 0, None, None) == kvs.KVS_ERR_INVALID_ARG
    assert L.kvs_paged_decode_attn(None, None, None, None, None, 1, 8, 1, 128, 16, 2**27, 8, 1.0,
                                   kvs.KVS_BF16, None, None, 0, None, None) == kvs.KVS_ERR_CAPACITY
    # the asynchronous mask build checks its arguments on the host and launches nothing
    # when they are bad: no mask struct, a B/N mismatch, or list buffers missing
    assert L.kvs_build_tile_mask_async(None, 0, 1, 100, None, None, None, 0, None,
                                       None) == kvs.KVS_ERR_INVALID_ARG
    mm = kvs._TileMaskC()
    mm.B, mm.N = 2, 100
    assert L.kvs_build_tile_mask_async(None, 0, 1, 100, ctypes.byref(mm), None, None, 0, None,
                                       None) == kvs.KVS_ERR_INVALID_ARG
    mm.B = 1
    assert L.kvs_build_tile_mask_async(None, 0, 1, 100, ctypes.byref(mm), None, None, 0, None,
                                       None) == kvs.KVS_ERR_INVALID_ARG
    m = kvs._TileMaskC()
    m.B, m.N, m.T = 1, 100, 1
    assert L.kvs_masked_attn_fwd(None, None, None, ctypes.byref(m), 1, 100, 4, 1, 96, 1.0, kvs.KVS_BF16,
                                 None, None, None, None, None) == kvs.KVS_ERR_INVALID_ARG


def test_product_path_has_no_oracle_import():
    # the library package never imports the CPU oracle
    pkg = os.path.join(ROOT, "eviction_masked_attention_b200")
    for dp, _, fs in os.walk(pkg):
        for f in fs:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dp, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "oracle.c" not in txt, f


def _plan_ws(B, Hq, Hkv, d, bs, max_blocks):
    """The work split as documented at kvs_paged_decode_ws_bytes: C = min(444, chunks of
    the full table) CTAs; scratch = 8 (B + 1) bytes of prefix counts (rounded up to 256)
    + (C + B Hkv) G (d + 2) fp32 partials."""
    tc = B * Hkv * -(-(max_blocks * bs) // 16)
    c = max(1, min(444, tc))
    G = Hq // Hkv
    return -(-(8 * (B + 1)) // 256) * 256 + (c + B * Hkv) * G * (d + 2) * 4


@pytest.mark.parametrize("shape", [(64, 32, 8, 128, 16, 2049),   # paged workload
                                   (2, 64, 8, 128, 1, 28701),    # two long sequences, 1-token blocks
                                   (3, 8, 2, 128, 16, 100),      # few units: short splits
                                   (1, 8, 1, 128, 16, 4)])       # one split: no partials
def test_decode_plan_workspace(built, shape):
    assert kvs.lib().kvs_paged_decode_ws_bytes(*shape) == _plan_ws(*shape)
