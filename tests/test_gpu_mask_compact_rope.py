"""GPU parity: tile-mask compiler, block-table compaction and logical RoPE
against the CPU oracle (bit-exact for integers, tolerance for floats)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import workloads as W
from gpu_util import compare_mask, dev, events_dev, host

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ mask

@pytest.mark.parametrize("cid,div", [(1, 1), (2, 8), (3, 16), (5, 32), (5, 16)])
def test_mask_configs_scaled(cid, div):
    cfg = W.scaled(W.CONFIGS[cid], div)
    ev = W.make_event_log(cfg)
    gm = kvs.kvs_build_tile_mask(events_dev(ev), cfg.batch, cfg.n_tokens)
    compare_mask(gm, ev, cfg.batch, cfg.n_tokens)


@pytest.mark.parametrize("cid", [2, 3, 5])
def test_mask_configs_full_size(cid):
    cfg = W.CONFIGS[cid]
    ev = W.make_event_log(cfg)
    gm = kvs.kvs_build_tile_mask(events_dev(ev), cfg.batch, cfg.n_tokens)
    compare_mask(gm, ev, cfg.batch, cfg.n_tokens)


@pytest.mark.parametrize("N,seed", [(128, 0), (300, 1), (1000, 2), (1, 3), (129, 4), (4096, 5)])
def test_mask_edge_cases(N, seed):
    rng = np.random.default_rng(seed)
    ev = W.random_event_log(rng, 3, N, 12, unit=1, max_span=max(1, N // 4))
    gm = kvs.kvs_build_tile_mask(events_dev(ev), 3, N)
    compare_mask(gm, ev, 3, N)


def test_mask_empty_log_and_tile_edges():
    gm = kvs.kvs_build_tile_mask(events_dev(np.zeros((0, 4))), 2, 640)
    compare_mask(gm, np.zeros((0, 4)), 2, 640)
    # ranges and times exactly on tile boundaries
    ev = np.array([[0, 256, 0, 128], [0, 384, 128, 256], [1, 512, 256, 384], [1, 512, 384, 512]])
    gm = kvs.kvs_build_tile_mask(events_dev(ev), 2, 640)
    compare_mask(gm, ev, 2, 640)
    g = json.load(open(os.path.join(GOLD, "mask_small.json")))
    gm = kvs.kvs_build_tile_mask(events_dev(g["events"]), 1, 512)
    assert gm.cls.cpu().numpy()[0].tolist() == g["classes"]
    assert gm.visible_pairs == g["visible_pairs"]


@pytest.mark.parametrize("bad,code", [
    ([[0, 100, 10, 20], [0, 50, 0, 10]], kvs.KVS_ERR_EVENT_ORDER),   # tau decreasing
    ([[0, 100, 10, 120]], kvs.KVS_ERR_EVENT_ORDER),                  # end > tau
    ([[0, 100, 20, 20]], kvs.KVS_ERR_EVENT_ORDER),                   # empty range
    ([[5, 100, 10, 20]], kvs.KVS_ERR_INVALID_ARG),                   # seq out of range
])
def test_mask_event_errors(bad, code):
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_build_tile_mask(events_dev(bad), 2, 256)
    assert e.value.code == code


# ------------------------------------------------- mask, asynchronous build

_SENT = -7


def _mask_buffers(B, N, nnz_cap, part_cap, extra=64):
    """A TileMask whose list buffers hold nnz_cap / part_cap entries (views of
    larger sentinel-filled stores, so writes past the capacity would stay in
    allocated memory and show up as changed sentinels)."""
    T = (N + 127) // 128
    i32 = dict(dtype=torch.int32, device="cuda")
    stores = [torch.full((max(nnz_cap, 1) + extra,), _SENT, **i32) for _ in range(4)]
    bstore = torch.full(((max(part_cap, 1) + 1) * 512,), _SENT, **i32)
    lists = [st[:max(nnz_cap, 1)] for st in stores]
    bits = bstore[:max(part_cap, 1) * 512].view(-1, 128, 4)
    m = kvs.TileMask(B, N, T, torch.full((B, N), _SENT, **i32),
                     torch.zeros((B, T, T), dtype=torch.uint8, device="cuda"),
                     torch.full((B * T + 1,), _SENT, **i32), lists[0], lists[1],
                     torch.full((B * T + 1,), _SENT, **i32), lists[2], lists[3], bits, 0, 0, 0)
    return m, stores, bstore


def _async_build(ev, m):
    sizes = torch.zeros(3, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvs.kvs_build_tile_mask_async(events_dev(ev), m, sizes=sizes, status=status)
    torch.cuda.synchronize()
    return [int(x) for x in sizes.cpu()], int(status.item())


@pytest.mark.parametrize("cid,div", [(1, 1), (2, 8), (5, 16)])
def test_mask_async_configs(cid, div):
    """The host-round-trip-free build, with capacities from the oracle's counts,
    equals the oracle bit for bit (lists, bits and the device-reported sizes)."""
    cfg = W.scaled(W.CONFIGS[cid], div)
    ev = W.make_event_log(cfg)
    B, N = cfg.batch, cfg.n_tokens
    om = oracle.tile_mask(oracle.kappa(ev, B, N))
    m, _, _ = _mask_buffers(B, N, om["nnz"], om["n_partial"])
    (nnz, npart, pairs), st = _async_build(ev, m)
    assert st == 0
    m.nnz, m.n_partial, m.visible_pairs = nnz, npart, pairs
    compare_mask(m, ev, B, N)


@pytest.mark.parametrize("N,seed", [(300, 1), (1000, 2), (129, 4)])
def test_mask_async_reuses_buffers(N, seed):
    """A training loop recompiles each step's log into the buffers of an earlier
    build: a second, different log into the same buffers gives its own mask."""
    rng = np.random.default_rng(seed)
    ev1 = W.random_event_log(rng, 3, N, 12, unit=1, max_span=max(1, N // 4))
    ev2 = W.random_event_log(rng, 3, N, 6, unit=1, max_span=max(1, N // 8))
    gm = kvs.kvs_build_tile_mask(events_dev(ev1), 3, N)
    om2 = oracle.tile_mask(oracle.kappa(ev2, 3, N))
    if om2["nnz"] > gm.row_col.numel() or om2["n_partial"] > gm.bits.shape[0]:
        gm, _, _ = _mask_buffers(3, N, om2["nnz"], om2["n_partial"])
    (nnz, npart, pairs), st = _async_build(ev2, gm)
    assert st == 0
    gm.nnz, gm.n_partial, gm.visible_pairs = nnz, npart, pairs
    compare_mask(gm, ev2, 3, N)


@pytest.mark.parametrize("short", ["nnz", "partial"])
def test_mask_async_over_capacity(short):
    """Lists that do not fit: KVS_ERR_CAPACITY in the status word, the sizes
    still reported, no list entry or bit row written, and every row/column
    offset zero (the mask reads as empty)."""
    rng = np.random.default_rng(11)
    B, N = 3, 1000
    ev = W.random_event_log(rng, B, N, 12, unit=1, max_span=N // 4)
    om = oracle.tile_mask(oracle.kappa(ev, B, N))
    assert om["nnz"] >= 2 and om["n_partial"] >= 2
    nc = om["nnz"] - (1 if short == "nnz" else 0)
    pc = om["n_partial"] - (1 if short == "partial" else 0)
    m, stores, bstore = _mask_buffers(B, N, nc, pc)
    (nnz, npart, pairs), st = _async_build(ev, m)
    assert st == kvs.KVS_ERR_CAPACITY
    assert (nnz, npart) == (om["nnz"], om["n_partial"])
    assert pairs == oracle.visible_pairs(oracle.kappa(ev, B, N))
    assert not m.row_ptr.any().item() and not m.col_ptr.any().item()
    for t in stores + [bstore]:
        assert bool((t == _SENT).all().item())


@pytest.mark.parametrize("bad,code", [
    ([[0, 100, 10, 20], [0, 50, 0, 10]], kvs.KVS_ERR_EVENT_ORDER),
    ([[5, 100, 10, 20]], kvs.KVS_ERR_INVALID_ARG),
])
def test_mask_async_event_errors(bad, code):
    """Event-log errors land in the status word and leave the mask empty."""
    m, _, _ = _mask_buffers(2, 256, 8, 8)
    _, st = _async_build(bad, m)
    assert st == code
    assert not m.row_ptr.any().item() and not m.col_ptr.any().item()


# ------------------------------------------------------------------ compaction

def _compact_gpu(st, events):
    bt, bl = dev(st.block_table), dev(st.block_lpos)
    nb, nt = dev(st.num_blocks), dev(st.num_tokens)
    fr, nf, status = kvs.kvs_compact_block_table(bt, bl, nb, nt, st.block_size, st.pool_blocks,
                                                 events_dev(events))
    torch.cuda.synchronize()
    return (int(status.item()), bt.cpu().numpy(), bl.cpu().numpy(), nb.cpu().numpy(),
            nt.cpu().numpy(), fr.cpu().numpy(), nf.cpu().numpy())


@pytest.mark.parametrize("div", [1, 8])
def test_compact_paged_config(div):
    st = W.make_paged_state(W.CONFIGS[4], div=div)
    st_rc, bt, bl, nb, nt, fr, nf = _compact_gpu(st, st.events)
    rc, obt, obl, onb, ont, ofr, onf = oracle.compact(st.block_table, st.block_lpos, st.num_blocks,
                                                      st.num_tokens, st.block_size, st.events)
    assert st_rc == 0 and rc == 0
    assert np.array_equal(bt, obt) and np.array_equal(bl, obl)
    assert np.array_equal(nb, onb) and np.array_equal(nt, ont) and np.array_equal(nf, onf)
    for b in range(len(nf)):
        assert np.array_equal(fr[b, :nf[b]], ofr[b, :onf[b]])


def test_compact_golden_and_errors():
    g = json.load(open(os.path.join(GOLD, "compact_small.json")))
    M = 8
    st = W.PagedState(block_size=16, pool_blocks=64, max_blocks=M,
                      block_table=np.full((1, M), -1, np.int32), block_lpos=np.full((1, M), -1, np.int32),
                      num_blocks=np.array([6], np.int32), num_tokens=np.array([96], np.int32),
                      next_lpos=np.array([128], np.int32), events=None, new_block=None)
    st.block_table[0, :6] = g["block_table"]
    st.block_lpos[0, :6] = g["block_lpos"]
    for c in g["cases"]:
        rc, bt, bl, nb, nt, fr, nf = _compact_gpu(st, c["events"])
        if c["status"] == "unaligned":
            assert rc == kvs.KVS_ERR_UNALIGNED and nf[0] == 0
            assert np.array_equal(bt, st.block_table)          # sequence left unchanged
            continue
        assert rc == 0
        assert bt[0, :nb[0]].tolist() == c["table"] and bl[0, :nb[0]].tolist() == c["lpos"]
        assert nt[0] == c["num_tokens"] and fr[0, :nf[0]].tolist() == c["freed"]
    # block id outside the pool
    st.block_table[0, 2] = 1000
    rc, *_ = _compact_gpu(st, [[0, 128, 16, 48]])
    assert rc == kvs.KVS_ERR_INVALID_ARG


def test_compact_bs1_random():
    rng = np.random.default_rng(3)
    B, M = 4, 3000
    bt = np.full((B, M), -1, np.int32); bl = np.full((B, M), -1, np.int32)
    nb = np.zeros(B, np.int32)
    perm = rng.permutation(B * M).astype(np.int32)
    rows = []
    for b in range(B):
        n = int(rng.integers(1, M))
        lp = np.sort(rng.choice(20000, n, replace=False)).astype(np.int32)
        bt[b, :n] = perm[b * M: b * M + n]; bl[b, :n] = lp; nb[b] = n
        for _ in range(int(rng.integers(0, 20))):
            s = int(rng.integers(0, 20000)); rows.append((b, 20000, s, s + int(rng.integers(1, 500))))
    rows.sort()
    ev = np.array(rows, np.int32).reshape(-1, 4)
    st = W.PagedState(1, B * M, M, bt, bl, nb, nb.copy(), None, ev, None)
    rc, gbt, gbl, gnb, gnt, gfr, gnf = _compact_gpu(st, ev)
    orc, obt, obl, onb, ont, ofr, onf = oracle.compact(bt, bl, nb, nb.copy(), 1, ev)
    assert rc == 0 and orc == 0
    assert np.array_equal(gbt, obt) and np.array_equal(gbl, obl) and np.array_equal(gnt, ont)
    for b in range(B):
        assert np.array_equal(gfr[b, :gnf[b]], ofr[b, :onf[b]])


# ------------------------------------------------------------------ rope

@pytest.mark.parametrize("dtype,d,theta", [(torch.float32, 64, 1e4), (torch.bfloat16, 128, 5e5),
                                           (torch.float32, 128, 5e5)])
def test_rope_vs_oracle(dtype, d, theta):
    rng = np.random.default_rng(0)
    n, H = 700, 5
    x = W.round_bf16(rng.standard_normal((n, H, d)).astype(np.float32)) if dtype == torch.bfloat16 \
        else rng.standard_normal((n, H, d)).astype(np.float32)
    lpos = rng.integers(0, 131072, n).astype(np.int32)
    lpos[:3] = [0, 1, 131071]
    xd = dev(x, dtype)
    for inv in (False, True):
        y = host(kvs.kvs_rope_logical(xd, dev(lpos), theta, inverse=inv))
        want = oracle.rope(x.astype(np.float64), lpos, theta, inverse=inv)
        if dtype == torch.float32:
            assert np.abs(y - want).max() <= 1e-5
        else:  # one bf16 rounding of the output
            assert (np.abs(y - want) <= np.abs(want) * 2.0 ** -8 + 1e-6).all()


def test_rope_roundtrip_and_strided_input():
    rng = np.random.default_rng(1)
    n, H, d = 300, 4, 64
    qkv = dev(rng.standard_normal((n, 3 * H * d)).astype(np.float32))
    k = qkv[:, H * d: 2 * H * d].view(n, H, d)                 # row stride 3*H*d
    lpos = dev(rng.integers(0, 100000, n).astype(np.int32))
    y = kvs.kvs_rope_logical(k, lpos, 1e4)
    back = kvs.kvs_rope_logical(y, lpos, 1e4, inverse=True)
    assert (back - k).abs().max().item() <= 1e-5


def test_rope_scatter_into_paged_cache():
    rng = np.random.default_rng(2)
    pool, H, bs, d = 40, 8, 16, 128
    n = 10
    kc = torch.zeros((pool, H, bs, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    k = dev(W.round_bf16(rng.standard_normal((n, H, d)).astype(np.float32)), torch.bfloat16)
    v = dev(W.round_bf16(rng.standard_normal((n, H, d)).astype(np.float32)), torch.bfloat16)
    lpos = rng.integers(0, 131072, n).astype(np.int32)
    slots = rng.choice(pool * bs, n, replace=False).astype(np.int64)
    kvs.kvs_rope_logical(k, dev(lpos), 5e5, out=kc, out_slot=dev(slots), block_size=bs, v=v, v_out=vc)
    want = oracle.rope(host(k), lpos, 5e5)
    for i, s in enumerate(slots):
        got_k = host(kc[s // bs, :, s % bs])
        assert (np.abs(got_k - want[i]) <= np.abs(want[i]) * 2.0 ** -8 + 1e-6).all()
        assert torch.equal(vc[s // bs, :, s % bs], v[i])


def test_rope_scatter_skips_slots_outside_the_cache():
    """A slot outside [0, pool * block_size) is reported (KVS_ERR_INVALID_ARG) and
    nothing is written for its row; every other byte of both caches is untouched
    except the valid rows' slots."""
    rng = np.random.default_rng(3)
    pool, H, bs, d = 12, 2, 16, 128
    n = 8
    kc = dev(W.round_bf16(rng.standard_normal((pool, H, bs, d)).astype(np.float32)), torch.bfloat16)
    vc = dev(W.round_bf16(rng.standard_normal((pool, H, bs, d)).astype(np.float32)), torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    k = dev(W.round_bf16(rng.standard_normal((n, H, d)).astype(np.float32)), torch.bfloat16)
    v = dev(W.round_bf16(rng.standard_normal((n, H, d)).astype(np.float32)), torch.bfloat16)
    lpos = rng.integers(0, 131072, n).astype(np.int32)
    slots = np.array([5, -1, pool * bs, 17, pool * bs + 100, 2**40, 190, 0], np.int64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvs.kvs_rope_logical(k, dev(lpos), 5e5, out=kc, out_slot=dev(slots), block_size=bs, v=v, v_out=vc,
                         status=status)
    torch.cuda.synchronize()
    assert status.item() == kvs.KVS_ERR_INVALID_ARG
    valid = [i for i, s in enumerate(slots) if 0 <= s < pool * bs]
    want = oracle.rope(host(k), lpos, 5e5)
    touched = torch.zeros((pool, bs), dtype=torch.bool)
    for i in valid:
        s = int(slots[i])
        touched[s // bs, s % bs] = True
        got = host(kc[s // bs, :, s % bs])
        assert (np.abs(got - want[i]) <= np.abs(want[i]) * 2.0 ** -8 + 1e-6).all()
        assert torch.equal(vc[s // bs, :, s % bs], v[i])
    keep = (~touched).cuda()[:, None, :, None].expand_as(kc)
    assert torch.equal(kc[keep], k0[keep]) and torch.equal(vc[keep], v0[keep])
