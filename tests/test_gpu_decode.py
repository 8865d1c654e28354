"""GPU parity: split-K paged decode over compacted block tables."""
import numpy as np
import pytest
import torch

import oracle
import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import workloads as W
from gpu_util import BF16_TOL, F32_TOL, assert_close, dev, events_dev, host

pytestmark = pytest.mark.gpu


def _snapshot_tables(kap_b, ts, bs, perm):
    """Generation-side paged state at each time t (one 'sequence' per t): the live
    blocks of positions <= t in logical order, placed at pool blocks perm[i]."""
    N = kap_b.shape[0]
    nblk_all = (N + bs - 1) // bs
    tables, ntok = [], []
    for t in ts:
        blocks = [i for i in range(t // bs + 1) if kap_b[i * bs] > t]
        n = 0
        for i in blocks:
            n += min(bs, t + 1 - i * bs)
        tables.append([perm[i] for i in blocks])
        ntok.append(n)
    M = max(len(x) for x in tables)
    bt = np.full((len(ts), M), -1, np.int32)
    for r, row in enumerate(tables):
        bt[r, :len(row)] = row
    return bt, np.array(ntok, np.int32), nblk_all


def _decode_vs_replay(cfg, ts, seed=0):
    """Decode every t in ts over the compacted paged cache; return GPU decode,
    oracle rows and (for bf16) the raw inputs."""
    N, Hq, Hkv, d, bs = cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d, cfg.block_size
    ev = W.make_event_log(W.replace(cfg, batch=1))
    kap = oracle.kappa(ev, 1, N)
    q, k, v, _ = W.replay_tensors(W.replace(cfg, batch=1))
    q, k, v = q[0], k[0], v[0]
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    rng = np.random.default_rng(seed)
    nblk = (N + bs - 1) // bs
    perm = rng.permutation(nblk + 7).astype(np.int32)
    bt, ntok, _ = _snapshot_tables(kap[0], ts, bs, perm)
    # cache: every position's rotated key at its block slot (logical position kept)
    pool = nblk + 7
    kc = torch.zeros((pool, Hkv, bs, d), dtype=tdt, device="cuda")
    vc = torch.zeros_like(kc)
    lpos = np.arange(N, dtype=np.int32)
    slots = (perm[lpos // bs].astype(np.int64) * bs + lpos % bs)
    kvs.kvs_rope_logical(dev(k, tdt), dev(lpos), cfg.theta, out=kc, out_slot=dev(slots), block_size=bs,
                         v=dev(v, tdt), v_out=vc)
    qt = dev(q[ts], tdt)                                    # [len(ts), Hq, d]
    qr = kvs.kvs_rope_logical(qt, dev(np.array(ts, np.int32)), cfg.theta)
    o = kvs.kvs_paged_decode_attn(qr, kc, vc, dev(bt), dev(ntok), bs, cfg.scale)
    got = host(o)
    # oracle: rotate in fp64, attend replay row t
    kr = oracle.rope(k.astype(np.float64), lpos, cfg.theta)
    qo = oracle.rope(q[ts].astype(np.float64), np.array(ts), cfg.theta)
    G = Hq // Hkv
    want = np.empty_like(got)
    for i, t in enumerate(ts):
        for h in range(Hq):
            r, _ = oracle.attn_rows(qo[i, h][None], [t], kr[:, h // G], v[:, h // G], kap[0], cfg.scale)
            want[i, h] = r[0]
    return got, want, (q, k, v, kap, ev)


def test_decode_fp32_tiny_config():
    cfg = W.CONFIGS[1]
    ts = [0, 1, 15, 16, 127, 128, 500, 1135, 1136, 1137, 1500, 1727, 1728, 2000, 2047]
    got, want, _ = _decode_vs_replay(cfg, ts)
    assert_close(got, want, F32_TOL, "fp32 decode")


def test_decode_bs1_bf16_scaled():
    cfg = W.replace(W.scaled(W.CONFIGS[5], 16), batch=1)
    ev = W.make_event_log(cfg)
    taus = sorted(set(ev[:, 1].tolist()))
    ts = sorted(set([0, 5, 127, 128, cfg.n_tokens - 1] + [t for x in taus for t in (x - 1, x, x + 1)
                                                           if 0 <= t < cfg.n_tokens]))
    got, want, _ = _decode_vs_replay(cfg, ts)
    assert_close(got, want, BF16_TOL, "bs1 decode")


def test_decode_bs1_full_size():
    """The bs1 trace workload's decode at full size, in the launch configuration the
    step times: two traces of 131 072 positions, 1-token blocks at random slots, each
    trace's table right before its last event compacted through the library, the new
    token roped and appended at its logical position, then one decode call (a wave of
    split CTAs and the merge). The compacted tables must hold exactly the keys the
    oracle's kill times keep, and every query head must match the oracle's replay
    row at that position."""
    cfg = W.CONFIGS[5]
    B, N, Hq, Hkv, d = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d
    G = Hq // Hkv
    ev = W.make_event_log(cfg)
    kap = oracle.kappa(ev, B, N)
    q_raw, k_raw, v, _ = W.replay_tensors_device(cfg, device="cuda", with_grad=False)
    pool = B * N + B
    perm = np.random.default_rng(77).permutation(pool).astype(np.int64)
    kc = torch.zeros((pool, Hkv, 1, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    lpos = torch.arange(N, dtype=torch.int32, device="cuda")
    taus, tables, lposs = [], [], []
    for b in range(B):
        tau = int(ev[ev[:, 0] == b, 1].max())
        j = np.arange(tau)
        live = j[kap[b, :tau] >= tau]  # alive right before the event at tau
        taus.append(tau)
        tables.append(perm[b * N + live].astype(np.int32))
        lposs.append(live.astype(np.int32))
        kvs.kvs_rope_logical(k_raw[b], lpos, cfg.theta, out=kc, out_slot=dev(perm[b * N:(b + 1) * N]),
                             block_size=1, v=v[b], v_out=vc)
    M = max(len(t) for t in tables) + 1
    bt = np.full((B, M), -1, np.int32)
    bl = np.full((B, M), -1, np.int32)
    for b in range(B):
        bt[b, :len(tables[b])] = tables[b]
        bl[b, :len(lposs[b])] = lposs[b]
    nb = np.array([len(t) for t in tables], np.int32)
    dbt, dbl, dnb, dnt = dev(bt), dev(bl), dev(nb), dev(nb)
    last = np.concatenate([ev[(ev[:, 0] == b) & (ev[:, 1] == taus[b])] for b in range(B)])
    _, _, status = kvs.kvs_compact_block_table(dbt, dbl, dnb, dnt, 1, pool, events_dev(last))
    # the new token of trace b: logical position tau_b, physical slot perm[B N + b]
    tl = dev(np.array(taus, np.int32))
    rows = torch.from_numpy(np.array([b * N + taus[b] for b in range(B)])).cuda()
    qn = q_raw.view(B * N, Hq, d).index_select(0, rows)
    kn = k_raw.view(B * N, Hkv, d).index_select(0, rows).contiguous()
    vn = v.view(B * N, Hkv, d).index_select(0, rows).contiguous()
    new_slot = perm[B * N:B * N + B]
    kvs.kvs_rope_logical(kn, tl, cfg.theta, out=kc, out_slot=dev(new_slot), block_size=1, v=vn, v_out=vc)
    qr = kvs.kvs_rope_logical(qn, tl, cfg.theta)
    # the oracle's inputs (raw rows up to tau) move to the host; the decode then runs
    # with only the caches and tables on the device
    raw = [(host(q_raw[b, taus[b]]), host(k_raw[b, :taus[b] + 1]), host(v[b, :taus[b] + 1])) for b in range(B)]
    del q_raw, k_raw, v, qn, kn, vn
    torch.cuda.empty_cache()
    nb_after = dnb.cpu().numpy()
    dbt[torch.arange(B, device="cuda"), torch.from_numpy(nb_after.astype(np.int64)).cuda()] = \
        dev(new_slot.astype(np.int32))
    dnt += 1
    o = host(kvs.kvs_paged_decode_attn(qr, kc, vc, dbt, dnt, 1, cfg.scale, status=status))
    assert int(status.item()) == 0
    got_bt = dbt.cpu().numpy()
    for b in range(B):
        tau = taus[b]
        keep = np.arange(tau)[kap[b, :tau] > tau]  # kept by the event at tau
        assert nb_after[b] == len(keep)
        assert np.array_equal(got_bt[b, :nb_after[b]], perm[b * N + keep].astype(np.int32))
        # oracle: raw keys and values up to tau, rotated in fp64, replay row tau
        qh, kh, vv = raw[b]
        kr = oracle.rope(kh, np.arange(tau + 1), cfg.theta)
        qo = oracle.rope(qh[None], [tau], cfg.theta)[0]
        want = np.empty((Hq, d))
        for h in range(Hq):
            r, _ = oracle.attn_rows(qo[h][None], [tau], kr[:, h // G], vv[:, h // G], kap[b, :tau + 1],
                                    cfg.scale)
            want[h] = r[0]
        assert_close(o[b], want, BF16_TOL, f"bs1 full-size decode seq {b}")


def _paged_step(div):
    """One generation step of the paged workload: compaction, RoPE + append of the
    new token at its logical position, decode. Returns what the oracle needs."""
    cfg = W.CONFIGS[4]
    st = W.make_paged_state(cfg, div=div)
    B, Hq, Hkv, d, bs = cfg.batch, cfg.hq, cfg.hkv, cfg.d, st.block_size
    g = torch.Generator(device="cuda")
    g.manual_seed(4000 + div)
    kc = torch.randn((st.pool_blocks, Hkv, bs, d), generator=g, device="cuda", dtype=torch.bfloat16)
    vc = torch.randn((st.pool_blocks, Hkv, bs, d), generator=g, device="cuda", dtype=torch.bfloat16)
    q_raw = torch.randn((B, Hq, d), generator=g, device="cuda", dtype=torch.bfloat16)
    k_new = torch.randn((B, Hkv, d), generator=g, device="cuda", dtype=torch.bfloat16)
    v_new = torch.randn((B, Hkv, d), generator=g, device="cuda", dtype=torch.bfloat16)
    M = st.max_blocks + 1
    bt = np.full((B, M), -1, np.int32); bt[:, :st.max_blocks] = st.block_table
    bl = np.full((B, M), -1, np.int32); bl[:, :st.max_blocks] = st.block_lpos
    dbt, dbl, dnb, dnt = dev(bt), dev(bl), dev(st.num_blocks), dev(st.num_tokens)
    _, _, status = kvs.kvs_compact_block_table(dbt, dbl, dnb, dnt, bs, st.pool_blocks, events_dev(st.events))
    # the new token opens a new block (live counts stay multiples of 16 after compaction)
    nb = dnb.cpu().numpy(); nt = dnt.cpu().numpy()
    assert (nt % bs == 0).all() and status.item() == 0
    rows = torch.arange(B, device="cuda")
    nbi = torch.from_numpy(nb.astype(np.int64)).cuda()
    dbt[rows, nbi] = dev(st.new_block)
    dbl[rows, nbi] = dev(st.next_lpos)
    slots = st.new_block.astype(np.int64) * bs
    lp = dev(st.next_lpos)
    kvs.kvs_rope_logical(k_new, lp, cfg.theta, out=kc, out_slot=dev(slots), block_size=bs, v=v_new,
                         v_out=vc)
    dnt += 1
    qr = kvs.kvs_rope_logical(q_raw, lp, cfg.theta)
    o = kvs.kvs_paged_decode_attn(qr, kc, vc, dbt, dnt, bs, cfg.scale)
    torch.cuda.synchronize()
    return cfg, st, dict(kc=kc, vc=vc, q=q_raw, k_new=k_new, v_new=v_new, bt=dbt.cpu().numpy(),
                         nt=dnt.cpu().numpy(), o=host(o))


@pytest.mark.parametrize("div", [8, 1])
def test_decode_paged_generation_step(div):
    cfg, st, r = _paged_step(div)
    B, bs = cfg.batch, st.block_size
    # oracle: compaction as a list filter, rotation in fp64, decode by walking the table
    rc, obt, obl, onb, ont, *_ = oracle.compact(st.block_table, st.block_lpos, st.num_blocks,
                                                st.num_tokens, bs, st.events)
    assert rc == 0
    check = [int(np.argmin(st.num_tokens)), int(np.argmax(st.num_tokens)), 0, B - 1, B // 2]
    for b in sorted(set(check)):
        live = obt[b, :onb[b]]
        assert np.array_equal(r["bt"][b, :onb[b]], live)
        # gather this sequence's live blocks into a small pool (inputs only)
        idx = torch.from_numpy(live.astype(np.int64)).cuda()
        kp = host(r["kc"].index_select(0, idx)); vp = host(r["vc"].index_select(0, idx))
        knew = oracle.rope(host(r["k_new"][b])[None], [st.next_lpos[b]], cfg.theta)[0]
        kp = np.concatenate([kp, np.zeros_like(kp[:1])]); vp = np.concatenate([vp, np.zeros_like(vp[:1])])
        kp[-1, :, 0] = knew; vp[-1, :, 0] = host(r["v_new"][b])
        table = np.arange(len(live) + 1, dtype=np.int32)[None]
        qo = oracle.rope(host(r["q"][b])[None], [st.next_lpos[b]], cfg.theta)
        want = oracle.paged_decode(qo, kp, vp, table, np.array([ont[b] + 1]), bs, cfg.scale)[0]
        assert_close(r["o"][b], want, BF16_TOL, f"paged decode seq {b}")


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_group_sizes_and_empty(G):
    rng = np.random.default_rng(G)
    B, Hkv, d, bs, M = 3, 2, 128, 16, 40
    Hq = G * Hkv
    pool = 200
    kc = W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    vc = W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    q = W.round_bf16(rng.standard_normal((B, Hq, d)).astype(np.float32))
    bt = rng.permutation(pool)[: B * M].reshape(B, M).astype(np.int32)
    nt = np.array([0, 1, M * bs - 5], np.int32)
    o = host(kvs.kvs_paged_decode_attn(dev(q, torch.bfloat16), dev(kc, torch.bfloat16),
                                       dev(vc, torch.bfloat16), dev(bt), dev(nt), bs, 1 / np.sqrt(d)))
    want = oracle.paged_decode(q, kc, vc, bt, nt, bs, 1 / np.sqrt(d))
    assert np.abs(o[0]).max() == 0.0                     # no live entries -> zeros
    assert_close(o, want, BF16_TOL, "decode G")


@pytest.mark.parametrize("dt,bs", [("bf16", 16), ("bf16", 1), ("bf16", 4), ("f32", 16)])
def test_decode_skips_block_ids_outside_the_pool(dt, bs):
    """Block ids < 0 or >= the pool size are reported (KVS_ERR_INVALID_ARG) and their
    entries left out of the softmax; nothing outside the pool is read. The expected
    output is the oracle's decode over the same table with those blocks removed."""
    rng = np.random.default_rng(11 + bs)
    B, Hkv, G = 3, 2, 4
    d = 128 if dt == "bf16" else 64
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    Hq, M = G * Hkv, (1200 + bs - 1) // bs
    pool = B * M + 5
    cast = W.round_bf16 if dt == "bf16" else (lambda a: a)
    kc = cast(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    vc = cast(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    q = cast(rng.standard_normal((B, Hq, d)).astype(np.float32))
    bt = rng.permutation(pool)[: B * M].reshape(B, M).astype(np.int32)
    bad = [(0, 0, -1), (0, M // 2, pool), (1, 3, -7), (2, M - 2, pool + 1000)]
    for b, i, v in bad:
        bt[b, i] = v
    nt = np.full(B, M * bs, np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = host(kvs.kvs_paged_decode_attn(dev(q, tdt), dev(kc, tdt), dev(vc, tdt), dev(bt), dev(nt), bs,
                                       1 / np.sqrt(d), status=status))
    torch.cuda.synchronize()
    assert status.item() == kvs.KVS_ERR_INVALID_ARG
    assert np.isfinite(o).all()
    keep = np.full((B, M), -1, np.int32)
    nt_keep = np.zeros(B, np.int32)
    for b in range(B):
        row = [x for x in bt[b] if 0 <= x < pool]
        keep[b, :len(row)] = row
        nt_keep[b] = len(row) * bs
    want = oracle.paged_decode(q, kc, vc, keep, nt_keep, bs, 1 / np.sqrt(d))
    assert_close(o, want, BF16_TOL if dt == "bf16" else F32_TOL, f"decode without bad blocks {dt} bs={bs}")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_decode_reports_token_counts_past_the_table(dt):
    """num_tokens beyond max_blocks * block_size is reported and clamped."""
    rng = np.random.default_rng(5)
    B, Hkv, Hq, bs, M = 2, 1, 2, 16, 9
    d = 128 if dt == "bf16" else 64
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    pool = B * M
    kc = W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    vc = W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    q = W.round_bf16(rng.standard_normal((B, Hq, d)).astype(np.float32))
    bt = rng.permutation(pool).reshape(B, M).astype(np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = host(kvs.kvs_paged_decode_attn(dev(q, tdt), dev(kc, tdt), dev(vc, tdt), dev(bt),
                                       dev(np.array([M * bs + 5, 20], np.int32)), bs, 0.1, status=status))
    torch.cuda.synchronize()
    assert status.item() == kvs.KVS_ERR_INVALID_ARG
    want = oracle.paged_decode(q, kc, vc, bt, np.array([M * bs, 20], np.int32), bs, 0.1)
    assert_close(o, want, BF16_TOL if dt == "bf16" else F32_TOL, "clamped count")


def test_decode_negative_block_id_reports():
    B, Hkv, d, bs = 1, 1, 128, 16
    kc = torch.zeros((4, Hkv, bs, d), dtype=torch.bfloat16, device="cuda")
    bt = dev(np.array([[0, -1, 2]], np.int32))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvs.kvs_paged_decode_attn(torch.zeros((1, 1, d), dtype=torch.bfloat16, device="cuda"), kc, kc, bt,
                              dev(np.array([40], np.int32)), bs, 0.1, status=status)
    assert status.item() == kvs.KVS_ERR_INVALID_ARG


@pytest.mark.parametrize("bs", [4, 8, 32])
def test_decode_other_block_sizes(bs):
    """Block sizes other than 16 and 1 take the kernel's general addressing path
    (the two the workloads use have their own); several splits per sequence."""
    rng = np.random.default_rng(100 + bs)
    B, Hkv, G, d = 3, 2, 4, 128
    Hq = G * Hkv
    M = (1600 + bs - 1) // bs
    pool = B * M + 7
    kc = W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    vc = W.round_bf16(rng.standard_normal((pool, Hkv, bs, d)).astype(np.float32))
    q = W.round_bf16(rng.standard_normal((B, Hq, d)).astype(np.float32))
    bt = rng.permutation(pool)[: B * M].reshape(B, M).astype(np.int32)
    nt = np.array([M * bs, M * bs - bs - 3, 5], np.int32)
    o = host(kvs.kvs_paged_decode_attn(dev(q, torch.bfloat16), dev(kc, torch.bfloat16),
                                       dev(vc, torch.bfloat16), dev(bt), dev(nt), bs, 1 / np.sqrt(d)))
    want = oracle.paged_decode(q, kc, vc, bt, nt, bs, 1 / np.sqrt(d))
    assert_close(o, want, BF16_TOL, f"decode bs={bs}")
