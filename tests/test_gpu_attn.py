"""GPU parity: eviction-masked attention forward and backward (fp32 CUDA-core
path and bf16 tcgen05 path) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import workloads as W
from gpu_util import (BF16_TOL, F32_ROUND, F32_TOL, GRAD_REL_L2, LSE_TOL, assert_close, dev, events_dev,
                      host, rel_l2)

pytestmark = pytest.mark.gpu


def _run(cfg, ev, q, k, v, do, bwd=True):
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    gm = kvs.kvs_build_tile_mask(events_dev(ev), cfg.batch, cfg.n_tokens)
    qd, kd, vd = dev(q, tdt), dev(k, tdt), dev(v, tdt)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, o_lo = kvs.kvs_masked_attn_fwd(qd, kd, vd, gm, cfg.scale, status=status)
    out = dict(o=o, lse=lse, mask=gm)
    if bwd:
        dq, dk, dv = kvs.kvs_masked_attn_bwd(qd, kd, vd, o, dev(do, tdt), lse, gm, cfg.scale, status=status,
                                             o_lo=o_lo)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert status.item() == 0, kvs.status_str(status.item())
    return out


def _check_full(cfg, ev, q, k, v, do, tol, bwd=True):
    r = _run(cfg, ev, q, k, v, do, bwd)
    kap = oracle.kappa(ev, cfg.batch, cfg.n_tokens)
    if bwd:
        o, lse, dq, dk, dv = oracle.attn_bwd(q, k, v, do, kap, cfg.scale)
    else:
        o, lse = oracle.attn_fwd(q, k, v, kap, cfg.scale)
    assert_close(host(r["o"]), o, tol, "O")
    # lse is fp32 on both paths: no bf16 rounding allowance
    assert_close(host(r["lse"]), lse, LSE_TOL if tol == BF16_TOL else F32_TOL, "LSE", rnd=F32_ROUND)
    if bwd:
        for name, want in (("dq", dq), ("dk", dk), ("dv", dv)):
            got = host(r[name])
            assert_close(got, want, tol, name)
            rl = rel_l2(got, want)
            assert rl is None or rl <= GRAD_REL_L2, (name, rl)
    return r


def test_fp32_tiny_config_fwd_bwd():
    cfg = W.CONFIGS[1]
    ev = W.make_event_log(cfg)
    q, k, v, do = W.replay_tensors(cfg)
    _check_full(cfg, ev, q, k, v, do, F32_TOL)


@pytest.mark.parametrize("cid,div,hq,hkv,batch", [
    (2, 8, 8, 2, 2),      # recent-turns policy, GQA 4
    (3, 16, 8, 2, 2),     # summary policy
    (5, 32, 16, 2, 1),    # 1-token blocks, unpadded turns, GQA 8
])
def test_bf16_scaled_configs_fwd_bwd(cid, div, hq, hkv, batch):
    cfg = W.replace(W.scaled(W.CONFIGS[cid], div), hq=hq, hkv=hkv, batch=batch)
    ev = W.make_event_log(cfg)
    assert len(ev) > 0
    q, k, v, do = W.replay_tensors(cfg)
    _check_full(cfg, ev, q, k, v, do, BF16_TOL)


@pytest.mark.parametrize("N,dtype,seed", [(300, "bf16", 0), (1000, "bf16", 1), (129, "bf16", 2),
                                          (1, "bf16", 3), (300, "f32", 4), (1000, "f32", 5)])
def test_ragged_lengths_random_events(N, dtype, seed):
    d = 128 if dtype == "bf16" else 64
    cfg = W.TraceConfig(cid=90 + seed, name="ragged", batch=2, n_tokens=N, hq=4, hkv=2, d=d,
                        theta=1e4, block_size=1, dtype=dtype, prompt=0)
    ev = W.random_event_log(np.random.default_rng(seed), 2, N, 10, unit=1, max_span=max(1, N // 3))
    q, k, v, do = W.replay_tensors(cfg)
    _check_full(cfg, ev, q, k, v, do, BF16_TOL if dtype == "bf16" else F32_TOL)


def test_bf16_no_events_and_mha():
    cfg = W.TraceConfig(cid=80, name="mha", batch=1, n_tokens=640, hq=3, hkv=3, d=128, theta=1e4,
                        block_size=1, dtype="bf16", prompt=0)
    q, k, v, do = W.replay_tensors(cfg)
    _check_full(cfg, np.zeros((0, 4), np.int32), q, k, v, do, BF16_TOL)


def test_bf16_rope_then_attention_end_to_end():
    # raw q, k -> logical RoPE -> masked attention, both sides from the same raw inputs
    cfg = W.replace(W.scaled(W.CONFIGS[5], 64), hq=8, hkv=1, batch=1)
    ev = W.make_event_log(cfg)
    q, k, v, _ = W.replay_tensors(cfg)
    N = cfg.n_tokens
    lp = np.arange(N, dtype=np.int32)
    qd = kvs.kvs_rope_logical(dev(q[0], torch.bfloat16), dev(lp), cfg.theta)[None]
    kd = kvs.kvs_rope_logical(dev(k[0], torch.bfloat16), dev(lp), cfg.theta)[None]
    gm = kvs.kvs_build_tile_mask(events_dev(ev), 1, N)
    o, lse, _ = kvs.kvs_masked_attn_fwd(qd.contiguous(), kd.contiguous(), dev(v, torch.bfloat16), gm, cfg.scale)
    kap = oracle.kappa(ev, 1, N)
    qo = oracle.rope(q[0], lp, cfg.theta)[None]
    ko = oracle.rope(k[0], lp, cfg.theta)[None]
    want, _ = oracle.attn_fwd(qo, ko, v.astype(np.float64), kap, cfg.scale)
    assert_close(host(o), want, BF16_TOL, "rope+attn")


# ------------------------------------------------------------------ full sizes (sampled)

def _sample_rows(N, ev_b, rng, n=24):
    taus = sorted(set(int(x) for x in ev_b[:, 1])) if len(ev_b) else []
    cand = [0, 1, 127, 128, N - 1] + [t + o for t in taus for o in (-1, 0, 1) if 0 <= t + o < N]
    cand += rng.integers(0, N, n).tolist()
    return sorted(set(cand))


@pytest.mark.parametrize("cid", [2, 3, 5])
def test_full_size_sampled(cid):
    cfg = W.CONFIGS[cid]
    B, N, Hq, Hkv = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv
    G = Hq // Hkv
    ev = W.make_event_log(cfg)
    q, k, v, do = W.replay_tensors_device(cfg)
    gm = kvs.kvs_build_tile_mask(events_dev(ev), B, N)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, o_lo = kvs.kvs_masked_attn_fwd(q, k, v, gm, cfg.scale, status=status)
    bwd = cid in (3, 5)
    if bwd:
        dq, dk, dv = kvs.kvs_masked_attn_bwd(q, k, v, o, do, lse, gm, cfg.scale, status=status, o_lo=o_lo)
    torch.cuda.synchronize()
    assert status.item() == 0
    kap = oracle.kappa(ev, B, N)
    rng = np.random.default_rng(cid)
    for b in (0, B - 1):
        rows = _sample_rows(N, ev[ev[:, 0] == b], rng)
        for h in (0, Hq - 1):
            kvh = h // G
            kk, vv = host(k[b, :, kvh]), host(v[b, :, kvh])
            want_o, want_l = oracle.attn_rows(host(q[b, rows, h]), rows, kk, vv, kap[b], cfg.scale)
            assert_close(host(o[b, rows, h]), want_o, BF16_TOL, f"O b{b} h{h}")
            assert_close(host(lse[b, h, rows]), want_l, LSE_TOL, f"LSE b{b} h{h}", rnd=F32_ROUND)
            if bwd:
                qg = host(q[b, :, kvh * G:(kvh + 1) * G].transpose(0, 1))
                dg = host(do[b, :, kvh * G:(kvh + 1) * G].transpose(0, 1))
                gr = np.full(len(rows), h - kvh * G)
                want = oracle.dq_rows(qg, kk, vv, dg, kap[b], cfg.scale, gr, rows)
                assert_close(host(dq[b, rows, h]), want, BF16_TOL, f"dQ b{b} h{h}")
                cols = list(range(N - 8, N))
                wk, wv = oracle.dkdv_cols(qg, kk, vv, dg, kap[b], cfg.scale, cols)
                assert_close(host(dk[b, cols, kvh]), wk, BF16_TOL, f"dK b{b}")
                assert_close(host(dv[b, cols, kvh]), wv, BF16_TOL, f"dV b{b}")
    if bwd:
        # properties at full size, exact for the true gradients:
        #   sum_j dV_j = sum over the group of dO_t   (every row of P sums to 1)
        #   sum_j dK_j = 0                            (every row of dS sums to 0)
        # The stored gradients are bf16, so each element may be off by half an
        # ulp (2^-9 |x|); and D_t = <dO_t, O_t> is formed from o + o_lo, whose
        # error moves row sums of dS by at most 2^-17 sum_i |dO_ti O_ti|.
        # The bounds below add those rounding terms up (worst case) plus 0.05.
        r9 = 2.0 ** -9
        for b in (0, B - 1):
            dkb, dvb, dob = dk[b].double(), dv[b].double(), do[b].double()
            sdv = dvb.sum(0)                                     # [Hkv, d]
            sdo = dob.sum(0).view(Hkv, G, -1).sum(1)
            tol_v = r9 * dvb.abs().sum(0) + 0.05
            assert ((sdv - sdo).abs() <= tol_v).all(), float((sdv - sdo).abs().max())
            ob, qb = o[b].double(), q[b].double()                # [N, Hq, d]
            dmax = (2.0 ** -17 * (dob * ob).abs().sum(-1))       # [N, Hq] bound on |dS row sum|
            qterm = (dmax[..., None] * qb.abs()).view(N, Hkv, G, -1).sum((0, 2)) * cfg.scale
            tol_k = r9 * dkb.abs().sum(0) + qterm + 0.05
            sdk = dkb.sum(0)
            assert (sdk.abs() <= tol_k).all(), float(sdk.abs().max())


# ------------------------------------------------------------------ dK/dV on long key columns
#
# dK/dV dominate the backward's time through long column walks: a prompt key is
# seen by every later query; a key inside an evicted range by every query up to
# the event (kappa_j < N); with unpadded turns the event falls mid-tile. These
# tests check such columns element by element.

def _long_columns(ev_b, N, prompt, rng, n_rand=6):
    """Prompt keys; for the first, a middle and the last event: the first two and
    the last key of its range and the key after it; the last keys of the trace;
    a few random keys."""
    cols = {0, 1, 127, max(prompt - 1, 0), N - 1, N - 9}
    if len(ev_b):
        for e in {0, len(ev_b) // 2, len(ev_b) - 1}:
            _, tau, s0, e0 = (int(x) for x in ev_b[e])
            cols.update({s0, s0 + 1, e0 - 1, e0})
    cols.update(int(x) for x in rng.integers(0, N, n_rand))
    return sorted(c for c in cols if 0 <= c < N)


def _group_fwd_rows(qg, kk, vv, kap_b, scale, rows):
    """Oracle forward O and LSE of the given rows for every head of one group."""
    G, N, d = qg.shape
    og, lg = np.zeros((G, N, d)), np.full((G, N), np.inf)
    for g in range(G):
        og[g, rows], lg[g, rows] = oracle.attn_rows(qg[g, rows], rows, kk, vv, kap_b, scale)
    return og, lg


@pytest.mark.parametrize("cid,div", [(3, 4), (5, 4)])
def test_dkdv_long_columns_scaled(cid, div):
    """Summary-policy and 1-token-block traces at 1/4 length (128 and 256 query tiles),
    full dO: dK/dV of prompt keys, keys of evicted ranges and keys after them against
    the oracle, element by element, for the first kv group of trace 0."""
    cfg = W.replace(W.scaled(W.CONFIGS[cid], div), batch=1)
    B, N, Hq, Hkv = 1, cfg.n_tokens, cfg.hq, cfg.hkv
    G = Hq // Hkv
    ev = W.make_event_log(cfg)
    assert len(ev) >= 2
    q, k, v, do = W.replay_tensors(cfg)
    r = _run(cfg, ev, q, k, v, do)
    kap = oracle.kappa(ev, B, N)
    cols = _long_columns(ev, N, cfg.prompt, np.random.default_rng(cid))
    kk, vv = k[0, :, 0].astype(np.float64), v[0, :, 0].astype(np.float64)
    qg = np.transpose(q[0, :, :G], (1, 0, 2)).astype(np.float64)
    dg = np.transpose(do[0, :, :G], (1, 0, 2)).astype(np.float64)
    og, lg = _group_fwd_rows(qg, kk, vv, kap[0], cfg.scale, np.arange(N))
    wk, wv = oracle.dkdv_cols_fwd(qg, kk, vv, dg, og, lg, kap[0], cfg.scale, cols)
    gk, gv = host(r["dk"][0, cols, 0]), host(r["dv"][0, cols, 0])
    assert_close(gk, wk, BF16_TOL, f"dK long columns cfg{cid}/{div}")
    assert_close(gv, wv, BF16_TOL, f"dV long columns cfg{cid}/{div}")
    for name, g, w in (("dK", gk, wk), ("dV", gv, wv)):
        rl = rel_l2(g, w)
        assert rl is None or rl <= GRAD_REL_L2, (name, rl)


@pytest.mark.parametrize("cid", [3, 5])
def test_full_size_dkdv_long_columns_banded(cid):
    """Full size (512 / 1024 query tiles): dO is zero outside four row bands -- the
    256 rows before each of three events and the last 256 rows -- so the exact dK/dV
    of any key sums over those rows only, while the kernel still walks every tile of
    the column. Checked element by element on long columns of trace 0, kv group 0
    and of the last trace's last group."""
    cfg = W.CONFIGS[cid]
    B, N, Hq, Hkv = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv
    G = Hq // Hkv
    ev = W.make_event_log(cfg)
    q, k, v, do = W.replay_tensors_device(cfg)
    gm = kvs.kvs_build_tile_mask(events_dev(ev), B, N)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, o_lo = kvs.kvs_masked_attn_fwd(q, k, v, gm, cfg.scale, status=status)
    band = torch.zeros((B, N), dtype=torch.bool, device="cuda")
    for b in range(B):
        evb = ev[ev[:, 0] == b]
        for e in {0, len(evb) // 2, len(evb) - 1}:
            tau = int(evb[e, 1])
            band[b, max(0, tau - 256): tau] = True
        band[b, N - 256:] = True
    do_b = do * band[:, :, None, None].to(do.dtype)
    dq, dk, dv = kvs.kvs_masked_attn_bwd(q, k, v, o, do_b, lse, gm, cfg.scale, status=status, o_lo=o_lo)
    torch.cuda.synchronize()
    assert status.item() == 0
    kap = oracle.kappa(ev, B, N)
    rng = np.random.default_rng(50 + cid)
    for b, kvh in ((0, 0), (B - 1, Hkv - 1)):
        evb = ev[ev[:, 0] == b]
        rows = np.flatnonzero(band[b].cpu().numpy())
        hs = slice(kvh * G, (kvh + 1) * G)
        kk, vv = host(k[b, :, kvh]), host(v[b, :, kvh])
        qg = host(q[b, :, hs].transpose(0, 1))
        dg = host(do_b[b, :, hs].transpose(0, 1))
        og, lg = _group_fwd_rows(qg, kk, vv, kap[b], cfg.scale, rows)
        cols = _long_columns(evb, N, cfg.prompt, rng)
        wk, wv = oracle.dkdv_cols_fwd(qg, kk, vv, dg, og, lg, kap[b], cfg.scale, cols)
        gk, gv = host(dk[b, cols, kvh]), host(dv[b, cols, kvh])
        assert_close(gk, wk, BF16_TOL, f"dK banded full cfg{cid} b{b}")
        assert_close(gv, wv, BF16_TOL, f"dV banded full cfg{cid} b{b}")
        # only a few hundred rows contribute, so the gradients are small: the relative
        # L2 bound is the meaningful one here
        for name, g_, w_ in (("dK", gk, wk), ("dV", gv, wv)):
            rl = rel_l2(g_, w_)
            assert rl is not None and rl <= GRAD_REL_L2, (name, rl)


def _bf16_round(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("hq,hkv,with_events", [(4, 2, False), (4, 2, True), (2, 2, False)])
def test_forward_running_max_rescale(hq, hkv, with_events):
    """Keys scaled up tile by tile so that each key tile's row maximum exceeds the
    running maximum by far more than the lazy-rescale threshold: the forward's O
    rescale (and, for an even group size, the two-half hand-over of P that
    follows it) runs on every tile. Compared with the oracle as usual."""
    N = 1024
    cfg = W.TraceConfig(cid=95, name="rescale", batch=1, n_tokens=N, hq=hq, hkv=hkv, d=128,
                        theta=1e4, block_size=1, dtype="bf16", prompt=0)
    q, k, v, do = W.replay_tensors(cfg)
    f = (1.0 + 4.0 * (np.arange(N) // 128)).reshape(1, N, 1, 1)
    k = _bf16_round(k * f)
    ev = (W.random_event_log(np.random.default_rng(11), 1, N, 4, unit=1, max_span=N // 4) if with_events
          else np.zeros((0, 4), dtype=np.int64))
    _check_full(cfg, ev, q, k, v, do, BF16_TOL, bwd=False)
