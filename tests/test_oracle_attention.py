"""Pins for the oracle's masked attention forward/backward and paged decode (CPU only).

Anchors: torch's fp64 scaled-dot-product attention with an explicit boolean
mask built event by event (a library routine, independent of the oracle's
kill-time formulation), causal attention when there are no events, central
finite differences of the backward, and torch autograd.
"""
import numpy as np
import pytest
import torch

import oracle
from eviction_masked_attention_b200 import workloads as W
from conftest import dense_mask_eventwise


def _sdpa(q, k, v, mask, scale):
    # q [Hq,N,d], k/v [Hkv,N,d] -> expand kv heads for GQA (kv = h // G)
    G = q.shape[0] // k.shape[0]
    k = k.repeat_interleave(G, 0)
    v = v.repeat_interleave(G, 0)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)


def _case(seed, N=200, Hq=4, Hkv=2, d=16, n_ev=5, B=2):
    rng = np.random.default_rng(seed)
    ev = W.random_event_log(rng, B, N, n_ev, unit=1, max_span=N // 3)
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    do = rng.standard_normal((B, N, Hq, d))
    return ev, q, k, v, do


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fwd_matches_torch_sdpa_with_eventwise_mask(seed):
    ev, q, k, v, _ = _case(seed)
    B, N, Hq, d = q.shape
    scale = 1 / np.sqrt(d)
    kap = oracle.kappa(ev, B, N)
    o, lse = oracle.attn_fwd(q, k, v, kap, scale)
    for b in range(B):
        mask = torch.from_numpy(dense_mask_eventwise(ev, b, N))
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)
        kt = torch.from_numpy(k[b]).permute(1, 0, 2)
        vt = torch.from_numpy(v[b]).permute(1, 0, 2)
        ref = _sdpa(qt, kt, vt, mask, scale).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(o[b], ref, rtol=0, atol=1e-12)
        G = Hq // kt.shape[0]
        s = torch.einsum("hnd,hmd->hnm", qt, kt.repeat_interleave(G, 0)) * scale
        s = s.masked_fill(~mask, float("-inf"))
        np.testing.assert_allclose(lse[b], torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_no_events_equals_causal():
    _, q, k, v, _ = _case(7, n_ev=0)
    B, N, Hq, d = q.shape
    kap = oracle.kappa(np.zeros((0, 4), np.int32), B, N)
    o, _ = oracle.attn_fwd(q, k, v, kap, 1 / np.sqrt(d))
    G = Hq // k.shape[2]
    for b in range(B):
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)
        kt = torch.from_numpy(k[b]).permute(1, 0, 2).repeat_interleave(G, 0)
        vt = torch.from_numpy(v[b]).permute(1, 0, 2).repeat_interleave(G, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        np.testing.assert_allclose(o[b], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 3])
def test_bwd_matches_torch_autograd(seed):
    ev, q, k, v, do = _case(seed, N=150)
    B, N, Hq, d = q.shape
    scale = 1 / np.sqrt(d)
    kap = oracle.kappa(ev, B, N)
    o, lse, dq, dk, dv = oracle.attn_bwd(q, k, v, do, kap, scale)
    for b in range(B):
        mask = torch.from_numpy(dense_mask_eventwise(ev, b, N))
        qt = torch.from_numpy(q[b]).permute(1, 0, 2).requires_grad_()
        kt = torch.from_numpy(k[b]).permute(1, 0, 2).requires_grad_()
        vt = torch.from_numpy(v[b]).permute(1, 0, 2).requires_grad_()
        out = _sdpa(qt, kt, vt, mask, scale)
        out.backward(torch.from_numpy(do[b]).permute(1, 0, 2))
        np.testing.assert_allclose(o[b], out.detach().permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(dq[b], qt.grad.permute(1, 0, 2).numpy(), atol=1e-11, rtol=0)
        np.testing.assert_allclose(dk[b], kt.grad.permute(1, 0, 2).numpy(), atol=1e-11, rtol=0)
        np.testing.assert_allclose(dv[b], vt.grad.permute(1, 0, 2).numpy(), atol=1e-11, rtol=0)


def test_bwd_finite_differences():
    # L = sum(O * dO); central differences in fp64 on a tiny case (N = 48, d = 8)
    ev, q, k, v, do = _case(11, N=48, Hq=2, Hkv=1, d=8, n_ev=3, B=1)
    N, d = q.shape[1], q.shape[3]
    scale = 1 / np.sqrt(d)
    kap = oracle.kappa(ev, 1, N)
    _, _, dq, dk, dv = oracle.attn_bwd(q, k, v, do, kap, scale)

    def loss(q_, k_, v_):
        o, _ = oracle.attn_fwd(q_, k_, v_, kap, scale)
        return float((o * do).sum())

    rng = np.random.default_rng(0)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            ap, am = dict(args), dict(args)
            ap[name], am[name] = xp, xm
            fd = (loss(ap["q"], ap["k"], ap["v"]) - loss(am["q"], am["k"], am["v"])) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_sampled_rows_and_cols_agree_with_full_bwd():
    ev, q, k, v, do = _case(5, N=180, Hq=4, Hkv=2, d=16, B=1)
    N, Hq, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    scale = 1 / np.sqrt(d)
    kap = oracle.kappa(ev, 1, N)
    _, _, dq, dk, dv = oracle.attn_bwd(q, k, v, do, kap, scale)
    for kvh in range(k.shape[2]):
        qg = np.transpose(q[0, :, kvh * G:(kvh + 1) * G], (1, 0, 2))
        dog = np.transpose(do[0, :, kvh * G:(kvh + 1) * G], (1, 0, 2))
        g_rows = np.array([0, 1, G - 1, 0]); t_rows = np.array([0, 77, 179, 130])
        got = oracle.dq_rows(qg, k[0, :, kvh], v[0, :, kvh], dog, kap[0], scale, g_rows, t_rows)
        want = np.stack([dq[0, t, kvh * G + g] for g, t in zip(g_rows, t_rows)])
        np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)
        cols = np.array([0, 5, 100, 179])
        gk, gv = oracle.dkdv_cols(qg, k[0, :, kvh], v[0, :, kvh], dog, kap[0], scale, cols)
        np.testing.assert_allclose(gk, dk[0, cols, kvh], atol=1e-12, rtol=0)
        np.testing.assert_allclose(gv, dv[0, cols, kvh], atol=1e-12, rtol=0)


def _autograd_dkdv(q, k, v, do, ev, b, scale):
    """dK, dV of one trace from torch autograd through fp64 SDPA with the event-wise mask."""
    N = q.shape[1]
    mask = torch.from_numpy(dense_mask_eventwise(ev, b, N))
    qt = torch.from_numpy(np.transpose(q[b], (1, 0, 2))).requires_grad_(True)
    kt = torch.from_numpy(np.transpose(k[b], (1, 0, 2))).requires_grad_(True)
    vt = torch.from_numpy(np.transpose(v[b], (1, 0, 2))).requires_grad_(True)
    out = _sdpa(qt, kt, vt, mask, scale)
    out.backward(torch.from_numpy(np.transpose(do[b], (1, 0, 2))))
    return kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("banded", [False, True])
def test_dkdv_cols_from_forward_rows(banded):
    """dK/dV by column from the forward's per-row O and LSE equals autograd; with dO
    zero outside a few row bands, rows outside them may carry O = 0, LSE = +inf."""
    ev, q, k, v, do = _case(7, N=260, Hq=6, Hkv=2, d=16, B=1)
    N, Hq, d = q.shape[1], q.shape[2], q.shape[3]
    Hkv = k.shape[2]
    G = Hq // Hkv
    scale = 1 / np.sqrt(d)
    rows = np.arange(N)
    if banded:
        band = ((rows >= 40) & (rows < 70)) | (rows >= 230)
        do = do * band[None, :, None, None]
    kap = oracle.kappa(ev, 1, N)
    gk_all, gv_all = _autograd_dkdv(q, k, v, do, ev, 0, scale)
    cols = np.array([0, 1, 39, 41, 100, 200, 259])
    for kvh in range(Hkv):
        hs = slice(kvh * G, (kvh + 1) * G)
        qg = np.transpose(q[0, :, hs], (1, 0, 2)); dog = np.transpose(do[0, :, hs], (1, 0, 2))
        og, lg = np.empty((G, N, d)), np.empty((G, N))
        for g in range(G):
            og[g], lg[g] = oracle.attn_rows(qg[g], rows, k[0, :, kvh], v[0, :, kvh], kap[0], scale)
        if banded:
            og[:, ~band] = 0.0
            lg[:, ~band] = np.inf
        gk, gv = oracle.dkdv_cols_fwd(qg, k[0, :, kvh], v[0, :, kvh], dog, og, lg, kap[0], scale, cols)
        np.testing.assert_allclose(gk, gk_all[kvh, cols], atol=1e-11, rtol=0)
        np.testing.assert_allclose(gv, gv_all[kvh, cols], atol=1e-11, rtol=0)


def test_dk_sums_to_zero_per_group():
    # sum_j dS_tj = 0 for every query row, so sum_j dK_j = 0 (a property at any size)
    ev, q, k, v, do = _case(9, N=160)
    kap = oracle.kappa(ev, q.shape[0], q.shape[1])
    _, _, dq, dk, dv = oracle.attn_bwd(q, k, v, do, kap, 1 / np.sqrt(q.shape[3]))
    assert np.abs(dk.sum(axis=1)).max() < 1e-10


@pytest.mark.parametrize("bs", [1, 16])
def test_paged_decode_equals_replay_row(bs):
    # walking a compacted block table == the replay row of the same logical position
    rng = np.random.default_rng(bs)
    N, Hq, Hkv, d = 256, 4, 2, 16
    ev = np.array([[0, 96, 32, 64], [0, 160, 80, 128], [0, 224, 0, 16]], np.int32)
    kap = oracle.kappa(ev, 1, N)
    k = rng.standard_normal((N, Hkv, d)); v = rng.standard_normal((N, Hkv, d))
    q = rng.standard_normal((Hq, d))
    t = 240
    live = [j for j in range(t + 1) if kap[0, j] > t]
    # physical pool: each live block goes to a random block id
    nblk = (len(live) + bs - 1) // bs
    pool = nblk + 5
    ids = rng.permutation(pool)[:nblk]
    kc = np.zeros((pool, Hkv, bs, d)); vc = np.zeros((pool, Hkv, bs, d))
    for i, j in enumerate(live):
        kc[ids[i // bs], :, i % bs] = k[j]
        vc[ids[i // bs], :, i % bs] = v[j]
    bt = ids[None, :].astype(np.int32)
    o = oracle.paged_decode(q[None], kc, vc, bt, np.array([len(live)]), bs, 1 / np.sqrt(d))
    G = Hq // Hkv
    for h in range(Hq):
        want, _ = oracle.attn_rows(q[h][None], [t], k[:, h // G], v[:, h // G], kap[0], 1 / np.sqrt(d))
        assert np.array_equal(o[0, h], want[0])
