"""Pins for the oracle's kill-time and tile-mask functions (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
from eviction_masked_attention_b200 import workloads as W
from conftest import dense_mask_eventwise

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_small_mask():
    g = json.load(open(os.path.join(GOLD, "mask_small.json")))
    kap = oracle.kappa(np.array(g["events"]), g["B"], g["N"])
    for j, val in g["kappa_samples"].items():
        assert kap[0, int(j)] == (oracle.INT32_MAX if val is None else val)
    m = oracle.tile_mask(kap)
    assert m["cls"][0].tolist() == g["classes"]
    assert oracle.visible_pairs(kap) == g["visible_pairs"]
    e = m["row_ptr"][1]  # first non-empty tile of row 1 is (1, 0)
    assert m["row_col"][e] == 0
    bits = m["bits"][m["row_pidx"][e]]
    assert (bits[:72] == np.array(g["tile_1_0_bits"]["rows_0_71"], np.uint32)).all()
    assert (bits[72:] == np.array(g["tile_1_0_bits"]["rows_72_127"], np.uint32)).all()


def _unpack(bits):
    """[128][4] words -> [128][128] booleans (bit c%32 of word c/32)."""
    w = bits.astype(np.uint64)
    cols = np.arange(128)
    return ((w[:, cols // 32] >> (cols % 32).astype(np.uint64)) & 1).astype(bool)


@pytest.mark.parametrize("N,seed", [(384, 0), (300, 1), (517, 2), (128, 3), (1000, 4)])
def test_mask_against_eventwise_dense(N, seed):
    rng = np.random.default_rng(seed)
    B = 2
    ev = W.random_event_log(rng, B, N, 9, unit=1, max_span=N // 3)
    kap = oracle.kappa(ev, B, N)
    m = oracle.tile_mask(kap)
    T = m["T"]
    for b in range(B):
        dense = dense_mask_eventwise(ev, b, N)
        pad = np.zeros((T * 128, T * 128), dtype=bool)
        pad[:N, :N] = dense
        for qi in range(T):
            lo, hi = m["row_ptr"][b * T + qi], m["row_ptr"][b * T + qi + 1]
            listed = dict(zip(m["row_col"][lo:hi].tolist(), m["row_pidx"][lo:hi].tolist()))
            for kj in range(T):
                tile = pad[qi * 128:(qi + 1) * 128, kj * 128:(kj + 1) * 128]
                c = m["cls"][b, qi, kj]
                if not tile.any():
                    assert c == oracle.EMPTY and kj not in listed
                elif tile.all():
                    assert c == oracle.FULL and listed[kj] == -1
                else:
                    assert c == oracle.PARTIAL
                    assert (_unpack(m["bits"][listed[kj]]) == tile).all()
        # pair count equals the dense count
        assert dense.sum() == sum(np.minimum(kap[b], N)[j] - j for j in range(N) if kap[b, j] > j)


def test_no_events_is_causal():
    N = 640
    kap = oracle.kappa(np.zeros((0, 4), np.int32), 1, N)
    m = oracle.tile_mask(kap)
    T = m["T"]
    want = np.where(np.tri(T, k=-1, dtype=bool), oracle.FULL, oracle.EMPTY)
    np.fill_diagonal(want, oracle.PARTIAL)
    assert (m["cls"][0] == want).all()
    tri = np.tril(np.ones((128, 128), bool))
    for p in range(m["n_partial"]):
        assert (_unpack(m["bits"][p]) == tri).all()
    assert oracle.visible_pairs(kap) == N * (N + 1) // 2


def test_csr_row_and_col_agree():
    cfg = W.scaled(W.CONFIGS[5], 16)
    ev = W.make_event_log(cfg)
    kap = oracle.kappa(ev, cfg.batch, cfg.n_tokens)
    m = oracle.tile_mask(kap)
    T, B = m["T"], cfg.batch
    rows = set()
    for b in range(B):
        for qi in range(T):
            for e in range(m["row_ptr"][b * T + qi], m["row_ptr"][b * T + qi + 1]):
                rows.add((b, qi, int(m["row_col"][e]), int(m["row_pidx"][e])))
    cols = set()
    for b in range(B):
        for kj in range(T):
            for e in range(m["col_ptr"][b * T + kj], m["col_ptr"][b * T + kj + 1]):
                cols.add((b, int(m["col_row"][e]), kj, int(m["col_pidx"][e])))
    assert rows == cols
    pids = sorted(p for (_, _, _, p) in rows if p >= 0)
    assert pids == list(range(m["n_partial"]))
    # every diagonal tile is non-empty: a query always sees itself
    for b in range(B):
        assert all(m["cls"][b, i, i] != oracle.EMPTY for i in range(T))


def test_config_event_counts():
    # event counts the configs state or imply (cfg1 ~2, cfg2 ~6, cfg3 4, cfg5 10..20)
    for cid in (1, 2, 3, 5):
        cfg = W.CONFIGS[cid]
        ev = W.make_event_log(cfg)
        per = np.bincount(ev[:, 0], minlength=cfg.batch)
        lo, hi = cfg.expect_events
        assert (per >= lo).all() and (per <= hi).all(), (cid, per)
        # events never remove tokens that do not exist yet, and tau is non-decreasing
        assert (ev[:, 3] <= ev[:, 1]).all() and (ev[:, 2] < ev[:, 3]).all()
        if cfg.pad > 1:
            assert (ev[:, 2] % cfg.pad == 0).all() and (ev[:, 3] % cfg.pad == 0).all()
