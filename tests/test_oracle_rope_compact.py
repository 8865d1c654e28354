"""Pins for the oracle's rotary embedding and block-table compaction (CPU only)."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from eviction_masked_attention_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_rope_golden():
    g = json.load(open(os.path.join(GOLD, "rope_small.json")))
    for c in g["cases"]:
        x = np.array(c["x"], float).reshape(1, 1, g["d"])
        y = oracle.rope(x, [c["p"]], g["theta"])[0, 0]
        want = [eval(e, {"cos": math.cos, "sin": math.sin}) for e in c["expect"]]
        np.testing.assert_allclose(y, want, atol=1e-15, rtol=0)


@pytest.mark.parametrize("theta,d", [(1e4, 64), (5e5, 128)])
def test_rope_relative_offset_and_isometry(theta, d):
    # <R(p+c) q, R(p'+c) k> == <R(p) q, R(p') k>; |R(p) x| == |x|; R(-p) R(p) = I
    rng = np.random.default_rng(0)
    n = 64
    q = rng.standard_normal((n, 1, d)); k = rng.standard_normal((n, 1, d))
    p = rng.integers(0, 131072, n); pp = rng.integers(0, 131072, n); c = rng.integers(-5000, 5000, n)
    c = np.maximum(c, -np.minimum(p, pp))
    a = (oracle.rope(q, p, theta) * oracle.rope(k, pp, theta)).sum(-1)
    b = (oracle.rope(q, p + c, theta) * oracle.rope(k, pp + c, theta)).sum(-1)
    assert np.abs(a - b).max() < 1e-9
    y = oracle.rope(q, p, theta)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(oracle.rope(y, p, theta, inverse=True), q, atol=1e-12, rtol=0)
    # position 0 is the identity
    np.testing.assert_array_equal(oracle.rope(q, np.zeros(n, np.int32), theta), q)


def test_compact_golden():
    g = json.load(open(os.path.join(GOLD, "compact_small.json")))
    M = 8
    bt = np.full((1, M), -1, np.int32); bl = np.full((1, M), -1, np.int32)
    n = len(g["block_table"])
    bt[0, :n] = g["block_table"]; bl[0, :n] = g["block_lpos"]
    for c in g["cases"]:
        rc, t, l, nb, nt, fr, nf = oracle.compact(bt, bl, [n], [g["num_tokens"]], g["block_size"],
                                                  np.array(c["events"]))
        if c["status"] == "unaligned":
            assert rc == 2
            continue
        assert rc == 0
        k = nb[0]
        assert t[0, :k].tolist() == c["table"] and l[0, :k].tolist() == c["lpos"]
        assert nt[0] == c["num_tokens"] and fr[0, :nf[0]].tolist() == c["freed"]


@pytest.mark.parametrize("div", [16, 4])
def test_compact_invariants_paged_config(div):
    st = W.make_paged_state(W.CONFIGS[4], div=div)
    bs = st.block_size
    rc, t, l, nb, nt, fr, nf = oracle.compact(st.block_table, st.block_lpos, st.num_blocks,
                                              st.num_tokens, bs, st.events)
    assert rc == 0
    for b in range(st.block_table.shape[0]):
        old = st.block_table[b, :st.num_blocks[b]].tolist()
        new = t[b, :nb[b]].tolist()
        freed = fr[b, :nf[b]].tolist()
        assert sorted(old) == sorted(new + freed)            # conservation
        it = iter(old)
        assert all(x in it for x in new)                     # order preserved
        it = iter(old)
        assert all(x in it for x in freed)                   # freed in table order
        assert nt[b] == st.num_tokens[b] - bs * len(freed)
        rng_b = [(s, e) for (q, _, s, e) in st.events if q == b]
        for lp in l[b, :nb[b]]:                              # kept blocks are untouched by ranges
            assert all(lp + bs <= s or e <= lp for s, e in rng_b)
        lp_of = dict(zip(old, st.block_lpos[b, :st.num_blocks[b]].tolist()))
        for f in freed:                                      # freed blocks lie inside a range
            assert any(s <= lp_of[f] and lp_of[f] + bs <= e for s, e in rng_b)
        assert (t[b, nb[b]:st.num_blocks[b]] == -1).all()


def test_compact_tail_block_rule():
    # a partly filled tail block can not be evicted block-wise
    bt = np.array([[4, 5, 6]], np.int32); bl = np.array([[0, 16, 32]], np.int32)
    rc, *_ = oracle.compact(bt, bl, [3], [40], 16, np.array([[0, 48, 32, 48]]))
    assert rc == 2
    rc, t, l, nb, nt, fr, nf = oracle.compact(bt, bl, [3], [48], 16, np.array([[0, 48, 32, 48]]))
    assert rc == 0 and nb[0] == 2 and nt[0] == 32 and fr[0, 0] == 6
