"""The re-prefill comparator's host side: the segments it builds and Fig. 3's
count of re-processed tokens ("KV-streams for Efficient Compaction in Agentic
Reinforcement Learning", Fig. 3), checked against the trace generator's summary
policy and against the oracle's re-prefill simulator."""
import numpy as np
import pytest

import oracle
from eviction_masked_attention_b200 import reprefill as R
from eviction_masked_attention_b200 import workloads as W


@pytest.mark.parametrize("div", [1, 4, 16])
def test_fig3_count_matches_summary_schedule(div):
    cfg = W.replace(W.scaled(W.CONFIGS[3], div), batch=1)
    ev = W.make_event_log(cfg)
    segs = R.schedule(ev[:, 1:4], cfg.n_tokens)
    kept = cfg.prompt + cfg.summary + cfg.overlap
    n_ev, extra = R.fig3_count(cfg.n_tokens, cfg.budget, kept)
    assert len(segs) == len(ev) + 1 == n_ev + 1
    assert R.reprocessed(segs) == extra == n_ev * kept
    # the closed form N/(B - kept) brackets the event count
    f = R.fig3_factor(cfg.n_tokens, cfg.budget, kept)
    assert n_ev <= f + 1 and n_ev >= f - cfg.budget / (cfg.budget - kept)


def test_segments_cover_the_trace_once_and_keep_order():
    cfg = W.replace(W.scaled(W.CONFIGS[5], 16), batch=1)
    ev = W.make_event_log(cfg)
    segs = R.schedule(ev[:, 1:4], cfg.n_tokens)
    new = np.concatenate([s.new for s in segs])
    assert np.array_equal(new, np.arange(cfg.n_tokens))
    kap = oracle.kappa(ev, 1, cfg.n_tokens)[0]
    for s in segs[1:]:
        t0 = s.new[0]
        # retained = exactly the tokens before t0 that no event up to t0 removed, ascending
        assert np.array_equal(s.retained, np.flatnonzero(kap[:t0] > t0))


def test_schedule_agrees_with_oracle_reprefill_position_count():
    """The oracle's re-prefill simulator renumbers positions; its final live count
    equals the last segment's retained + new tokens."""
    cfg = W.replace(W.scaled(W.CONFIGS[1], 8), batch=1)
    ev = W.make_event_log(cfg)
    N = cfg.n_tokens
    toy = oracle.Toy(L=1, Dm=8, Hq=2, Hkv=1, d=4, theta=cfg.theta, seed=1)
    rc, *_, ntok = toy.generate(np.zeros((N, 8)), ev[:, 1:4], 16, pool=N // 16 + 8, reprefill=True)
    assert rc == 0
    segs = R.schedule(ev[:, 1:4], N)
    assert ntok == len(segs[-1].retained) + len(segs[-1].new)
