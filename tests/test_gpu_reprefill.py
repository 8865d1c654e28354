"""GPU parity of the re-prefill comparator ("KV-streams for Efficient Compaction
in Agentic Reinforcement Learning", Fig. 2(A)): the library's kernels run on the
re-prefill schedule -- each segment's retained tokens renumbered from position 0
and processed again, a causal attention over the segment -- and must reproduce
the oracle's re-prefill simulator token by token; on the same trace the
KV-streams replay agrees with it before the first event and differs after."""
import numpy as np
import pytest
import torch

import oracle
import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import reprefill as R
from eviction_masked_attention_b200 import workloads as W
from gpu_util import F32_TOL, assert_close, dev, events_dev, host

pytestmark = pytest.mark.gpu


def _segment_attention(q_raw, k_raw, v_raw, seg, theta, scale):
    """Causal attention over one segment at its renumbered positions (fp32)."""
    tok = seg.tokens
    n = len(tok)
    lp = dev(seg.positions)
    q = kvs.kvs_rope_logical(dev(q_raw[tok], torch.float32), lp, theta)[None].contiguous()
    k = kvs.kvs_rope_logical(dev(k_raw[tok], torch.float32), lp, theta)[None].contiguous()
    v = dev(v_raw[tok], torch.float32)[None].contiguous()
    gm = kvs.kvs_build_tile_mask(events_dev(np.zeros((0, 4), np.int32)), 1, n)
    o, _, _ = kvs.kvs_masked_attn_fwd(q, k, v, gm, scale)
    return host(o[0])


def test_reprefill_schedule_matches_oracle_simulator():
    cfg = W.replace(W.scaled(W.CONFIGS[1], 4), batch=1)
    ev = W.make_event_log(cfg)
    assert len(ev) >= 1
    N, Dm, Hq, Hkv, d = cfg.n_tokens, 16, 4, 1, 64
    toy = oracle.Toy(L=1, Dm=Dm, Hq=Hq, Hkv=Hkv, d=d, theta=cfg.theta, seed=9)
    x0 = np.random.default_rng(9).standard_normal((N, Dm))
    rc, _, attn, *_ = toy.generate(x0, ev[:, 1:4], 16, pool=N // 16 + 8, reprefill=True)
    assert rc == 0
    q_raw = (x0 @ toy.Wq[0]).reshape(N, Hq, d)
    k_raw = (x0 @ toy.Wk[0]).reshape(N, Hkv, d)
    v_raw = (x0 @ toy.Wv[0]).reshape(N, Hkv, d)
    got = np.empty((N, Hq, d))
    for seg in R.schedule(ev[:, 1:4], N):
        o = _segment_attention(q_raw, k_raw, v_raw, seg, cfg.theta, toy.scale)
        got[seg.new] = o[len(seg.retained):]
    assert_close(got, attn[:, 0].reshape(N, Hq, d), F32_TOL, "re-prefill rows")
    # KV-streams replay of the same trace: equal before the first event, different after
    lp = dev(np.arange(N, dtype=np.int32))
    q = kvs.kvs_rope_logical(dev(q_raw, torch.float32), lp, cfg.theta)[None].contiguous()
    k = kvs.kvs_rope_logical(dev(k_raw, torch.float32), lp, cfg.theta)[None].contiguous()
    gm = kvs.kvs_build_tile_mask(events_dev(ev), 1, N)
    o, _, _ = kvs.kvs_masked_attn_fwd(q, k, dev(v_raw, torch.float32)[None].contiguous(), gm, toy.scale)
    kv = host(o[0])
    t0 = int(ev[0, 1])
    assert np.abs(kv[:t0] - got[:t0]).max() <= 1e-5
    diff = np.abs(kv[t0:] - got[t0:]).max(axis=(1, 2))
    assert (diff > 1e-4).mean() > 0.9 and diff.max() > 1e-2
