"""GPU parity of generation with in-place compaction, token by token.

The generation side of the method ("KV-streams: speeding up agentic RL by
operating on the KV cache directly", first and second fix): each new token's
query and key are rotated at their logical position (the position count is
never reset), the key and value go to a slot of a paged cache, attention runs
over the cache's block table; at a compaction event whole blocks leave the
cache and the table is packed. Driven through the library one token at a
time, every decoded row must equal the replay row of the same position (the
oracle's, and on the 1-token-block trace also the GPU forward's), and the
block table after every event must equal the oracle's generation simulator.

The host-side bookkeeping (free list, next block, counts) is the caller's part
of each step; it lives in the helper class below.
"""
from collections import deque

import numpy as np
import pytest
import torch

import oracle
import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import workloads as W
from gpu_util import BF16_TOL, F32_ROUND, F32_TOL, assert_close, dev, events_dev, host

pytestmark = pytest.mark.gpu


class PagedSequence:
    """One sequence's paged cache and the caller's bookkeeping around the library
    calls: a FIFO free list of pool blocks (freed blocks return to its tail in table
    order), a new block whenever the tail block is full, num_tokens that falls at a
    compaction, and a logical position that only grows."""

    def __init__(self, pool, max_blocks, bs, Hkv, d, dtype, theta):
        self.bs, self.pool, self.theta = bs, pool, theta
        self.free = deque(range(pool))
        self.kc = torch.zeros((pool, Hkv, bs, d), dtype=dtype, device="cuda")
        self.vc = torch.zeros_like(self.kc)
        self.bt = torch.full((1, max_blocks), -1, dtype=torch.int32, device="cuda")
        self.bl = torch.full((1, max_blocks), -1, dtype=torch.int32, device="cuda")
        self.nb = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.nt = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.freed = torch.full((1, max_blocks), -1, dtype=torch.int32, device="cuda")
        self.n_freed = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.n_blocks = 0
        self.n_tokens = 0
        self.table = []  # host copy of the live block ids

    def compact(self, ev_rows):
        kvs.kvs_compact_block_table(self.bt, self.bl, self.nb, self.nt, self.bs, self.pool, events_dev(ev_rows),
                                    freed=self.freed, n_freed=self.n_freed, status=self.status)
        nf = int(self.n_freed.item())
        self.free.extend(self.freed[0, :nf].tolist())
        self.n_blocks, self.n_tokens = int(self.nb.item()), int(self.nt.item())
        self.table = self.bt[0, :self.n_blocks].tolist()

    def append(self, k_raw, v_raw, lpos):
        """Rotate the new key at its logical position and write key and value to the
        next slot (a new block when the tail block is full)."""
        if self.n_tokens % self.bs == 0:
            blk = self.free.popleft()
            self.table.append(blk)
            self.bt[0, self.n_blocks] = blk
            self.bl[0, self.n_blocks] = lpos
            self.n_blocks += 1
            self.nb.fill_(self.n_blocks)
        slot = self.table[-1] * self.bs + self.n_tokens % self.bs
        kvs.kvs_rope_logical(k_raw, self.lp(lpos), self.theta, out=self.kc,
                             out_slot=torch.tensor([slot], dtype=torch.int64, device="cuda"),
                             block_size=self.bs, v=v_raw, v_out=self.vc, status=self.status)
        self.n_tokens += 1
        self.nt.fill_(self.n_tokens)

    @staticmethod
    def lp(pos):
        return torch.tensor([pos], dtype=torch.int32, device="cuda")

    def decode(self, q_raw, lpos, scale, out):
        qr = kvs.kvs_rope_logical(q_raw, self.lp(lpos), self.theta, status=self.status)
        kvs.kvs_paged_decode_attn(qr, self.kc, self.vc, self.bt, self.nt, self.bs, scale, out=out,
                                  status=self.status)


def _generate(cfg, ev, q, k, v, check_tables=True):
    """Walk the trace token by token through the library; returns decode rows [N, Hq, d]."""
    N, Hq, Hkv, d, bs = cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d, cfg.block_size
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    pool = (N + bs - 1) // bs + 8
    seq = PagedSequence(pool, (N + bs - 1) // bs + 1, bs, Hkv, d, tdt, cfg.theta)
    qd, kd, vd = dev(q[0], tdt), dev(k[0], tdt), dev(v[0], tdt)
    out = torch.empty((N, 1, Hq, d), dtype=tdt, device="cuda")
    by_tau = {}
    for row in ev:
        by_tau.setdefault(int(row[1]), []).append(row)
    toy = oracle.Toy(L=1, Dm=4, Hq=1, Hkv=1, d=2, theta=cfg.theta, seed=0)
    checked = 0
    for t in range(N):
        if t in by_tau:
            seq.compact(np.asarray(by_tau[t], np.int32))
        seq.append(kd[t:t + 1], vd[t:t + 1], t)
        if check_tables and t in by_tau:
            # the oracle's simulator after the same events and the append of token t
            rc, _, _, tab, lps, ntok = toy.generate(np.zeros((t + 1, 4)), ev[ev[:, 1] <= t][:, 1:4], bs, pool)
            assert rc == 0
            assert seq.n_tokens == ntok and seq.n_blocks == len(tab)
            assert np.array_equal(seq.bt[0, :seq.n_blocks].cpu().numpy(), tab), t
            assert np.array_equal(seq.bl[0, :seq.n_blocks].cpu().numpy(), lps), t
            checked += 1
        seq.decode(qd[t:t + 1], t, cfg.scale, out[t])
    torch.cuda.synchronize()
    assert seq.status.item() == 0, kvs.status_str(seq.status.item())
    if check_tables:
        assert checked == len(by_tau)
    return out[:, 0], seq


def _oracle_rows(cfg, ev, q, k, v):
    N, Hq, Hkv = cfg.n_tokens, cfg.hq, cfg.hkv
    G = Hq // Hkv
    lp = np.arange(N, dtype=np.int32)
    kap = oracle.kappa(ev, 1, N)
    qo = oracle.rope(q[0].astype(np.float64), lp, cfg.theta)
    ko = oracle.rope(k[0].astype(np.float64), lp, cfg.theta)
    want = np.empty((N, Hq, cfg.d))
    for h in range(Hq):
        want[:, h], _ = oracle.attn_rows(qo[:, h], lp, ko[:, h // G], v[0, :, h // G], kap[0], cfg.scale)
    return want


def test_generation_tiny_fp32_token_by_token():
    """The tiny fp32 trace (2048 tokens, 16-token blocks, two compaction events):
    every decoded token against the oracle's replay row, tables after each event
    against the oracle's generation simulator."""
    cfg = W.CONFIGS[1]
    ev = W.make_event_log(cfg)
    assert len(ev) >= 2
    q, k, v, _ = W.replay_tensors(cfg)
    got, seq = _generate(cfg, ev, q, k, v)
    want = _oracle_rows(cfg, ev, q, k, v)
    assert_close(host(got), want, F32_TOL, "generation fp32 rows")
    # the final cache holds exactly the never-evicted positions
    kap = oracle.kappa(ev, 1, cfg.n_tokens)
    assert seq.n_tokens == int((kap[0] == oracle.INT32_MAX).sum())


def test_generation_bs1_bf16_token_by_token():
    """A 1-token-block trace at 1/16 length (8192 tokens, unpadded turns, events at
    arbitrary offsets), G = 8: every decoded token against the oracle's replay row
    and against the GPU forward's replay row of the same position."""
    cfg = W.replace(W.scaled(W.CONFIGS[5], 16), batch=1, hq=16, hkv=2)
    ev = W.make_event_log(cfg)
    assert len(ev) >= 5
    q, k, v, _ = W.replay_tensors(cfg)
    got, _ = _generate(cfg, ev, q, k, v)
    want = _oracle_rows(cfg, ev, q, k, v)
    assert_close(host(got), want, BF16_TOL, "generation bs1 rows")
    # the GPU replay of the same trace: RoPE at positions 0..N-1, masked forward
    N = cfg.n_tokens
    lp = dev(np.arange(N, dtype=np.int32))
    qr = kvs.kvs_rope_logical(dev(q[0], torch.bfloat16), lp, cfg.theta)[None].contiguous()
    kr = kvs.kvs_rope_logical(dev(k[0], torch.bfloat16), lp, cfg.theta)[None].contiguous()
    gm = kvs.kvs_build_tile_mask(events_dev(ev), 1, N)
    o, _, _ = kvs.kvs_masked_attn_fwd(qr, kr, dev(v, torch.bfloat16), gm, cfg.scale)
    assert_close(host(got), host(o[0]), BF16_TOL, "generation vs GPU replay")
