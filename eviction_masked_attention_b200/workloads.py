"""Seeded synthetic workloads: multi-turn traces, the compaction-event log that a
compaction policy records while generating them, paged-cache states, and the
Q/K/V/dO tensors.

This module only produces inputs. It holds none of the attention, masking,
compaction or rotary arithmetic; both the CUDA path and the CPU oracle consume
what it returns.

Workload shapes follow the KV-streams description ("KV-streams: speeding up
agentic RL by operating on the KV cache directly", the thread's explanation of
16-token blocks, padding of completions to a multiple of 16, whole-turn
eviction and the recorded compaction events; and the paper listing "KV-streams
for Efficient Compaction in Agentic Reinforcement Learning", Fig. 2 and
Fig. 3 for the prompt / summary / overlap policies).

Event convention: an event ``(seq, tau, start, end)`` removes logical token
positions ``[start, end)`` of sequence ``seq`` at time ``tau``; ``tau`` is the
logical position of the first token generated after the compaction, so query
position ``t`` can no longer see the range exactly when ``tau <= t``.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import List, Optional, Tuple

import numpy as np

INT32_MAX = 2**31 - 1


@dataclass(frozen=True)
class TraceConfig:
    """One synthetic workload family.

    policy:
      ``"oldest"``  -- at a turn end, if live > budget, drop the oldest non-prompt
                       turns until live <= target.
      ``"recent"``  -- at a turn end, if live > budget, keep the prompt plus the
                       longest suffix of most recent whole turns whose total
                       length is <= overlap.
      ``"summary"`` -- no turns: when live reaches the budget, keep the prompt
                       and the last ``summary + overlap`` tokens before the event.
      ``"paged"``   -- one generation step on a paged cache (no replay trace).
    """

    cid: int
    name: str
    batch: int
    n_tokens: int
    hq: int
    hkv: int
    d: int
    theta: float
    block_size: int
    dtype: str
    prompt: int
    turn_min: int = 0
    turn_max: int = 0
    pad: int = 16
    budget: int = 0
    target: int = 0
    overlap: int = 0
    summary: int = 0
    policy: str = "oldest"
    # paged-generation parameters
    pool_blocks: int = 0
    live_min: int = 0
    live_max: int = 0
    max_lpos: int = 0
    events_min: int = 0
    events_max: int = 0
    range_min: int = 0
    range_max: int = 0
    expect_events: Tuple[int, int] = (0, 1 << 30)

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def seed(self, b: int) -> int:
        return 1000 * self.cid + b


CONFIGS = {
    1: TraceConfig(cid=1, name="tiny-fp32", batch=1, n_tokens=2048, hq=4, hkv=1, d=64,
                   theta=1e4, block_size=16, dtype="f32", prompt=128, turn_min=32,
                   turn_max=256, pad=16, budget=1024, target=512, policy="oldest",
                   expect_events=(1, 4)),
    2: TraceConfig(cid=2, name="replay-bf16", batch=8, n_tokens=32768, hq=32, hkv=8, d=128,
                   theta=5e5, block_size=16, dtype="bf16", prompt=1024, turn_min=256,
                   turn_max=2048, pad=16, budget=8192, overlap=4096, policy="recent",
                   expect_events=(3, 10)),
    3: TraceConfig(cid=3, name="summary-bf16", batch=4, n_tokens=65536, hq=32, hkv=8, d=128,
                   theta=5e5, block_size=16, dtype="bf16", prompt=1024, pad=16, budget=16384,
                   summary=512, overlap=2048, policy="summary", expect_events=(4, 4)),
    4: TraceConfig(cid=4, name="paged-decode-bf16", batch=64, n_tokens=0, hq=32, hkv=8, d=128,
                   theta=5e5, block_size=16, dtype="bf16", prompt=1024, pool_blocks=131072,
                   live_min=4096, live_max=32768, max_lpos=131072, events_min=1, events_max=8,
                   range_min=256, range_max=2048, policy="paged"),
    5: TraceConfig(cid=5, name="bs1-bf16", batch=2, n_tokens=131072, hq=64, hkv=8, d=128,
                   theta=5e5, block_size=1, dtype="bf16", prompt=1024, turn_min=64,
                   turn_max=4096, pad=1, budget=32768, target=28672, policy="oldest",
                   expect_events=(10, 20)),
}


def policy_mix(hq: int = 32, hkv: int = 8, div: int = 1) -> List[TraceConfig]:
    """One trace each of the compaction policies of the paper listing's Fig. 2(B) and
    Table 2 (prompt + summary + overlap, Markovian carry-over of the last tokens only,
    sliding window of recent turns, oldest turns out with unpadded 1-token granularity),
    at several (budget, summary, overlap) points and ragged lengths, for packed
    multi-trace replay. ``div`` shrinks them like :func:`scaled`."""
    base = dict(batch=1, hq=hq, hkv=hkv, d=128, theta=5e5, block_size=16, dtype="bf16", prompt=1024, pad=16)
    mix = [
        TraceConfig(cid=61, name="summary B16k s512 o2048", n_tokens=40960 + 77, budget=16384, summary=512,
                    overlap=2048, policy="summary", **base),
        TraceConfig(cid=62, name="summary B8k s256 o1024", n_tokens=24576 + 33, budget=8192, summary=256,
                    overlap=1024, policy="summary", **base),
        TraceConfig(cid=63, name="markovian B8k o2048", n_tokens=30720 + 101, budget=8192, summary=0,
                    overlap=2048, policy="summary", **base),
        TraceConfig(cid=64, name="recent turns o4096", n_tokens=20480 + 45, turn_min=256, turn_max=2048,
                    budget=8192, overlap=4096, policy="recent", **base),
        TraceConfig(cid=65, name="oldest turns bs1", n_tokens=36864 + 13, turn_min=64, turn_max=4096,
                    budget=16384, target=14336, policy="oldest",
                    **dict(base, block_size=1, pad=1)),
    ]
    if div > 1:
        mix = [replace(scaled(c, div), n_tokens=max(128, c.n_tokens // div)) for c in mix]
    return mix


def scaled(cfg: TraceConfig, div: int) -> TraceConfig:
    """A smaller twin of a trace config: the logical length, prompt, turn lengths,
    budgets and spans are divided by ``div`` (kept multiples of the padding unit),
    so the trace keeps the same structure at a size the oracle finishes quickly."""
    if div == 1:
        return cfg
    u = max(cfg.pad, 1)

    def sc(x, lo=1):
        if x == 0:
            return 0
        return max(lo, (x // div) // u * u)

    return replace(
        cfg,
        name=f"{cfg.name}/{div}",
        n_tokens=sc(cfg.n_tokens, 128),
        prompt=sc(cfg.prompt, u),
        turn_min=sc(cfg.turn_min, u),
        turn_max=sc(cfg.turn_max, u),
        budget=sc(cfg.budget, u),
        target=sc(cfg.target, u),
        overlap=sc(cfg.overlap, u),
        summary=sc(cfg.summary, u),
        expect_events=(0, 1 << 30),
    )


# --------------------------------------------------------------------------------------
# Traces and event logs
# --------------------------------------------------------------------------------------

def _pad_up(x: int, p: int) -> int:
    return (x + p - 1) // p * p


def make_turns(cfg: TraceConfig, rng: np.random.Generator) -> List[Tuple[int, int]]:
    """Turn spans ``[a, b)`` after the prompt; lengths uniform in
    [turn_min, turn_max] (inclusive), padded up to ``cfg.pad``; the last turn is
    cut at ``n_tokens``."""
    turns = []
    pos = cfg.prompt
    while pos < cfg.n_tokens:
        ln = int(rng.integers(cfg.turn_min, cfg.turn_max + 1))
        ln = _pad_up(ln, cfg.pad)
        end = min(pos + ln, cfg.n_tokens)
        turns.append((pos, end))
        pos = end
    return turns


def _merge(spans: List[Tuple[int, int]]) -> List[Tuple[int, int]]:
    out: List[Tuple[int, int]] = []
    for a, b in sorted(spans):
        if out and out[-1][1] == a:
            out[-1] = (out[-1][0], b)
        else:
            out.append((a, b))
    return out


def make_trace_events(cfg: TraceConfig, b: int) -> List[Tuple[int, int, int]]:
    """Compaction events ``(tau, start, end)`` of trace ``b`` under ``cfg``'s policy."""
    rng = np.random.default_rng(cfg.seed(b))
    events: List[Tuple[int, int, int]] = []
    if cfg.policy == "summary":
        keep = cfg.summary + cfg.overlap
        live_lo = cfg.prompt  # first live non-prompt position
        t = cfg.prompt
        while t < cfg.n_tokens:
            t += cfg.pad
            live = cfg.prompt + (t - live_lo)
            if live >= cfg.budget and t < cfg.n_tokens:
                cut = t - keep
                events.append((t, live_lo, cut))
                live_lo = cut
        return events

    turns = make_turns(cfg, rng)
    live_turns: List[Tuple[int, int]] = []
    for (a, e) in turns:
        live_turns.append((a, e))
        if e >= cfg.n_tokens:
            break
        live = cfg.prompt + sum(y - x for x, y in live_turns)
        if live <= cfg.budget:
            continue
        if cfg.policy == "oldest":
            evict = []
            while live > cfg.target and len(live_turns) > 1:
                x, y = live_turns.pop(0)
                evict.append((x, y))
                live -= y - x
        elif cfg.policy == "recent":
            keep, tot = [], 0
            for x, y in reversed(live_turns):
                if tot + (y - x) > cfg.overlap:
                    break
                keep.append((x, y))
                tot += y - x
            nkeep = len(keep)
            evict = live_turns[: len(live_turns) - nkeep]
            live_turns = live_turns[len(live_turns) - nkeep:]
        else:
            raise ValueError(cfg.policy)
        for (x, y) in _merge(evict):
            events.append((e, x, y))
    return events


def make_event_log(cfg: TraceConfig) -> np.ndarray:
    """The batch's event log as an ``int32[E, 4]`` array of ``(seq, tau, start, end)``
    rows sorted by (seq, tau, start)."""
    rows = []
    for b in range(cfg.batch):
        for (tau, s, e) in make_trace_events(cfg, b):
            rows.append((b, tau, s, e))
    rows.sort()
    if not rows:
        return np.zeros((0, 4), dtype=np.int32)
    return np.asarray(rows, dtype=np.int32)


def random_event_log(rng: np.random.Generator, batch: int, n_tokens: int, n_events: int,
                     unit: int = 1, max_span: Optional[int] = None) -> np.ndarray:
    """Unstructured events for edge-case tests: ranges may overlap or repeat,
    ``end <= tau``; spans are multiples of ``unit``."""
    rows = []
    max_span = max_span or n_tokens
    for _ in range(n_events):
        b = int(rng.integers(0, batch))
        tau = int(rng.integers(1, n_tokens + 1)) // unit * unit
        if tau == 0:
            continue
        s = int(rng.integers(0, tau)) // unit * unit
        e = min(tau, s + unit * int(rng.integers(1, max(2, max_span // unit + 1))))
        if e <= s:
            continue
        rows.append((b, tau, s, e))
    rows.sort()
    return np.asarray(rows, dtype=np.int32).reshape(-1, 4)


# --------------------------------------------------------------------------------------
# Paged-generation state (one decode step after a compaction)
# --------------------------------------------------------------------------------------

@dataclass
class PagedState:
    """A paged KV cache just before a compaction + decode step.

    ``block_table[b, i]`` is the physical block of the i-th live block of sequence
    ``b``; ``block_lpos[b, i]`` the logical position of its first token (a block
    holds ``block_size`` consecutive logical positions). ``num_tokens[b]`` counts
    live tokens, ``next_lpos[b]`` is the logical position the next generated token
    takes. ``events`` is this step's event log (``tau = next_lpos``). ``new_block``
    is the physical block the next token goes to when it opens a new block.
    """

    block_size: int
    pool_blocks: int
    max_blocks: int
    block_table: np.ndarray
    block_lpos: np.ndarray
    num_blocks: np.ndarray
    num_tokens: np.ndarray
    next_lpos: np.ndarray
    events: np.ndarray
    new_block: np.ndarray
    meta: dict = field(default_factory=dict)


def make_paged_state(cfg: TraceConfig, div: int = 1) -> PagedState:
    """Sequence lengths, historic eviction gaps, physical block placement and this
    step's 1..8 block-aligned eviction ranges, all from ``cfg.seed``.

    ``div`` shrinks lengths, pool and range sizes for quick tests."""
    bs = cfg.block_size
    rng = np.random.default_rng(cfg.seed(0))
    pool = cfg.pool_blocks // div
    live_min, live_max = cfg.live_min // div, cfg.live_max // div
    max_lpos = cfg.max_lpos // div
    prompt = max(bs, cfg.prompt // div // bs * bs)
    rmin, rmax = max(bs, cfg.range_min // div), max(bs, cfg.range_max // div)
    max_blocks = live_max // bs + 1
    B = cfg.batch
    perm = rng.permutation(pool).astype(np.int32)
    bt = np.full((B, max_blocks), -1, dtype=np.int32)
    bl = np.full((B, max_blocks), -1, dtype=np.int32)
    nb = np.zeros(B, dtype=np.int32)
    nt = np.zeros(B, dtype=np.int32)
    nl = np.zeros(B, dtype=np.int32)
    new_block = np.zeros(B, dtype=np.int32)
    rows = []
    used = 0
    for b in range(B):
        L = int(rng.integers(live_min, live_max + 1)) // bs * bs
        L = max(L, prompt + 4 * rmax)
        nblk = L // bs
        # historic gaps: evicted before this step, so next_lpos exceeds L
        hist_blocks = int(rng.integers(0, (max_lpos - L) // bs)) if max_lpos > L + bs else 0
        n_gaps = int(rng.integers(1, 9))
        gap_at = np.sort(rng.choice(np.arange(prompt // bs, nblk), size=n_gaps, replace=False))
        cuts = np.sort(rng.integers(0, hist_blocks + 1, size=n_gaps - 1))
        parts = np.diff(np.concatenate([[0], cuts, [hist_blocks]]))
        lpos = np.arange(nblk, dtype=np.int64) * bs
        for g, p in zip(gap_at, parts):
            lpos[g:] += int(p) * bs
        nxt = int(lpos[-1]) + bs
        assert nxt <= max_lpos
        bt[b, :nblk] = perm[used: used + nblk]
        used += nblk
        bl[b, :nblk] = lpos
        nb[b], nt[b], nl[b] = nblk, L, nxt
        # this step's evictions: disjoint block-index intervals, past the prompt,
        # leaving the most recent rmax tokens alone
        lo_blk, hi_blk = prompt // bs, nblk - rmax // bs
        k = int(rng.integers(cfg.events_min, cfg.events_max + 1))
        taken = np.zeros(nblk, dtype=bool)
        for _ in range(k):
            for _try in range(50):
                ln = int(rng.integers(rmin // bs, rmax // bs + 1))
                s = int(rng.integers(lo_blk, max(lo_blk + 1, hi_blk - ln)))
                if s + ln <= hi_blk and not taken[max(0, s - 1): s + ln + 1].any():
                    taken[s: s + ln] = True
                    rows.append((b, nxt, int(lpos[s]), int(lpos[s + ln - 1]) + bs))
                    break
    for b in range(B):
        new_block[b] = perm[used]
        used += 1
    rows.sort()
    ev = np.asarray(rows, dtype=np.int32).reshape(-1, 4)
    return PagedState(block_size=bs, pool_blocks=pool, max_blocks=max_blocks, block_table=bt,
                      block_lpos=bl, num_blocks=nb, num_tokens=nt, next_lpos=nl, events=ev,
                      new_block=new_block, meta={"blocks_used": used})


# --------------------------------------------------------------------------------------
# Tensors
# --------------------------------------------------------------------------------------

def normal(shape, seed: int, dtype=np.float32) -> np.ndarray:
    """N(0,1) samples from numpy's PCG64 stream for ``seed``."""
    return np.random.default_rng(seed).standard_normal(shape, dtype=np.float32).astype(dtype)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round an fp32 array to the nearest bfloat16 (ties to even), returned as fp32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    out = ((u + r) & np.uint32(0xFFFF0000)).view(np.float32)
    nan = np.isnan(x)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def replay_tensors(cfg: TraceConfig, salt: int = 0):
    """Pre-rotation q ``[B,N,Hq,d]``, k and v ``[B,N,Hkv,d]`` and dO ``[B,N,Hq,d]``,
    N(0,1) and rounded to bf16 for bf16 configs (fp32 for fp32 configs)."""
    B, N = cfg.batch, cfg.n_tokens
    base = cfg.seed(0) * 16 + salt
    q = normal((B, N, cfg.hq, cfg.d), base + 1)
    k = normal((B, N, cfg.hkv, cfg.d), base + 2)
    v = normal((B, N, cfg.hkv, cfg.d), base + 3)
    do = normal((B, N, cfg.hq, cfg.d), base + 4)
    if cfg.dtype == "bf16":
        q, k, v, do = (round_bf16(t) for t in (q, k, v, do))
    return q, k, v, do


def replay_tensors_device(cfg: TraceConfig, device="cuda", salt: int = 0, with_grad: bool = True):
    """Full-size twin of :func:`replay_tensors` drawn with torch's CUDA generator
    (same shapes and distribution, different stream); rounded to bf16 for bf16
    configs. Returns (q, k, v, dO) as torch tensors on ``device``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed(0) * 16 + salt)
    B, N = cfg.batch, cfg.n_tokens
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32

    def draw(h):
        return torch.randn((B, N, h, cfg.d), generator=g, device=device, dtype=torch.float32).to(dt)

    q, k, v = draw(cfg.hq), draw(cfg.hkv), draw(cfg.hkv)
    do = draw(cfg.hq) if with_grad else None
    return q, k, v, do
