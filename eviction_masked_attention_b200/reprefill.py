"""Re-prefill compaction: the schedule KV-streams replaces, as a comparator.

"KV-streams for Efficient Compaction in Agentic Reinforcement Learning",
Fig. 2(A) and Fig. 3: under re-prefill compaction every event starts a new,
shorter sequence -- the retained tokens are processed again from scratch with
their positions renumbered 0..r-1, and generation continues after them -- so
each kept token is processed once per later compaction. KV-streams keeps the
cache and trains on one continuous trace under the eviction mask instead
("KV-streams: speeding up agentic RL by operating on the KV cache directly",
the first paragraphs of the thread).

This module is host-side bookkeeping only: it turns an event log into the
re-prefill segments (which token ids each segment processes, at which
positions) and evaluates Fig. 3's count of re-processed tokens. The attention
over the segments runs through the library's kernels like any other trace.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import numpy as np


@dataclass
class Segment:
    """One re-prefill sequence: ``retained`` token ids are processed again at
    positions 0..r-1, then ``new`` token ids continue at positions r, r+1, ..."""

    retained: np.ndarray
    new: np.ndarray

    @property
    def tokens(self) -> np.ndarray:
        return np.concatenate([self.retained, self.new])

    @property
    def positions(self) -> np.ndarray:
        return np.arange(len(self.retained) + len(self.new), dtype=np.int32)


def schedule(events3, n_tokens: int) -> List[Segment]:
    """Segments of one trace. ``events3`` holds rows (tau, start, end) sorted by tau:
    positions [start, end) leave the cache before token tau is generated."""
    ev = np.asarray(events3, dtype=np.int64).reshape(-1, 3)
    alive = np.zeros(0, dtype=np.int64)
    retained = np.zeros(0, dtype=np.int64)
    segs: List[Segment] = []
    start = 0
    for tau in sorted(set(int(t) for t in ev[:, 0])):
        if tau >= n_tokens:
            break
        new = np.arange(start, tau, dtype=np.int64)
        segs.append(Segment(retained, new))
        alive = np.concatenate([alive, new])
        for _, s, e in ev[ev[:, 0] == tau]:
            alive = alive[(alive < s) | (alive >= e)]
        retained = alive.copy()
        start = tau
    segs.append(Segment(retained, np.arange(start, n_tokens, dtype=np.int64)))
    return segs


def reprocessed(segs: List[Segment]) -> int:
    """Tokens processed again under re-prefill (KV-streams processes none again)."""
    return int(sum(len(s.retained) for s in segs))


def fig3_count(n_tokens: int, budget: int, kept: int) -> Tuple[int, int]:
    """Fig. 3's accounting for a rollout that compacts whenever the live length
    reaches ``budget`` and keeps ``kept`` tokens (prompt, summary and overlap):
    events fall at budget, budget + (budget - kept), ... below n_tokens; each
    re-processes ``kept`` tokens. Returns (events, re-processed tokens)."""
    if n_tokens <= budget or budget <= kept:
        return 0, 0
    n_ev = (n_tokens - budget - 1) // (budget - kept) + 1
    return n_ev, n_ev * kept


def fig3_factor(n_tokens: int, budget: int, kept: int) -> float:
    """The figure's closed form N / (B - kept): how many times a kept token is
    processed again over the rollout (the event count, for N >> B)."""
    return n_tokens / (budget - kept)
