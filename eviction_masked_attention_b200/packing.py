"""Several traces of different lengths replayed as one packed buffer.

Traces b = 0..B-1 of lengths N_b are laid end to end (trace b occupies rows
[cu[b], cu[b+1]) of q, k, v, dO; cu is the running sum of the lengths) and
replayed by one call of the library as a single trace of length cu[B]. Nothing
in the kernels changes: the separation between traces is itself expressed as
an eviction. Trace b's keys are removed, in the packed trace, before the first
token of trace b+1 -- the event (0, cu[b+1], cu[b], cu[b+1]) -- so a query of a
later trace never sees them, while trace b's own queries see exactly what its
own event log allows (its events shifted by cu[b]). The kill time of every key
is then its own trace's kill time, or the end of its trace, whichever comes
first; the compiled mask is block diagonal, and the 128x128 tiles that lie
wholly across traces are EMPTY and skipped like any evicted span. Rotary
positions stay per trace: row cu[b] + i is rotated at logical position i.

Host-side bookkeeping only ("KV-streams for Efficient Compaction in Agentic
Reinforcement Learning", Fig. 2(B): the prompt / summary / overlap policies
whose traces are packed together here).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def pack(lengths: Sequence[int], events: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Packed layout of ``len(lengths)`` traces.

    ``events[b]`` holds trace b's rows (tau, start, end) in its own positions.
    Returns (cu int64 [B+1], the packed trace's event log int32 [E, 4] with seq 0,
    sorted by (tau, start), and the logical position of every packed row int32
    [cu[B]])."""
    n = np.asarray(lengths, dtype=np.int64)
    if (n <= 0).any():
        raise ValueError("trace lengths must be positive")
    cu = np.concatenate([[0], np.cumsum(n)])
    rows: List[Tuple[int, int, int, int]] = []
    for b, ev in enumerate(events):
        ev = np.asarray(ev, dtype=np.int64).reshape(-1, 3)
        off = int(cu[b])
        for tau, s, e in ev:
            if not (0 <= s < e <= tau <= n[b]):
                raise ValueError(f"trace {b}: event ({tau}, {s}, {e}) outside the trace")
            if tau < n[b]:                      # an event at the trace's end changes nothing in it
                rows.append((0, off + int(tau), off + int(s), off + int(e)))
        if b + 1 < len(n):
            rows.append((0, int(cu[b + 1]), off, int(cu[b + 1])))
    rows.sort()
    ev_out = np.asarray(rows, dtype=np.int32).reshape(-1, 4)
    lpos = np.concatenate([np.arange(x, dtype=np.int32) for x in n])
    return cu, ev_out, lpos
