"""Packed multi-trace replay: the packed trace's mask (boundaries expressed as
evictions) is block diagonal, each block being the trace's own eviction mask,
checked element by element against the event-by-event dense mask of each trace."""
import numpy as np
import pytest

import oracle
from eviction_masked_attention_b200 import packing
from eviction_masked_attention_b200 import workloads as W
from conftest import dense_mask_eventwise


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_packed_mask_is_block_diagonal_of_trace_masks(seed):
    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in rng.integers(1, 400, 4)]
    evs = [W.random_event_log(rng, 1, n, 4, unit=1, max_span=max(1, n // 3))[:, 1:4] for n in lengths]
    cu, ev, lpos = packing.pack(lengths, evs)
    Nt = int(cu[-1])
    kap = oracle.kappa(ev, 1, Nt)[0]
    got = np.zeros((Nt, Nt), dtype=bool)
    t, j = np.nonzero(np.tril(np.ones((Nt, Nt), dtype=bool)))
    vis = t < kap[j]
    got[t[vis], j[vis]] = True
    want = np.zeros((Nt, Nt), dtype=bool)
    for b, n in enumerate(lengths):
        sl = slice(cu[b], cu[b + 1])
        rows = np.concatenate([np.zeros((len(evs[b]), 1), np.int64), evs[b]], axis=1)
        want[sl, sl] = dense_mask_eventwise(rows, 0, n)
    assert np.array_equal(got, want)
    assert np.array_equal(lpos[cu[1]:cu[2]], np.arange(lengths[1]))


def test_pack_rejects_events_outside_a_trace():
    with pytest.raises(ValueError):
        packing.pack([10, 20], [np.array([[12, 0, 5]]), np.zeros((0, 3))])
