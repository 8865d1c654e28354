"""Host logic of the multi-process bench on CPU (gloo, two ranks): each rank takes
its own traces, the job time is the slowest rank's and the credited pairs are
summed over ranks. No GPU is involved."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        elapsed, pairs = bench.over_ranks(10.0 + rank, 100.0 * (rank + 1), torch.device("cpu"))
        out.put((rank, elapsed, pairs))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_time_max_and_pairs_sum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]      # slowest rank's time on every rank
    assert [r[2] for r in res] == [300.0, 300.0]    # pairs of both ranks' traces


def test_single_process_returns_its_own_figures():
    import bench

    assert not dist.is_initialized()
    assert bench.over_ranks(7.5, 42.0, torch.device("cpu")) == (7.5, 42.0)


def test_ranks_take_distinct_traces():
    import bench
    from eviction_masked_attention_b200 import workloads as W

    cfg = W.scaled(W.CONFIGS[5], 16)
    e0, e1 = bench.rank_events(cfg, 0), bench.rank_events(cfg, 1)
    for e in (e0, e1):
        assert len(e) and e[:, 0].min() >= 0 and e[:, 0].max() < cfg.batch
        key = e[:, 0].astype(np.int64) * 2**40 + e[:, 1].astype(np.int64) * 2**20 + e[:, 2]
        assert np.all(np.diff(key) >= 0)             # sorted by (seq, tau, start)
    assert not (e0.shape == e1.shape and np.array_equal(e0, e1))
    # rank 1's traces are traces B..2B-1 of the same seeded family
    both = W.make_event_log(W.replace(cfg, batch=2 * cfg.batch))
    tail = both[both[:, 0] >= cfg.batch].copy()
    tail[:, 0] -= cfg.batch
    np.testing.assert_array_equal(e1, tail)


def test_cpu_baseline_entry_extrapolates_linearly():
    import bench

    e = bench.cpu_baseline_entry(2.0e12, 4.0, 16, 1.0e15, "sample")
    assert e["value"] == 0.5 and e["unit"] == "TFLOP/s" and e["kind"] == "oracle" and e["cores"] == 16
    assert e["extrapolated_full_step_s"] == 2000.0


def test_host_visible_pairs_counts_the_eventwise_mask():
    """The reference arm's workload description counts visible pairs on the host;
    it must equal the pairs of the mask built event by event from the replay rule."""
    import bench
    from conftest import dense_mask_eventwise
    rng = np.random.default_rng(7)
    for _ in range(20):
        B, N = int(rng.integers(1, 3)), int(rng.integers(1, 300))
        ev = []
        for b in range(B):
            for _ in range(int(rng.integers(0, 4))):
                tau = int(rng.integers(1, N + 1))
                a = int(rng.integers(0, tau))
                e = int(rng.integers(a + 1, tau + 1))
                ev.append((b, tau, a, e))
        ev = np.array(ev, dtype=np.int64).reshape(-1, 4)
        want = sum(int(dense_mask_eventwise(ev, b, N).sum()) for b in range(B))
        assert bench.host_visible_pairs(ev, B, N) == want
