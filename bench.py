#!/usr/bin/env python
"""Benchmark of the KV-streams hot path on B200.

One step = one pass of the whole path over one batch of synthetic traces of the
1-token-block workload (2 traces x 131072 logical tokens, Hq=64, Hkv=8, d=128,
budget 32768, whole unpadded turns of 64..4096 tokens evicted at arbitrary
offsets, 15 events per trace):

  training side   event log -> tile mask (kill times, classes, row/col lists,
                  partial bits), recompiled each step into the buffers counted
                  at set-up with no host round trip; logical RoPE of q and k; eviction-masked
                  attention forward; backward (prep, dK/dV, dQ kernels); inverse
                  RoPE of dq and dk
  generation side block-table compaction at each trace's last event; RoPE of the
                  next token's q and k at its logical position with k/v scattered
                  into a free slot; split-K paged decode over the compacted table

``value`` = unmasked fwd+bwd TFLOP/s of the whole step: 14*d flops per visible
(query, key) pair and query head (4d forward, 10d backward), over the step time.
The decode GB/s, per-kernel times and the roofline of the dominant kernel are
reported beside it. Inputs (4.3 GB q alone) exceed the 126 MB L2, so no flush
is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from eviction_masked_attention_b200 import workloads as W  # noqa: E402

METRIC = "eviction-masked attn fwd+bwd TFLOP/s (unmasked); compacted paged-decode GB/s"
FLOPS_PER_PAIR_D = 14  # 4d forward + 10d backward per visible pair and query head


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--scale", type=int, default=1, help="divide the trace length (profiling runs)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-per-config", action="store_true")
    return p.parse_args()


def _peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "fallback": True}


def workload_cfg(scale: int):
    return W.scaled(W.CONFIGS[5], scale) if scale > 1 else W.CONFIGS[5]


def rank_events(cfg, rank: int):
    """This rank's traces: trace ids rank*B .. rank*B+B-1 of the seeded family,
    renumbered 0..B-1."""
    big = W.replace(cfg, batch=cfg.batch * (rank + 1))
    ev = W.make_event_log(big)
    ev = ev[ev[:, 0] >= rank * cfg.batch].copy()
    ev[:, 0] -= rank * cfg.batch
    return ev


# ----------------------------------------------------------------------------- CPU oracle

CPU_SAMPLE_TOKENS = 3584  # about 10-15 s of the oracle on the 16 host cores of a B200 machine


def oracle_sample(cfg, budget_tokens: int):
    """The fp64 oracle (as it stands) on a bounded sample of the workload: the
    first ``budget_tokens`` tokens of trace 0 for one kv group (G query heads),
    forward + full backward. Returns (credited flops, seconds, threads)."""
    import oracle

    n = min(budget_tokens, cfg.n_tokens)
    sub = W.replace(cfg, batch=1, n_tokens=n)
    ev = W.make_event_log(W.replace(cfg, batch=1))
    ev = ev[ev[:, 1] < n]
    G, d = cfg.hq // cfg.hkv, cfg.d
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, n, G, d))
    k = rng.standard_normal((1, n, 1, d))
    v = rng.standard_normal((1, n, 1, d))
    do = rng.standard_normal((1, n, G, d))
    kap = oracle.kappa(ev, 1, n)
    pairs = oracle.visible_pairs(kap)
    t0 = time.perf_counter()
    oracle.attn_bwd(q, k, v, do, kap, sub.scale)
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return FLOPS_PER_PAIR_D * d * pairs * G, dt, threads


def cpu_baseline_entry(flops: float, secs: float, threads: int, flops_step: float, sample: str):
    """The oracle's measured rate on its sample, and the time a whole step of the
    workload would take at that rate (extrapolated linearly in credited flops,
    i.e. in visible pairs, and labelled as such)."""
    rate = flops / secs
    return {"value": rate / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample,
            "extrapolated_full_step_s": flops_step / rate}


def host_visible_pairs(ev, B: int, N: int) -> int:
    """Visible (query, key) pairs of the event log: key j is visible from queries j..kappa_j-1,
    kappa_j the earliest event time covering j (N if none). Host integer arithmetic, used
    only to describe the workload in the reference arm's config."""
    total = 0
    for b in range(B):
        kap = np.full(N, N, dtype=np.int64)
        for (s, tau, a, e) in np.asarray(ev).reshape(-1, 4):
            if s == b:
                kap[a:e] = np.minimum(kap[a:e], tau)
        total += int((kap - np.arange(N)).sum())
    return total


def workload_config(cfg, world: int, n_events: int, pairs: float) -> dict:
    """The bench line's config (both arms)."""
    return {"workload": f"cfg5 bs1: {cfg.batch}x{cfg.n_tokens} tokens/rank, Hq={cfg.hq}, "
                        f"Hkv={cfg.hkv}, d={cfg.d}, budget {cfg.budget}, {n_events} events/rank",
            "global_batch": cfg.batch * world, "seq_len": cfg.n_tokens,
            "parallelism": f"replicas x{world} (independent traces per rank)",
            "l2": "inputs larger than L2 (4.3 GB q per rank), no flush",
            "visible_pair_fraction": pairs / (cfg.batch * cfg.n_tokens * (cfg.n_tokens + 1) / 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = workload_cfg(args.scale)
    ev = rank_events(cfg, 0)
    budget = 768
    for _ in range(args.warmup):
        oracle_sample(cfg, 256)
    flops = secs = 0.0
    threads = 1
    for _ in range(args.steps):
        f, s, threads = oracle_sample(cfg, budget)
        flops += f
        secs += s
    value = flops / secs / 1e12
    sample = (f"first {budget} tokens of trace 0, one kv group ({cfg.hq // cfg.hkv} query heads), "
              f"fwd + full bwd, per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(cfg, args.gpus, len(ev), host_visible_pairs(ev, cfg.batch, cfg.n_tokens)),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- our path

class Step:
    """Device buffers and one step of the hot path for this rank."""

    def __init__(self, cfg, rank: int, device):
        import eviction_masked_attention_b200 as kvs

        self.kvs, self.cfg, self.dev = kvs, cfg, device
        B, N, Hq, Hkv, d = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d
        self.ev_host = rank_events(cfg, rank)
        self.events = torch.from_numpy(self.ev_host).to(device)
        self.q_raw, self.k_raw, self.v, self.do = W.replay_tensors_device(cfg, device=device, salt=rank)
        self.lpos = torch.arange(N, dtype=torch.int32, device=device).repeat(B)
        self.q = torch.empty_like(self.q_raw)
        self.k = torch.empty_like(self.k_raw)
        self.o = torch.empty_like(self.q_raw)
        self.o_lo = torch.empty_like(self.q_raw)
        self.lse = torch.empty((B, Hq, N), dtype=torch.float32, device=device)
        self.dq = torch.empty_like(self.q_raw)
        self.dk = torch.empty_like(self.k_raw)
        self.dv = torch.empty_like(self.v)
        self.dq_raw = torch.empty_like(self.q_raw)
        self.dk_raw = torch.empty_like(self.k_raw)
        L = kvs.lib()
        self.bwd_ws = torch.empty(L.kvs_masked_attn_bwd_ws_bytes(B, N, Hq, Hkv, d, kvs.KVS_BF16),
                                  dtype=torch.uint8, device=device)
        self.mask_ws = torch.empty(L.kvs_build_tile_mask_ws_bytes(B, N), dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        # counted once here; every step recompiles the log into these buffers
        mask = kvs.kvs_build_tile_mask(self.events, B, N, ws=self.mask_ws)
        self.mask = mask
        self.pairs = mask.visible_pairs
        self._setup_generation(mask)

    def _setup_generation(self, mask):
        """Paged (1-token block) cache of every trace just before its last event:
        live slots in logical order, keys rotated at their logical positions."""
        kvs, cfg, dev = self.kvs, self.cfg, self.dev
        B, N, Hq, Hkv, d = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d
        ev = self.ev_host
        kap = mask.kappa
        self.tau = []
        tables, lposs = [], []
        pool = B * N + B
        perm = torch.from_numpy(np.random.default_rng(77).permutation(pool).astype(np.int32)).to(dev)
        for b in range(B):
            taus = ev[ev[:, 0] == b, 1]
            tau = int(taus.max()) if len(taus) else N - 1
            self.tau.append(tau)
            j = torch.arange(tau, device=dev, dtype=torch.int32)
            live = j[kap[b, :tau] >= tau]                      # alive right before the event
            tables.append(perm[b * N + live.long()])
            lposs.append(live)
        M = max(len(t) for t in tables) + 1
        self.M = M
        bt = torch.full((B, M), -1, dtype=torch.int32, device=dev)
        bl = torch.full((B, M), -1, dtype=torch.int32, device=dev)
        for b in range(B):
            bt[b, :len(tables[b])] = tables[b]
            bl[b, :len(lposs[b])] = lposs[b]
        self.bt0, self.bl0 = bt, bl
        self.nb0 = torch.tensor([len(t) for t in tables], dtype=torch.int32, device=dev)
        self.bt, self.bl = bt.clone(), bl.clone()
        self.nb, self.nt = self.nb0.clone(), self.nb0.clone()
        last = [ev[(ev[:, 0] == b) & (ev[:, 1] == self.tau[b])] for b in range(B)]
        self.gen_events = torch.from_numpy(np.concatenate(last).astype(np.int32)).to(dev)
        self.pool = pool
        self.kc = torch.zeros((pool, Hkv, 1, d), dtype=torch.bfloat16, device=dev)
        self.vc = torch.zeros_like(self.kc)
        # every position's rotated key / value at its slot (the cache as generation left it)
        for b in range(B):
            s = perm[b * N: (b + 1) * N].to(torch.int64)
            kvs.kvs_rope_logical(self.k_raw[b], self.lpos[:N], cfg.theta, out=self.kc, out_slot=s,
                                 block_size=1, v=self.v[b], v_out=self.vc)
        # the next token of each trace takes logical position tau, physical slot B*N + b
        self.new_slot = torch.tensor([perm[B * N + b].item() for b in range(B)], dtype=torch.int64,
                                     device=dev)
        self.new_lpos = torch.tensor(self.tau, dtype=torch.int32, device=dev)
        # rows of the token each trace generates next (gathered from this step's inputs)
        self.new_rows = torch.tensor([b * N + t for b, t in enumerate(self.tau)], device=dev, dtype=torch.long)
        self.q_new = torch.empty((B, Hq, d), dtype=self.q_raw.dtype, device=dev)
        self.k_new = torch.empty((B, Hkv, d), dtype=self.q_raw.dtype, device=dev)
        self.v_new = torch.empty((B, Hkv, d), dtype=self.q_raw.dtype, device=dev)
        self.q_new_r = torch.empty_like(self.q_new)
        self.o_dec = torch.empty_like(self.q_new)
        L = kvs.lib()
        self.dec_ws = torch.zeros(L.kvs_paged_decode_ws_bytes(B, Hq, Hkv, d, 1, M), dtype=torch.uint8,
                                  device=dev)
        self.freed = torch.empty((B, M), dtype=torch.int32, device=dev)
        self.n_freed = torch.empty(B, dtype=torch.int32, device=dev)
        self.rows = torch.arange(B, device=dev)

    # launches of our kernels per step (see each call)
    def launches(self) -> int:
        has_ev = 1 if len(self.ev_host) else 0
        mask = 3 + has_ev + 2 + 1          # checks, kill times, classes, scans, 2 fills, finish
        # RoPE of q and k, forward, prep + dK/dV + dQ, inverse RoPE of dq and dk, compaction,
        # RoPE + scatter of the new key and value, RoPE of the new query, decode split + merge
        return mask + 2 + 1 + 3 + 2 + 1 + 1 + 1 + 2

    def run(self, ev_rec=None, bwd_wait=None):
        """One step; if ev_rec is a dict, records CUDA events around each call. With
        bwd_wait (a CUDA event) the backward waits for it: the forward may start
        while dO is still being copied in."""
        kvs, cfg = self.kvs, self.cfg
        B, N, Hq, Hkv, d = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d

        def mark(name):
            if ev_rec is not None:
                e = torch.cuda.Event(enable_timing=True)
                e.record()
                ev_rec.setdefault(name, []).append(e)

        mark("start")
        mask = kvs.kvs_build_tile_mask_async(self.events, self.mask, ws=self.mask_ws, status=self.status)
        mark("mask")
        kvs.kvs_rope_logical(self.q_raw.view(B * N, Hq, d), self.lpos, cfg.theta, out=self.q.view(B * N, Hq, d))
        kvs.kvs_rope_logical(self.k_raw.view(B * N, Hkv, d), self.lpos, cfg.theta, out=self.k.view(B * N, Hkv, d))
        mark("rope")
        kvs.kvs_masked_attn_fwd(self.q, self.k, self.v, mask, cfg.scale, out=self.o, lse=self.lse,
                                out_lo=self.o_lo, status=self.status)
        mark("fwd")
        if bwd_wait is not None:
            torch.cuda.current_stream().wait_event(bwd_wait)
        for st, name in ((kvs.KVS_BWD_PREP, "bwd_prep"), (kvs.KVS_BWD_DKDV, "dkdv"), (kvs.KVS_BWD_DQ, "dq")):
            kvs.kvs_masked_attn_bwd(self.q, self.k, self.v, self.o, self.do, self.lse, mask, cfg.scale,
                                    dq=self.dq, dk=self.dk, dv=self.dv, ws=self.bwd_ws, status=self.status,
                                    stages=st, o_lo=self.o_lo)
            mark(name)
        kvs.kvs_rope_logical(self.dq.view(B * N, Hq, d), self.lpos, cfg.theta, inverse=True,
                             out=self.dq_raw.view(B * N, Hq, d))
        kvs.kvs_rope_logical(self.dk.view(B * N, Hkv, d), self.lpos, cfg.theta, inverse=True,
                             out=self.dk_raw.view(B * N, Hkv, d))
        mark("rope_inv")
        # generation side: restore the pre-event table, compact, append the new token, decode
        self.bt.copy_(self.bt0)
        self.bl.copy_(self.bl0)
        self.nb.copy_(self.nb0)
        self.nt.copy_(self.nb0)
        torch.index_select(self.q_raw.view(B * N, Hq, d), 0, self.new_rows, out=self.q_new)
        torch.index_select(self.k_raw.view(B * N, Hkv, d), 0, self.new_rows, out=self.k_new)
        torch.index_select(self.v.view(B * N, Hkv, d), 0, self.new_rows, out=self.v_new)
        mark("restore")
        kvs.kvs_compact_block_table(self.bt, self.bl, self.nb, self.nt, 1, self.pool, self.gen_events,
                                    freed=self.freed, n_freed=self.n_freed, status=self.status)
        mark("compact")
        kvs.kvs_rope_logical(self.k_new, self.new_lpos, cfg.theta, out=self.kc, out_slot=self.new_slot,
                             block_size=1, v=self.v_new, v_out=self.vc)
        kvs.kvs_rope_logical(self.q_new, self.new_lpos, cfg.theta, out=self.q_new_r)
        self.bt.view(-1)[self.rows * self.M + self.nb.long()] = self.new_slot.to(torch.int32)
        self.nt.add_(1)
        mark("append")
        kvs.kvs_paged_decode_attn(self.q_new_r, self.kc, self.vc, self.bt, self.nt, 1, cfg.scale,
                                  out=self.o_dec, ws=self.dec_ws, status=self.status)
        mark("decode")
        return mask

    def decode_bytes(self) -> int:
        cfg = self.cfg
        nt = int(self.nt.sum().item())
        kv = nt * cfg.hkv * cfg.d * 2 * 2
        return kv + 2 * self.q_new.numel() * 2 + nt * 4 + cfg.batch * 4


def _durations(rec):
    names = ["mask", "rope", "fwd", "bwd_prep", "dkdv", "dq", "rope_inv", "restore", "compact", "append",
             "decode"]
    out = {n: [] for n in names}
    for i in range(len(rec["start"])):
        prev = rec["start"][i]
        for n in names:
            e = rec[n][i]
            out[n].append(prev.elapsed_time(e))
            prev = e
    return {n: float(np.mean(v)) for n, v in out.items()}


# DRAM traffic of one launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum) on the
# 1/16-scale bs1 workload: kernel -> (bytes of that launch, visible pairs x query heads it processed,
# sha1 prefix of the kernel sources it was taken with). The bench scales it to its own launch by the
# pairs processed and reports null once the sources have changed.
TRAFFIC = {"dkdv": (1.779736e9 + 56.255488e6, 27713931 * 64, "3fc511ecb941")}


def _src_hash(files):
    h = hashlib.sha1()
    for f in files:
        h.update(open(os.path.join(ROOT, "eviction_masked_attention_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:12]


def over_ranks(elapsed_ms: float, pairs: float, device):
    """Job-wide figures of a timed region: the slowest rank's time and the visible
    pairs of all ranks' traces. One collective of each kind, taken by every rank in
    the same order; a single process returns its own figures."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return elapsed_ms, pairs
    t = torch.tensor([elapsed_ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    p = torch.tensor([pairs], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(p)
    return float(t.item()), float(p.item())


# ----------------------------------------------------------------------------- other configurations

def _time_ms(fn, iters: int, warmup: int = 2) -> float:
    """Mean device time of fn() over iters calls (CUDA events on the current stream)."""
    for _ in range(warmup):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def _attn_config(cid: int, dev, peaks, bwd: bool, scale: int = 1):
    """Masked forward (and backward) on one replay configuration at full size."""
    import eviction_masked_attention_b200 as kvs

    cfg = W.CONFIGS[cid] if scale == 1 else W.scaled(W.CONFIGS[cid], scale)
    B, N, Hq, Hkv, d = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d
    ev = torch.from_numpy(W.make_event_log(cfg)).to(dev)
    q, k, v, do = W.replay_tensors_device(cfg, device=dev, with_grad=bwd)
    mask_ws = torch.empty(kvs.lib().kvs_build_tile_mask_ws_bytes(B, N), dtype=torch.uint8, device=dev)
    mask = kvs.kvs_build_tile_mask(ev, B, N, ws=mask_ws)
    t_mask = _time_ms(lambda: kvs.kvs_build_tile_mask_async(ev, mask, ws=mask_ws), 5)
    P = float(mask.visible_pairs)
    o, lse, o_lo = torch.empty_like(q), torch.empty((B, Hq, N), dtype=torch.float32, device=dev), torch.empty_like(q)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    fwd = lambda: kvs.kvs_masked_attn_fwd(q, k, v, mask, cfg.scale, out=o, lse=lse, out_lo=o_lo, status=st)
    t_fwd = _time_ms(fwd, 10 if not bwd else 5)
    out = {"workload": f"cfg{cid}: {B}x{N}, Hq={Hq}, Hkv={Hkv}, d={d}, {len(ev)} events",
           "visible_pair_fraction": P / (B * N * (N + 1) / 2), "mask_ms": t_mask, "fwd_ms": t_fwd,
           "fwd_tflops": 4 * d * P * Hq / (t_fwd * 1e-3) / 1e12}
    if bwd:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(kvs.lib().kvs_masked_attn_bwd_ws_bytes(B, N, Hq, Hkv, d, kvs.KVS_BF16),
                         dtype=torch.uint8, device=dev)
        bw = lambda: kvs.kvs_masked_attn_bwd(q, k, v, o, do, lse, mask, cfg.scale, dq=dq, dk=dk, dv=dv, ws=ws,
                                             status=st, o_lo=o_lo)
        t_bwd = _time_ms(bw, 5)
        # 10 d per pair counts the backward's five products (S recomputed); 8 d leaves the recompute out
        out.update({"bwd_ms": t_bwd, "bwd_tflops": 10 * d * P * Hq / (t_bwd * 1e-3) / 1e12,
                    "bwd_tflops_8d": 8 * d * P * Hq / (t_bwd * 1e-3) / 1e12,
                    "fwd_bwd_tflops": 14 * d * P * Hq / ((t_fwd + t_bwd) * 1e-3) / 1e12})
        tf = out["fwd_bwd_tflops"]
    else:
        tf = out["fwd_tflops"]
    torch.cuda.synchronize()
    assert st.item() == 0, f"device status {st.item()}"
    out["frac_bf16_burst"] = tf / float(peaks.get("bf16_tflops", 1590.0))
    out["frac_bf16_sustained"] = tf / float(peaks.get("bf16_tflops_sustained", 1400.0))
    return out


def _paged_config(dev, peaks):
    """The paged-generation configuration: 64 sequences on a 131072-block pool of
    16-token blocks; one compaction step, then decode over the compacted tables.
    Also decode over the first 1, 2, ..., 64 sequences (tokens/s against live
    sequences)."""
    import eviction_masked_attention_b200 as kvs

    cfg = W.CONFIGS[4]
    st = W.make_paged_state(cfg)
    B, Hq, Hkv, d, bs = cfg.batch, cfg.hq, cfg.hkv, cfg.d, st.block_size
    g = torch.Generator(device=dev)
    g.manual_seed(4004)
    kc = torch.randn((st.pool_blocks, Hkv, bs, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn((st.pool_blocks, Hkv, bs, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    q = torch.randn((B, Hq, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    bt0, bl0 = torch.from_numpy(st.block_table).to(dev), torch.from_numpy(st.block_lpos).to(dev)
    nb0, nt0 = torch.from_numpy(st.num_blocks).to(dev), torch.from_numpy(st.num_tokens).to(dev)
    ev = torch.from_numpy(st.events).to(dev)
    bt, bl, nb, nt = bt0.clone(), bl0.clone(), nb0.clone(), nt0.clone()
    freed = torch.empty_like(bt)
    n_freed = torch.empty_like(nb)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def compact():
        bt.copy_(bt0); bl.copy_(bl0); nb.copy_(nb0); nt.copy_(nt0)
        kvs.kvs_compact_block_table(bt, bl, nb, nt, bs, st.pool_blocks, ev, freed=freed, n_freed=n_freed,
                                    status=status)

    t_restore = _time_ms(lambda: (bt.copy_(bt0), bl.copy_(bl0), nb.copy_(nb0), nt.copy_(nt0)), 20)
    t_compact = _time_ms(compact, 20) - t_restore
    compact()
    torch.cuda.synchronize()
    ntoks = nt.cpu().numpy().astype(np.int64)
    nblks = nb.cpu().numpy().astype(np.int64)
    o = torch.empty_like(q)

    def decode_entry(nseq):
        ws = torch.empty(kvs.lib().kvs_paged_decode_ws_bytes(nseq, Hq, Hkv, d, bs, bt.shape[1]),
                         dtype=torch.uint8, device=dev)
        qs, os_, bts, nts = q[:nseq], o[:nseq], bt[:nseq], nt[:nseq]
        t = _time_ms(lambda: kvs.kvs_paged_decode_attn(qs, kc, vc, bts, nts, bs, cfg.scale, out=os_, ws=ws,
                                                       status=status), 20, 3)
        byts = int(ntoks[:nseq].sum()) * Hkv * d * 2 * 2 + 2 * nseq * Hq * d * 2 + int(nblks[:nseq].sum()) * 4
        gbs = byts / (t * 1e-3) / 1e9
        return {"seqs": nseq, "ms": t, "bytes": byts, "gbs": gbs, "tokens_per_s": nseq / (t * 1e-3),
                "frac_hbm_measured": gbs / float(peaks["hbm_gbs"]), "frac_8tbs": gbs / 8000.0}

    full = decode_entry(B)
    sweep = [decode_entry(n) for n in (1, 2, 4, 8, 16, 32)] + [full]
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item()}"
    full.update({"workload": f"cfg4: {B} seqs, bs {bs}, pool {st.pool_blocks} blocks, live "
                             f"{int(ntoks.min())}..{int(ntoks.max())} tokens after compaction "
                             f"({len(st.events)} events)",
                 "compact_us": t_compact * 1e3})
    return full, [{k: e[k] for k in ("seqs", "ms", "gbs", "tokens_per_s")} for e in sweep]


def _reprefill_config(dev, scale: int = 1):
    """Re-prefill against KV-streams on the summary-policy configuration (4 x 65536
    tokens, budget 16384, each compaction keeps prompt + summary + overlap = 3584):
    device time of RoPE + forward + backward of the training replay under each
    schedule (KV-streams: one continuous trace under the eviction mask; re-prefill:
    every segment re-processes its retained tokens from position 0), and of the
    generation-side work at the events (re-prefill: a causal forward over the
    retained tokens; KV-streams: block-table compaction)."""
    import eviction_masked_attention_b200 as kvs
    from eviction_masked_attention_b200 import reprefill as R

    cfg = W.CONFIGS[3] if scale == 1 else W.scaled(W.CONFIGS[3], scale)
    B, N, Hq, Hkv, d = cfg.batch, cfg.n_tokens, cfg.hq, cfg.hkv, cfg.d
    ev_np = W.make_event_log(cfg)
    ev = torch.from_numpy(ev_np).to(dev)
    q_raw, k_raw, v, do = W.replay_tensors_device(cfg, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    L = kvs.lib()

    # KV-streams: the continuous trace
    lp = torch.arange(N, dtype=torch.int32, device=dev).repeat(B)
    q, k = torch.empty_like(q_raw), torch.empty_like(k_raw)
    mask = kvs.kvs_build_tile_mask(ev, B, N)
    o, lse, o_lo = torch.empty_like(q), torch.empty((B, Hq, N), dtype=torch.float32, device=dev), torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(L.kvs_masked_attn_bwd_ws_bytes(B, N, Hq, Hkv, d, kvs.KVS_BF16), dtype=torch.uint8, device=dev)

    def kv_train():
        kvs.kvs_rope_logical(q_raw.view(B * N, Hq, d), lp, cfg.theta, out=q.view(B * N, Hq, d))
        kvs.kvs_rope_logical(k_raw.view(B * N, Hkv, d), lp, cfg.theta, out=k.view(B * N, Hkv, d))
        kvs.kvs_masked_attn_fwd(q, k, v, mask, cfg.scale, out=o, lse=lse, out_lo=o_lo, status=st)
        kvs.kvs_masked_attn_bwd(q, k, v, o, do, lse, mask, cfg.scale, dq=dq, dk=dk, dv=dv, ws=ws, status=st,
                                o_lo=o_lo)

    t_kv = _time_ms(kv_train, 3, 1)
    pairs_kv = float(mask.visible_pairs)
    del q, k, o, lse, o_lo, dq, dk, dv, ws, mask
    torch.cuda.empty_cache()

    # re-prefill: per trace, per segment, a causal sequence at renumbered positions
    segs, n_reproc = [], 0
    none = torch.zeros((0, 4), dtype=torch.int32, device=dev)
    for b in range(B):
        for sg in R.schedule(ev_np[ev_np[:, 0] == b][:, 1:4], N):
            n = len(sg.tokens)
            idx = torch.from_numpy(sg.tokens).to(dev)
            seg = {"b": b, "idx": idx, "n": n, "r": len(sg.retained),
                   "lp": torch.from_numpy(sg.positions).to(dev), "mask": kvs.kvs_build_tile_mask(none, 1, n)}
            for nm, h in (("q", Hq), ("k", Hkv), ("v", Hkv), ("do", Hq), ("o", Hq), ("olo", Hq), ("dq", Hq),
                          ("dk", Hkv), ("dv", Hkv), ("qr", Hq), ("kr", Hkv)):
                seg[nm] = torch.empty((1, n, h, d), dtype=torch.bfloat16, device=dev)
            seg["lse"] = torch.empty((1, Hq, n), dtype=torch.float32, device=dev)
            seg["ws"] = torch.empty(L.kvs_masked_attn_bwd_ws_bytes(1, n, Hq, Hkv, d, kvs.KVS_BF16),
                                    dtype=torch.uint8, device=dev)
            segs.append(seg)
            n_reproc += len(sg.retained)

    def rp_train():
        for sg in segs:
            b, idx, n = sg["b"], sg["idx"], sg["n"]
            torch.index_select(q_raw[b], 0, idx, out=sg["q"][0])
            torch.index_select(k_raw[b], 0, idx, out=sg["k"][0])
            torch.index_select(v[b], 0, idx, out=sg["v"][0])
            torch.index_select(do[b], 0, idx, out=sg["do"][0])
            kvs.kvs_rope_logical(sg["q"][0], sg["lp"], cfg.theta, out=sg["qr"][0])
            kvs.kvs_rope_logical(sg["k"][0], sg["lp"], cfg.theta, out=sg["kr"][0])
            kvs.kvs_masked_attn_fwd(sg["qr"], sg["kr"], sg["v"], sg["mask"], cfg.scale, out=sg["o"], lse=sg["lse"],
                                    out_lo=sg["olo"], status=st)
            kvs.kvs_masked_attn_bwd(sg["qr"], sg["kr"], sg["v"], sg["o"], sg["do"], sg["lse"], sg["mask"],
                                    cfg.scale, dq=sg["dq"], dk=sg["dk"], dv=sg["dv"], ws=sg["ws"], status=st,
                                    o_lo=sg["olo"])

    t_rp = _time_ms(rp_train, 3, 1)
    pairs_rp = float(sum(sg["n"] * (sg["n"] + 1) // 2 for sg in segs))

    # generation side at the events: re-prefill runs a causal forward over the
    # retained tokens of each new segment; KV-streams compacts the block table
    pre = [sg for sg in segs if sg["r"] > 0]
    pre_masks = [kvs.kvs_build_tile_mask(none, 1, sg["r"]) for sg in pre]

    def rp_prefill():
        for sg, m in zip(pre, pre_masks):
            r = sg["r"]
            kvs.kvs_masked_attn_fwd(sg["qr"][:, :r], sg["kr"][:, :r], sg["v"][:, :r], m, cfg.scale,
                                    out=sg["o"][:, :r], lse=sg["lse_pre"], residual=False, status=st)

    for sg in pre:
        sg["lse_pre"] = torch.empty((1, Hq, sg["r"]), dtype=torch.float32, device=dev)
    t_pre = _time_ms(rp_prefill, 3, 1)
    torch.cuda.synchronize()
    assert st.item() == 0, f"device status {st.item()}"
    kept = cfg.prompt + cfg.summary + cfg.overlap
    n_ev, extra = R.fig3_count(N, cfg.budget, kept)
    return {"workload": f"cfg3: {B}x{N}, budget {cfg.budget}, kept {kept} per compaction, {len(ev_np)} events",
            "kvstreams_train_ms": t_kv, "reprefill_train_ms": t_rp, "train_ratio": t_rp / t_kv,
            "kvstreams_pairs": pairs_kv, "reprefill_pairs": pairs_rp,
            "tokens_processed": {"kvstreams": B * N, "reprefill": B * N + n_reproc},
            "reprefill_prefill_ms": t_pre, "reprocessed_tokens": n_reproc,
            "fig3": {"events_per_trace": n_ev, "reprocessed_per_trace": extra,
                     "factor_N_over_B_minus_kept": R.fig3_factor(N, cfg.budget, kept)}}


def _packed_config(dev, peaks, scale: int = 1):
    """Packed multi-trace replay: five traces of different lengths and compaction
    policies (summary at two points, Markovian carry-over, recent turns, oldest
    turns at 1-token granularity) in one buffer, RoPE at per-trace positions +
    forward + backward in one call each, against the same traces run one call
    per trace."""
    import eviction_masked_attention_b200 as kvs
    from eviction_masked_attention_b200 import packing

    mix = W.policy_mix(hq=32, hkv=8, div=scale)
    Hq, Hkv, d = 32, 8, 128
    lengths = [c.n_tokens for c in mix]
    evs = [np.asarray(W.make_trace_events(c, 0), np.int64).reshape(-1, 3) for c in mix]
    cu, ev, lpos = packing.pack(lengths, evs)
    Nt = int(cu[-1])
    g = torch.Generator(device=dev)
    g.manual_seed(6100)
    rnd = lambda h: torch.randn((1, Nt, h, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    q_raw, k_raw, v, do = rnd(Hq), rnd(Hkv), rnd(Hkv), rnd(Hq)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    L = kvs.lib()

    def job(lo, hi, events):
        n = hi - lo
        e = torch.from_numpy(events).to(dev)
        j = {"n": n, "lp": torch.from_numpy(lpos[lo:hi].copy()).to(dev), "mask": kvs.kvs_build_tile_mask(e, 1, n),
             "q": torch.empty((1, n, Hq, d), dtype=torch.bfloat16, device=dev),
             "k": torch.empty((1, n, Hkv, d), dtype=torch.bfloat16, device=dev),
             "o": torch.empty((1, n, Hq, d), dtype=torch.bfloat16, device=dev),
             "olo": torch.empty((1, n, Hq, d), dtype=torch.bfloat16, device=dev),
             "lse": torch.empty((1, Hq, n), dtype=torch.float32, device=dev),
             "dq": torch.empty((1, n, Hq, d), dtype=torch.bfloat16, device=dev),
             "dk": torch.empty((1, n, Hkv, d), dtype=torch.bfloat16, device=dev),
             "dv": torch.empty((1, n, Hkv, d), dtype=torch.bfloat16, device=dev),
             "ws": torch.empty(L.kvs_masked_attn_bwd_ws_bytes(1, n, Hq, Hkv, d, kvs.KVS_BF16),
                               dtype=torch.uint8, device=dev),
             "src": (q_raw[:, lo:hi], k_raw[:, lo:hi], v[:, lo:hi].contiguous(), do[:, lo:hi].contiguous())}
        return j

    def run(j):
        qs, ks, vs, dos = j["src"]
        kvs.kvs_rope_logical(qs[0], j["lp"], 5e5, out=j["q"][0])
        kvs.kvs_rope_logical(ks[0], j["lp"], 5e5, out=j["k"][0])
        kvs.kvs_masked_attn_fwd(j["q"], j["k"], vs, j["mask"], 1 / np.sqrt(d), out=j["o"], lse=j["lse"],
                                out_lo=j["olo"], status=st)
        kvs.kvs_masked_attn_bwd(j["q"], j["k"], vs, j["o"], dos, j["lse"], j["mask"], 1 / np.sqrt(d), dq=j["dq"],
                                dk=j["dk"], dv=j["dv"], ws=j["ws"], status=st, o_lo=j["olo"])

    packed = job(0, Nt, ev)
    pairs = float(packed["mask"].visible_pairs)
    t_packed = _time_ms(lambda: run(packed), 3, 1)
    del packed
    torch.cuda.empty_cache()
    sep = []
    for b in range(len(mix)):
        rows = np.concatenate([np.zeros((len(evs[b]), 1), np.int64), evs[b]], axis=1).astype(np.int32)
        sep.append(job(int(cu[b]), int(cu[b + 1]), rows))
    t_sep = _time_ms(lambda: [run(j) for j in sep], 3, 1)
    torch.cuda.synchronize()
    assert st.item() == 0, f"device status {st.item()}"
    tf = 14 * d * pairs * Hq / (t_packed * 1e-3) / 1e12
    return {"workload": "packed: " + ", ".join(f"{c.name} ({c.n_tokens})" for c in mix) +
                        f"; Hq={Hq}, Hkv={Hkv}, d={d}",
            "tokens": Nt, "visible_pairs": pairs, "packed_ms": t_packed, "separate_ms": t_sep,
            "fwd_bwd_tflops": tf, "frac_bf16_sustained": tf / float(peaks.get("bf16_tflops_sustained", 1400.0))}


def per_config(dev, peaks, scale: int = 1):
    """Throughput on the other configurations at 1 GPU, each kernel timed alone
    with CUDA events: configuration 2 forward, configuration 3 forward + backward
    (TFLOP/s on visible pairs), configuration 4 paged decode (GB/s)."""
    out = {"cfg2_fwd": _attn_config(2, dev, peaks, bwd=False, scale=scale)}
    torch.cuda.empty_cache()
    out["cfg3_fwd_bwd"] = _attn_config(3, dev, peaks, bwd=True, scale=scale)
    torch.cuda.empty_cache()
    out["cfg4_decode"], out["decode_sweep"] = _paged_config(dev, peaks)
    torch.cuda.empty_cache()
    out["packed_policy_mix"] = _packed_config(dev, peaks, scale)
    torch.cuda.empty_cache()
    rp = _reprefill_config(dev, scale)
    rp["kvstreams_compact_us_cfg4"] = out["cfg4_decode"]["compact_us"]
    out["reprefill_vs_kvstreams"] = rp
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))
    cfg = workload_cfg(args.scale)
    step = Step(cfg, rank, dev)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.5)
    rec = {}
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step.run(rec)
    t1.record()
    torch.cuda.synchronize()
    elapsed = t0.elapsed_time(t1)
    clk = clocks.stop() if clocks else None
    elapsed, pairs_all = over_ranks(elapsed, float(step.pairs), dev)
    assert step.status.item() == 0, f"device status {step.status.item()}"
    ms = elapsed / args.steps
    flops_step = FLOPS_PER_PAIR_D * cfg.d * pairs_all * cfg.hq
    value = flops_step / (ms * 1e-3) / 1e12
    dur = _durations(rec)
    peaks = _peaks()

    # e2e: same step through the public API with inputs from pinned host memory,
    # gradients and the decode output read back
    e2e = None
    if not args.no_e2e:
        e2e = _e2e(step, args, flops_step)

    line = None
    if rank == 0:
        d, Hq = cfg.d, cfg.hq
        P = float(step.pairs)
        alg = {"fwd": 4 * d * P * Hq, "dkdv": 8 * d * P * Hq, "dq": 2 * d * P * Hq}
        dom = max(alg, key=lambda k: dur[k])
        achieved = alg[dom] / (dur[dom] * 1e-3) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", 1400.0))
        srcs = {"fwd": ["attn_fwd_tc.cu", "common.cuh"], "dkdv": ["attn_bwd_tc.cu", "common.cuh"],
                "dq": ["attn_bwd_tc.cu", "common.cuh"]}[dom]
        tr = TRAFFIC.get(dom)
        traffic = None
        if tr and tr[2] == _src_hash(srcs):
            traffic = tr[0] * (P * Hq / tr[1])
        dec_b = step.decode_bytes()
        dec_gbs = dec_b / (dur["decode"] * 1e-3) / 1e9
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            ntok = CPU_SAMPLE_TOKENS
            f, s, thr = oracle_sample(cfg, ntok)
            cpu = cpu_baseline_entry(f, s, thr, flops_step,
                                     f"first {ntok} tokens of trace 0, one kv group (8 query heads), "
                                     f"fwd + full bwd, {s:.1f} s")
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(cfg, world, len(step.ev_host), P),
            "roofline": {"bound": "tensor", "kernel": {"fwd": "k_attn_fwd_tc", "dkdv": "k_attn_dkdv_tc",
                                                       "dq": "k_attn_dq_tc"}[dom],
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_kind": "measured bf16 sustained" if "fallback" not in peaks else "fallback",
                         "traffic": traffic},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": step.launches() * args.steps,
            "clocks": clk,
            "ms": {k: round(v, 3) for k, v in dur.items()},
            "fwd_tflops": 4 * cfg.d * P * Hq / (dur["fwd"] * 1e-3) / 1e12,
            "bwd_tflops": 10 * cfg.d * P * Hq / ((dur["bwd_prep"] + dur["dkdv"] + dur["dq"]) * 1e-3) / 1e12,
            "decode": {"gbs": dec_gbs, "bytes": dec_b, "frac_hbm_measured": dec_gbs / peaks["hbm_gbs"],
                       "frac_8tbs": dec_gbs / 8000.0},
        }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if line is not None:
        if not args.no_per_config:
            del step
            torch.cuda.empty_cache()
            line["per_config"] = per_config(dev, peaks, args.scale)
        print(json.dumps(line), flush=True)


IN_NAMES = ("events", "q_raw", "k_raw", "v", "do")     # a step's inputs (copied in this order)
N_FWD_IN = 4                                             # the first four feed the forward
OUT_NAMES = ("dq_raw", "dk_raw", "dv", "o_dec")          # a step's results


def _e2e(step, args, flops_step):
    """Every step copies its inputs (raw q, k, v, dO, event log) from pinned host
    memory and reads its results (dq, dk in the pre-RoPE basis, dv, the decode
    output) back, timed with CUDA events from the first copy in to the last copy
    out. Steps are pipelined as a training loop would run them: two sets of device
    inputs and results, the copy of step i+1's inputs on one copy stream and of
    step i-1's results on another while step i computes; a set is refilled only
    after the step that read it has finished. Within a step the forward starts once
    its inputs (event log, q, k, v) are in; the backward also waits for dO."""
    ins = [getattr(step, n) for n in IN_NAMES]
    outs = [getattr(step, n) for n in OUT_NAMES]
    h_in = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ins]
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    for h, t in zip(h_in, ins):
        h.copy_(t)
    sets = [(ins, outs), ([torch.empty_like(t) for t in ins], [torch.empty_like(t) for t in outs])]
    n = max(3, args.steps)  # as many steps as the device-timed region: fill and drain amortise alike
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, in_free, out_ready, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]
    fwd_ready = [ev(), ev()]
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(h2d)
    for i in range(n):
        k = i % 2
        s_in, s_out = sets[k]
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(in_free[k])
            for j, (h, t) in enumerate(zip(h_in, s_in)):
                t.copy_(h, non_blocking=True)
                if j == N_FWD_IN - 1:
                    fwd_ready[k].record(h2d)
            in_ready[k].record(h2d)
        comp.wait_event(fwd_ready[k])
        if i >= 2:
            comp.wait_event(out_free[k])
        for nm, t in zip(IN_NAMES + OUT_NAMES, s_in + s_out):
            setattr(step, nm, t)
        step.run(bwd_wait=in_ready[k])
        in_free[k].record(comp)
        out_ready[k].record(comp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(out_ready[k])
            for h, t in zip(h_out, s_out):
                h.copy_(t, non_blocking=True)
            out_free[k].record(d2h)
    e.record(d2h)
    torch.cuda.synchronize()
    for nm, t in zip(IN_NAMES + OUT_NAMES, ins + outs):
        setattr(step, nm, t)
    ms = s.elapsed_time(e) / n
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        t = torch.tensor([ms], device=step.dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return {"value": flops_step / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in ins)),
            "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in outs)),
            "ms_per_step": ms, "steps": n,
            "pipelined": "copies of step i+1 in and i-1 out overlap step i; dO's copy overlaps the forward"}


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
