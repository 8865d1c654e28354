"""GPU parity of packed multi-trace replay: traces of different lengths and
compaction policies (prompt + summary + overlap at several points, Markovian
carry-over, recent turns, oldest turns with 1-token granularity; the paper
listing's Fig. 2(B) and Table 2) packed into one buffer, rotated at per-trace
positions and replayed by one forward and one backward call; every trace's
slice must equal the oracle run on that trace alone."""
import numpy as np
import pytest
import torch

import oracle
import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import packing
from eviction_masked_attention_b200 import workloads as W
from gpu_util import BF16_TOL, F32_ROUND, F32_TOL, GRAD_REL_L2, assert_close, dev, events_dev, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_packed_policy_mix_fwd_bwd(dtype):
    d = 128 if dtype == "bf16" else 64
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    mix = W.policy_mix(hq=8, hkv=2, div=16)
    lengths = [c.n_tokens for c in mix]
    evs = [np.asarray(W.make_trace_events(c, 0), np.int64).reshape(-1, 3) for c in mix]
    cu, ev, lpos = packing.pack(lengths, evs)
    Nt, Hq, Hkv = int(cu[-1]), 8, 2
    G = Hq // Hkv
    rng = np.random.default_rng(17)
    cast = W.round_bf16 if dtype == "bf16" else (lambda a: a)
    q = cast(rng.standard_normal((Nt, Hq, d)).astype(np.float32))
    k = cast(rng.standard_normal((Nt, Hkv, d)).astype(np.float32))
    v = cast(rng.standard_normal((Nt, Hkv, d)).astype(np.float32))
    do = cast(rng.standard_normal((Nt, Hq, d)).astype(np.float32))
    theta, scale = 5e5, 1 / np.sqrt(d)
    lp = dev(lpos)
    qr = kvs.kvs_rope_logical(dev(q, tdt), lp, theta)[None].contiguous()
    kr = kvs.kvs_rope_logical(dev(k, tdt), lp, theta)[None].contiguous()
    gm = kvs.kvs_build_tile_mask(events_dev(ev), 1, Nt)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse, o_lo = kvs.kvs_masked_attn_fwd(qr, kr, dev(v, tdt)[None].contiguous(), gm, scale, status=status)
    dq, dk, dv = kvs.kvs_masked_attn_bwd(qr, kr, dev(v, tdt)[None].contiguous(), o, dev(do, tdt)[None].contiguous(),
                                         lse, gm, scale, status=status, o_lo=o_lo)
    torch.cuda.synchronize()
    assert status.item() == 0
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    for b, n in enumerate(lengths):
        sl = slice(int(cu[b]), int(cu[b + 1]))
        pos = np.arange(n, dtype=np.int32)
        qb = oracle.rope(q[sl].astype(np.float64), pos, theta)[None]
        kb = oracle.rope(k[sl].astype(np.float64), pos, theta)[None]
        rows = np.concatenate([np.zeros((len(evs[b]), 1), np.int64), evs[b]], axis=1)
        kap = oracle.kappa(rows, 1, n)
        wo, wl, wdq, wdk, wdv = oracle.attn_bwd(qb, kb, v[sl][None].astype(np.float64), do[sl][None].astype(np.float64),
                                                kap, scale)
        name = mix[b].name
        assert_close(host(o[0, sl]), wo[0], tol, f"O packed {name}")
        # the attention inputs here are the rotary kernel's bf16 outputs: their rounding
        # (2^-9 per element) moves a score by up to ~2^-8 |q||k| scale, which the
        # exact-input log-sum-exp bound does not cover; bf16 inputs get the bf16 bound
        assert_close(host(lse[0][:, sl]), wl[0], BF16_TOL if dtype == "bf16" else F32_TOL, f"LSE packed {name}",
                     rnd=F32_ROUND)
        for nm, got, want in (("dq", dq, wdq), ("dk", dk, wdk), ("dv", dv, wdv)):
            g_ = host(got[0, sl])
            assert_close(g_, want[0], tol, f"{nm} packed {name}")
            rl = rel_l2(g_, want[0])
            assert rl is None or rl <= GRAD_REL_L2, (nm, name, rl)
