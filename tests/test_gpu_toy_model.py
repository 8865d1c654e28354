"""A random-weight two-layer attention model run end to end on the GPU, both ways.

Generation with compaction ("KV-streams: speeding up agentic RL by operating on
the KV cache directly", first and second fix): token by token, every layer
rotates its new query and key at the token's logical position, writes key and
value into its paged cache (one block table shared by the layers, one cache per
layer), attends over the compacted table, and at each event the table loses the
evicted blocks. Training replay (the thread's trainer paragraph; "KV-streams for
Efficient Compaction in Agentic Reinforcement Learning", Fig. 2(A)): layer by
layer over the whole trace under the eviction mask. The thread reports a
train/inference mismatch KL of about 0.001 in its validation runs; here the
two GPU paths (bf16 kernels, fp32 accumulation) are compared token by token
and through the KL of a 64-way output head, and both against the fp64 oracle.

The model's dense projections are test scaffolding computed with torch.matmul
in fp32; every KV-streams step (RoPE at logical positions, cache scatter,
compaction, paged decode, mask compile, masked forward) runs in the library.
"""
import numpy as np
import pytest
import torch

import oracle
import eviction_masked_attention_b200 as kvs
from eviction_masked_attention_b200 import workloads as W
from gpu_util import events_dev, rel_l2

pytestmark = pytest.mark.gpu


def _kl(la, lb):
    """Mean and max over tokens of KL(softmax(la) || softmax(lb)), fp64."""
    pa = torch.log_softmax(la.double(), -1)
    pb = torch.log_softmax(lb.double(), -1)
    kl = (pa.exp() * (pa - pb)).sum(-1)
    return float(kl.mean()), float(kl.max())


def test_toy_two_layer_generation_vs_replay_bf16():
    cfg = W.replace(W.scaled(W.CONFIGS[5], 64), batch=1)      # 1-token blocks, unpadded turns
    ev = W.make_event_log(cfg)
    assert len(ev) >= 3
    N, L, Dm, Hq, Hkv, d = cfg.n_tokens, 2, 64, 8, 2, 128
    theta, bs = cfg.theta, 1
    toy = oracle.Toy(L=L, Dm=Dm, Hq=Hq, Hkv=Hkv, d=d, theta=theta, seed=21)
    x0 = np.random.default_rng(21).standard_normal((N, Dm))
    dev = torch.device("cuda")
    Wq, Wk, Wv, Wo = (torch.from_numpy(w).float().to(dev) for w in (toy.Wq, toy.Wk, toy.Wv, toy.Wo))
    bf = torch.bfloat16
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    # ---------------- replay: layer by layer over the trace under the eviction mask
    gm = kvs.kvs_build_tile_mask(events_dev(ev), 1, N)
    lp = torch.arange(N, dtype=torch.int32, device=dev)
    x = torch.from_numpy(x0).float().to(dev)
    rep_attn = []
    for layer in range(L):
        q = (x @ Wq[layer]).to(bf).view(N, Hq, d)
        k = (x @ Wk[layer]).to(bf).view(N, Hkv, d)
        v = (x @ Wv[layer]).to(bf).view(1, N, Hkv, d)
        qr = kvs.kvs_rope_logical(q, lp, theta, status=status)[None].contiguous()
        kr = kvs.kvs_rope_logical(k, lp, theta, status=status)[None].contiguous()
        o, _, _ = kvs.kvs_masked_attn_fwd(qr, kr, v.contiguous(), gm, toy.scale, status=status, residual=False)
        a = o[0].reshape(N, Hq * d).float()
        rep_attn.append(a)
        x = x + a @ Wo[layer]
    x_rep = x

    # ---------------- generation: token by token with compaction
    pool = N + 8
    M = N + 1
    kc = [torch.zeros((pool, Hkv, bs, d), dtype=bf, device=dev) for _ in range(L)]
    vc = [torch.zeros_like(kc[0]) for _ in range(L)]
    bt = torch.full((1, M), -1, dtype=torch.int32, device=dev)
    bl = torch.full((1, M), -1, dtype=torch.int32, device=dev)
    nb = torch.zeros(1, dtype=torch.int32, device=dev)
    nt = torch.zeros(1, dtype=torch.int32, device=dev)
    freed = torch.full((1, M), -1, dtype=torch.int32, device=dev)
    n_freed = torch.zeros(1, dtype=torch.int32, device=dev)
    free = list(range(pool))
    n_blocks = 0
    by_tau = {}
    for row in ev:
        by_tau.setdefault(int(row[1]), []).append(row)
    gen_attn = [torch.empty((N, Hq * d), device=dev) for _ in range(L)]
    x_gen = torch.empty((N, Dm), device=dev)
    ws = torch.empty(kvs.lib().kvs_paged_decode_ws_bytes(1, Hq, Hkv, d, bs, M), dtype=torch.uint8, device=dev)
    for t in range(N):
        if t in by_tau:
            kvs.kvs_compact_block_table(bt, bl, nb, nt, bs, pool, events_dev(by_tau[t]), freed=freed,
                                        n_freed=n_freed, status=status)
            nf = int(n_freed.item())
            free.extend(freed[0, :nf].tolist())
            n_blocks = int(nb.item())
        blk = free.pop(0)                  # a new 1-token block for the new token
        bt[0, n_blocks] = blk
        bl[0, n_blocks] = t
        n_blocks += 1
        nb.fill_(n_blocks)
        nt.fill_(n_blocks)
        slot = torch.tensor([blk], dtype=torch.int64, device=dev)
        pos = lp[t:t + 1]
        xt = torch.from_numpy(x0[t:t + 1]).float().to(dev)
        for layer in range(L):
            q = (xt @ Wq[layer]).to(bf).view(1, Hq, d)
            k = (xt @ Wk[layer]).to(bf).view(1, Hkv, d)
            v = (xt @ Wv[layer]).to(bf).view(1, Hkv, d)
            kvs.kvs_rope_logical(k, pos, theta, out=kc[layer], out_slot=slot, block_size=bs, v=v,
                                 v_out=vc[layer], status=status)
            qr = kvs.kvs_rope_logical(q, pos, theta, status=status)
            o = kvs.kvs_paged_decode_attn(qr, kc[layer], vc[layer], bt, nt, bs, toy.scale, ws=ws, status=status)
            a = o.reshape(1, Hq * d).float()
            gen_attn[layer][t] = a[0]
            xt = xt + a @ Wo[layer]
        x_gen[t] = xt[0]
    torch.cuda.synchronize()
    assert status.item() == 0, kvs.status_str(status.item())

    # ---------------- the two GPU paths agree token by token, and with the oracle
    head = torch.from_numpy(np.random.default_rng(99).standard_normal((Dm, 64))).float().to(dev)
    kl_mean, kl_max = _kl(x_gen @ head, x_rep @ head)
    print(f"\nKL(generation || replay) over a 64-way head, {N} tokens, {len(ev)} events: "
          f"mean {kl_mean:.3g}, max {kl_max:.3g}")
    assert kl_mean <= 1e-3 and kl_max <= 1e-2
    for layer in range(L):
        rl = rel_l2(gen_attn[layer].cpu().double().numpy(), rep_attn[layer].cpu().double().numpy())
        assert rl is not None and rl <= 2e-2, (layer, rl)
    kap = oracle.kappa(ev, 1, N)
    xo, _ = toy.replay(x0, kap[0])
    for name, xg in (("replay", x_rep), ("generation", x_gen)):
        rl = rel_l2(xg.cpu().double().numpy(), xo)
        assert rl is not None and rl <= 2e-2, (name, rl)
    kl_o, _ = _kl(x_rep @ head, torch.from_numpy(xo).to(dev).float() @ head)
    assert kl_o <= 1e-3
