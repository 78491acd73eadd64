"""Helix-style decode completion on the GPU: the round-robin KV append
("NVIDIA unveils Helix Parallelism", KV cache growth) against the oracle's
token-by-token placement (bit-exact cache contents and counters), the fused
one-launch decode (partials plus the last-CTA merge) against the fp64 oracle
and against the two-launch path, decode over appended shards, and the
capacity error."""
import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import oracle
import workloads as W
from oracle import helix
from tests.helpers import margin, TOL_BF16_LSE, TOL_BF16_OUT, host, need_cuda
from tests.test_gpu_decode import oracle_decode

pytestmark = pytest.mark.gpu


def _tokens(B, T, Hkv, D, seed, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = torch.randn((B, T, Hkv, D), generator=g, device="cuda").to(dtype)
    v = torch.randn((B, T, Hkv, D), generator=g, device="cuda").to(dtype)
    return k, v


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("P,block,T,calls", [(4, 16, 40, 3), (8, 1, 5, 4), (3, 64, 200, 2), (32, 64, 130, 1)])
def test_append_matches_round_robin_simulation(dtype, P, block, T, calls):
    need_cuda()
    B, Hkv, D, Smax = 2, 2, 128, P * 2048
    C = Smax // P
    kc = torch.zeros((B, Smax, Hkv, D), device="cuda", dtype=dtype)
    vc = torch.zeros_like(kc)
    rng = np.random.default_rng(P * 1000 + T)
    lens0 = rng.integers(0, C // 4, size=(B, P)).astype(np.int32)   # a prompt already spread over the shards
    nap0 = np.array([0, 5], dtype=np.int32)
    shard_lens = torch.from_numpy(lens0).cuda()
    n_app = torch.from_numpy(nap0).cuda()
    sims = [[[("p", b, p, r) for r in range(lens0[b, p])] for p in range(P)] for b in range(B)]
    nsim = [int(x) for x in nap0]
    news = []
    for c in range(calls):
        kn, vn = _tokens(B, T, Hkv, D, 300 + c, dtype)
        news.append((host(kn), host(vn)))
        ra.ring_attn_kv_append(kc, vc, kn, vn, shard_lens, n_app, P, block)
        for b in range(B):
            sims[b], nsim[b], _, dropped = helix.simulate_appends(sims[b], nsim[b], [("n", c, b, j) for j in range(T)],
                                                                  block, P, C)
            assert dropped == 0
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    assert host(n_app).astype(int).tolist() == nsim
    assert host(shard_lens).astype(int).tolist() == [[len(s) for s in sims[b]] for b in range(B)]
    kh, vh = host(kc), host(vc)
    for b in range(B):
        for p in range(P):
            for r, tok in enumerate(sims[b][p]):
                if tok[0] == "n":
                    _, c, _, j = tok
                    assert np.array_equal(kh[b, p * C + r], news[c][0][b, j])
                    assert np.array_equal(vh[b, p * C + r], news[c][1][b, j])
            # nothing written past the fill count
            assert not kh[b, p * C + len(sims[b][p]):(p + 1) * C].any()


def test_append_capacity_error_and_no_overrun():
    need_cuda()
    B, P, Hkv, D, Smax, block = 1, 2, 1, 128, 64, 4
    C = Smax // P
    kc = torch.zeros((B, Smax, Hkv, D), device="cuda", dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    shard_lens = torch.tensor([[C - 2, C - 6]], dtype=torch.int32, device="cuda")
    n_app = torch.zeros(1, dtype=torch.int32, device="cuda")
    kn, vn = _tokens(B, 12, Hkv, D, 7)
    ra.ring_attn_kv_append(kc, vc, kn, vn, shard_lens, n_app, P, block)
    st, site = ra.ring_attn_device_error()
    assert st == ra.RING_ECAPACITY and site == 0x100
    sims = [[None] * (C - 2), [None] * (C - 6)]
    sims, n, placements, dropped = helix.simulate_appends(sims, 0, list(range(12)), block, P, C)
    assert dropped > 0
    assert host(shard_lens).astype(int).tolist() == [[len(s) for s in sims]]
    assert int(host(n_app)[0]) == n
    kh = host(kc)
    for j, pl in enumerate(placements):
        if pl is not None:
            p, r = pl
            assert np.array_equal(kh[0, p * C + r], host(kn)[0, j])
    # the context is still usable and the word is clear again
    assert ra.ring_attn_device_error()[0] == ra.RING_OK


def _fused_vs_oracle(q, k, v, sl, P, scale, lens):
    out, lse = ra.ring_attn_decode_fused(q, k, v, P, seqlens=sl, scale=scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    ref_o, ref_l = oracle_decode(q, k, v, lens, scale)
    oh, lh = host(out), host(lse)
    for (b, h), ro in ref_o.items():
        if np.isneginf(ref_l[(b, h)]):
            assert np.isneginf(lh[b, h]) and not oh[b, h].any()
        else:
            margin("lse", abs(lh[b, h] - ref_l[(b, h)]), TOL_BF16_LSE)
            margin("out", np.max(np.abs(oh[b, h] - ro)), TOL_BF16_OUT)
    return out, lse


@pytest.mark.parametrize("Hq,Hkv,cap,P,lens", [
    (8, 2, 8192, 4, (8192, 5000, 1, 0)),
    (8, 4, 12000, 3, (12000, 7777, 4032, 4033)),
    (2, 2, 4096, 1, (4096, 100)),
    (16, 4, 16384, 16, (16384, 3, 9000, 16383)),
    (16, 2, 8192, 2, (8192, 4097, 130)),      # G = 8
    (16, 1, 4096, 4, (4096, 1025)),           # G = 16
    (8, 2, 24576, 1, (24576, 8193, 17000)),   # chunks over 3, 2, 3 sub-splits, folded before the merge
])
def test_fused_decode_against_oracle_and_two_launch_path(Hq, Hkv, cap, P, lens):
    need_cuda()
    cfg = W.Decode("fused", len(lens), Hq, Hkv, 128, cap, P, 311, fixed_lens=lens)
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    out, lse = _fused_vs_oracle(q, k, v, sl, P, cfg.scale, lens)
    # the same partials as the two-launch path, and the same merged values
    o2, l2 = ra.ring_attn_decode(q, k, v, sl, P, cfg.scale)
    torch.cuda.synchronize()
    assert (out.float() - o2.float()).abs().max().item() <= 1e-2
    fin = torch.isfinite(l2)
    assert torch.equal(fin, torch.isfinite(lse)) and (lse[fin] - l2[fin]).abs().max().item() <= 1e-5


def test_fused_decode_twice_on_one_workspace():
    need_cuda()
    cfg = W.Decode("twice", 3, 8, 2, 128, 16384, 8, 312, fixed_lens=(16384, 9000, 40))
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    ws = ra.decode_workspace(3, 8, 2, 16384, 128, 8)
    o1, l1 = ra.ring_attn_decode_fused(q, k, v, 8, seqlens=sl, scale=cfg.scale, workspace=ws)
    o2, l2 = ra.ring_attn_decode_fused(q, k, v, 8, seqlens=sl, scale=cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert not ws.any()   # every counter back at zero


def test_fused_decode_full_size_sampled():
    # B8 Hq32 Hkv8 D128, 2^20-token capacity in 32 chunks: sampled heads against the oracle
    need_cuda()
    cfg = W.CFG5
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    out, lse = ra.ring_attn_decode_fused(q, k, v, cfg.P, seqlens=sl, scale=cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    heads = {(b, (5 * b + 3) % cfg.Hq) for b in range(cfg.B)}
    lens = host(sl).astype(int)
    ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale, heads=heads)
    for (b, h), ro in ref_o.items():
        margin("lse", abs(host(lse)[b, h] - ref_l[(b, h)]), TOL_BF16_LSE)
        margin("out", np.max(np.abs(host(out)[b, h] - ro)), TOL_BF16_OUT)


@pytest.mark.parametrize("P,block,steps,T", [(4, 8, 6, 7), (8, 32, 3, 50), (2, 1, 5, 3)])
def test_decode_after_round_robin_appends(P, block, steps, T):
    # prompt spread contiguously over the shards, then `steps` appends of T tokens; the fused decode
    # over shard_lens must equal attention over exactly the stored tokens
    need_cuda()
    B, Hq, Hkv, D, Smax = 2, 8, 2, 128, 16384
    C = Smax // P
    g = torch.Generator(device="cuda").manual_seed(400 + P)
    kc = torch.zeros((B, Smax, Hkv, D), device="cuda", dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    prompt = [3000, 1234]
    lens = np.zeros((B, P), dtype=np.int32)
    for b, L in enumerate(prompt):
        kp = torch.randn((L, Hkv, D), generator=g, device="cuda").to(torch.bfloat16)
        vp = torch.randn((L, Hkv, D), generator=g, device="cuda").to(torch.bfloat16)
        per = -(-L // P)
        for p in range(P):
            lo, hi = p * per, min(L, (p + 1) * per)
            if hi > lo:
                kc[b, p * C:p * C + hi - lo] = kp[lo:hi]
                vc[b, p * C:p * C + hi - lo] = vp[lo:hi]
                lens[b, p] = hi - lo
    shard_lens = torch.from_numpy(lens).cuda()
    n_app = torch.zeros(B, dtype=torch.int32, device="cuda")
    for s in range(steps):
        kn, vn = _tokens(B, T, Hkv, D, 500 + s)
        ra.ring_attn_kv_append(kc, vc, kn, vn, shard_lens, n_app, P, block)
    q = torch.randn((B, Hq, D), generator=g, device="cuda").to(torch.bfloat16)
    scale = 1 / np.sqrt(D)
    out, lse = ra.ring_attn_decode_fused(q, kc, vc, P, shard_lens=shard_lens, scale=scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    sl = host(shard_lens).astype(int)
    assert sl.sum(axis=1).tolist() == [L + steps * T for L in prompt]
    G = Hq // Hkv
    for b in range(B):
        rows = np.concatenate([np.arange(p * C, p * C + sl[b, p]) for p in range(P)])
        ks, vs = host(kc)[b:b + 1, rows], host(vc)[b:b + 1, rows]
        for gk in range(Hkv):
            qq = host(q)[b:b + 1, None, gk * G:(gk + 1) * G]
            o, l = oracle.attention_rows(qq, ks[:, :, gk:gk + 1], vs[:, :, gk:gk + 1],
                                         [(0, h, 0) for h in range(G)], scale=scale, causal=False)
            for h in range(G):
                margin("lse", abs(host(lse)[b, gk * G + h] - l[h]), TOL_BF16_LSE)
                margin("out", np.max(np.abs(host(out)[b, gk * G + h] - o[h])), TOL_BF16_OUT)
