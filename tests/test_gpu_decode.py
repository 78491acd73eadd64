"""GPU parity of the split-KV decode (per-chunk partials, intra-chunk
sub-split combine, the (O, lse) merge) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import oracle
import workloads as W
from oracle import merge as omerge
from tests.helpers import margin, TOL_BF16_LSE, TOL_BF16_OUT, host, need_cuda

pytestmark = pytest.mark.gpu


def oracle_decode(q, k, v, lens, scale, heads=None, chunk=None):
    """Per (b, hq): attention of the single query over keys j < lens[b]
    (restricted to [p*chunk, (p+1)*chunk) when chunk=(p, C))."""
    qh, B = host(q), q.shape[0]
    Hq, Hkv = q.shape[1], k.shape[2]
    G = Hq // Hkv
    outs, lses = {}, {}
    for b in range(B):
        for g in range(Hkv):
            hs = [h for h in range(g * G, (g + 1) * G) if heads is None or (b, h) in heads]
            if not hs:
                continue
            L = int(lens[b])
            lo, hi = (0, k.shape[1]) if chunk is None else (chunk[0] * chunk[1], (chunk[0] + 1) * chunk[1])
            ks = host(k[b:b + 1, lo:hi, g:g + 1])
            vs = host(v[b:b + 1, lo:hi, g:g + 1])
            kl = np.array([max(0, min(L - lo, hi - lo))])
            qq = qh[b:b + 1, None, g * G:(g + 1) * G, :]
            rows = [(0, h - g * G, 0) for h in hs]
            o, l = oracle.attention_rows(qq, ks, vs, rows, scale=scale, causal=False, kv_len=kl)
            for n, h in enumerate(hs):
                outs[(b, h)] = o[n]
                lses[(b, h)] = l[n]
    return outs, lses


def make(B, Hq, Hkv, cap, lens, seed):
    cfg = W.Decode("t", B, Hq, Hkv, 128, cap, 1, seed, fixed_lens=tuple(lens))
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    return cfg, q, k, v, sl


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 2), (3, 3), (16, 2), (32, 2)])   # G = 4, 2, 1, 8, 16
def test_decode_small(Hq, Hkv):
    need_cuda()
    lens = [0, 1, 5000, 8192, 8193, 32768, 12345, 20000]
    cfg, q, k, v, sl = make(len(lens), Hq, Hkv, 32768, lens, 61)
    P = 4
    ws = ra.decode_workspace(cfg.B, Hq, Hkv, cfg.capacity, 128, P)
    part, plse = ra.ring_attn_decode_partial(q, k, v, sl, P, cfg.scale, workspace=ws)
    out, out_lse = ra.ring_attn_merge(part, plse)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    C = cfg.capacity // P
    # per-chunk partials: the oracle over each chunk's valid keys
    for p in range(P):
        ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale, chunk=(p, C))
        for (b, h), ro in ref_o.items():
            rl = ref_l[(b, h)]
            gl = float(host(plse)[b, h, p])
            if np.isneginf(rl):
                assert np.isneginf(gl) and np.all(host(part)[b, h, p] == 0)
            else:
                margin("lse", abs(gl - rl), TOL_BF16_LSE)
                margin("out", np.max(np.abs(host(part)[b, h, p] - ro)), TOL_BF16_OUT)
    # merged result: attention over all valid keys
    ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale)
    for (b, h), ro in ref_o.items():
        if lens[b] == 0:
            assert np.isneginf(host(out_lse)[b, h]) and np.all(host(out)[b, h] == 0)
            continue
        margin("lse", abs(host(out_lse)[b, h] - ref_l[(b, h)]), TOL_BF16_LSE)
        margin("out", np.max(np.abs(host(out)[b, h] - ro)), TOL_BF16_OUT)
    # the arrival counters are back at zero: a second call on the same workspace agrees
    out2, lse2 = ra.ring_attn_decode(q, k, v, sl, P, cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out2, out) and torch.equal(lse2, out_lse)



@pytest.mark.parametrize("fused", [False, True])
def test_decode_ignores_rows_past_the_length(fused):
    # A cache's rows past a sequence's length may hold anything (here NaN and Inf): they get
    # weight 0 and must not reach the result (0 x NaN would).  The oracle reads valid rows only.
    need_cuda()
    lens = [1, 300, 4096, 4097, 6000, 8191]
    cfg, q, k, v, sl = make(len(lens), 8, 2, 8192, lens, 83)
    P = 2
    kg, vg = k.clone(), v.clone()
    for b, L in enumerate(lens):
        kg[b, L:] = float("nan")
        vg[b, L:] = float("inf") if b % 2 else float("nan")
    ws = ra.decode_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.capacity, 128, P)
    if fused:
        out, out_lse = ra.ring_attn_decode_fused(q, kg, vg, P, seqlens=sl, scale=cfg.scale, workspace=ws)
    else:
        out, out_lse = ra.ring_attn_decode(q, kg, vg, sl, P, cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    assert np.all(np.isfinite(host(out))) and np.all(np.isfinite(host(out_lse)))
    ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale)
    for (b, h), ro in ref_o.items():
        margin("lse", abs(host(out_lse)[b, h] - ref_l[(b, h)]), TOL_BF16_LSE)
        margin("out", np.max(np.abs(host(out)[b, h] - ro)), TOL_BF16_OUT)


@pytest.mark.parametrize("Hq,Hkv,P", [(8, 2, 3), (16, 2, 1), (16, 1, 2)])   # G = 4, 8, 16
@pytest.mark.parametrize("fused", [False, True])
def test_decode_head_dim_64(Hq, Hkv, P, fused):
    # D = 64: one 64-column block per K/V row; with P = 1 the 24576-row chunk spans 3 sub-splits
    need_cuda()
    lens = [1, 300, 8192, 8193, 20000, 24576]
    cfg = W.Decode("d64", len(lens), Hq, Hkv, 64, 24576, P, 97, fixed_lens=tuple(lens))
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    ws = ra.decode_workspace(cfg.B, Hq, Hkv, cfg.capacity, 64, P)
    if fused:
        out, out_lse = ra.ring_attn_decode_fused(q, k, v, P, seqlens=sl, scale=cfg.scale, workspace=ws)
    else:
        out, out_lse = ra.ring_attn_decode(q, k, v, sl, P, cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale)
    for (b, h), ro in ref_o.items():
        margin("lse", abs(host(out_lse)[b, h] - ref_l[(b, h)]), TOL_BF16_LSE)
        margin("out", np.max(np.abs(host(out)[b, h] - ro)), TOL_BF16_OUT)

def test_merge_kernel_against_oracle_formula():
    need_cuda()
    g = torch.Generator(device="cuda").manual_seed(71)
    B, Hq, P, D = 3, 5, 37, 128
    part = torch.randn((B, Hq, P, D), generator=g, device="cuda")
    plse = torch.randn((B, Hq, P), generator=g, device="cuda") * 4
    plse[0, 1, ::3] = float("-inf")
    plse[2, 4, :] = float("-inf")           # every part empty
    for dt in (torch.float32, torch.bfloat16):
        out, lse = ra.ring_attn_merge(part, plse, dtype=dt)
        ro, rl = omerge.merge(host(part), host(plse))
        tol = 1e-5 if dt == torch.float32 else TOL_BF16_OUT
        margin("out", np.max(np.abs(host(out) - ro)), tol)
        fin = np.isfinite(rl)
        assert np.max(np.abs(host(lse)[fin] - rl[fin])) <= 1e-5
        assert np.all(np.isneginf(host(lse)[~fin]))


@pytest.mark.parametrize("P,D", [(1, 128), (7, 64), (32, 128), (37, 96), (100, 128)])
def test_merge_part_counts_head_sizes_and_nan_in_empty_parts(P, D):
    # part counts around the kernel's 32-part weight blocks and 8-deep load batches, head sizes
    # that leave lanes idle (64, 96 dims for 32 lanes of 4), and empty parts (lse = -inf) whose O
    # holds NaN: an empty part must not enter the sum whatever its O holds.  The oracle gets the
    # same parts with those O set to zero (what the decode writes for an empty chunk).
    need_cuda()
    mc = W.Merge(f"merge_P{P}_D{D}", 3, 5, P, D, 72 + P, empty_frac=0.3)
    part, plse = W.merge_inputs(mc, "cuda")
    plse[1, 2, :] = float("-inf")            # one row with every part empty
    part[1, 2] = float("nan")
    ref_part = torch.nan_to_num(part, nan=0.0)
    ro, rl = omerge.merge(host(ref_part), host(plse))
    for dt in (torch.float32, torch.bfloat16):
        out, lse = ra.ring_attn_merge(part, plse, dtype=dt)
        torch.cuda.synchronize()
        assert np.all(np.isfinite(host(out)))
        margin("out", np.max(np.abs(host(out) - ro)), 1e-5 if dt == torch.float32 else TOL_BF16_OUT, str(dt))
        fin = np.isfinite(rl)
        margin("lse", np.max(np.abs(host(lse)[fin] - rl[fin])), 1e-5, str(dt))
        assert np.all(np.isneginf(host(lse)[~fin])) and np.all(host(out)[~fin] == 0)


def test_merge_only_workload_every_row():
    # the merge alone at the size bench.py times (B*Hq = 8192 rows, P = 32, D = 128, 134 MB of
    # partials), every row against the merge formula
    need_cuda()
    mc = W.MERGE_ONLY
    part, plse = W.merge_inputs(mc, "cuda")
    out, lse = ra.ring_attn_merge(part, plse, dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ro, rl = omerge.merge(host(part), host(plse))
    margin("out", np.max(np.abs(host(out) - ro)), TOL_BF16_OUT)
    margin("lse", np.max(np.abs(host(lse) - rl)), 1e-5)


def test_cfg5_full_size_sampled():
    # KV-sharded decode at full size: B8, Hq32, Hkv8, D128, 2^20 context, P=32, lengths U[0.5M, 1M].
    # One seeded kv head per sequence (all its query heads): the 32 per-chunk partials (O_p, lse_p)
    # and the merged result, each against the oracle over the same keys
    need_cuda()
    cfg = W.CFG5
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    part = torch.empty((cfg.B, cfg.Hq, cfg.P, cfg.D), device="cuda", dtype=torch.float32)
    plse = torch.empty((cfg.B, cfg.Hq, cfg.P), device="cuda", dtype=torch.float32)
    out, out_lse = ra.ring_attn_decode(q, k, v, sl, cfg.P, cfg.scale, partials=part, part_lse=plse)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    lens = host(sl).astype(np.int64)
    rng = np.random.default_rng(cfg.seed + 1000)
    G = cfg.Hq // cfg.Hkv
    groups = {b: int(rng.integers(cfg.Hkv)) for b in range(cfg.B)}   # one kv head per sequence, all its q heads
    heads = {(b, g * G + i) for b, g in groups.items() for i in range(G)}
    hp, hl = host(part), host(plse)
    C = cfg.capacity // cfg.P
    for p in range(cfg.P):
        ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale, heads=heads, chunk=(p, C))
        for (b, h), ro in ref_o.items():
            if np.isneginf(ref_l[(b, h)]):      # a chunk past the sequence's length
                assert np.isneginf(hl[b, h, p]) and np.all(hp[b, h, p] == 0)
                continue
            margin("lse", abs(hl[b, h, p] - ref_l[(b, h)]), TOL_BF16_LSE, "chunk partials")
            margin("out", np.max(np.abs(hp[b, h, p] - ro)), TOL_BF16_OUT, "chunk partials")
    ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale, heads=heads)
    for (b, h), ro in ref_o.items():
        margin("out", np.max(np.abs(host(out)[b, h] - ro)), TOL_BF16_OUT, "merged")
        margin("lse", abs(host(out_lse)[b, h] - ref_l[(b, h)]), TOL_BF16_LSE, "merged")
