"""Edge cases of the GPU path against the fp64 oracle: ragged chunks in the
step API, batch > 1 with GQA head pairs, many virtual ranks (one 128-row tile
per chunk), out-of-range decode lengths (clamped), decode chunks that are not
a multiple of the TMA stage, a single decode chunk, and a one-part merge."""
import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import workloads as W
from oracle import merge as omerge
from tests.helpers import margin, TOL_BF16_LSE, TOL_BF16_OUT, TOL_FP32, check_rows, host, need_cuda, oracle_rows
from tests.test_gpu_decode import oracle_decode
from tests.test_gpu_simt import ring_by_steps

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,tol_o,tol_l", [("bf16", TOL_BF16_OUT, TOL_BF16_LSE), ("fp32", TOL_FP32, TOL_FP32)])
def test_steps_ragged_chunks_gqa(dtype, tol_o, tol_l):
    # chunks of 200 tokens (not a multiple of the 128-row tile), GQA group 4 (head pairs), causal zig-zag
    need_cuda()
    cfg = W.Prefill("steps_ragged", dtype, True, "zigzag", 1, 8, 2, 1600, 128, 4, 141)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = ring_by_steps(q, k, v, cfg.P, "zigzag", True, cfg.scale)
    rows = W.sample_rows(cfg, 0)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, True)
    check_rows(out, lse, rows, ref_out, ref_lse, tol_o, tol_l, cfg.name)


@pytest.mark.parametrize("cfg", [
    W.Prefill("batch2_headpairs", "bf16", True, "zigzag", 2, 8, 2, 2048, 128, 4, 142),
    W.Prefill("P64_one_tile_per_chunk", "bf16", True, "zigzag", 1, 2, 1, 16384, 128, 64, 143),
    W.Prefill("contiguous_P1_causal", "bf16", True, "contiguous", 1, 4, 4, 1024, 128, 1, 144),
    W.Prefill("gqa_group8_d64", "bf16", True, "contiguous", 1, 16, 2, 1024, 64, 8, 145),
], ids=lambda c: c.name)
def test_prefill_shapes(cfg):
    need_cuda()
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = ra.ring_attn_fwd(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    rows = W.sample_rows(cfg, 0) if cfg.S <= 4096 else W.sample_rows(cfg, 128)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, cfg.causal)
    check_rows(out, lse, rows, ref_out, ref_lse, TOL_BF16_OUT, TOL_BF16_LSE, cfg.name)


def test_decode_lengths_out_of_range_are_clamped():
    need_cuda()
    cap, P = 4096, 4
    cfg = W.Decode("clamp", 4, 8, 2, 128, cap, P, 151, fixed_lens=(0, 100, 4096, 4096))
    q, k, v, _ = W.decode_inputs(cfg, "cuda")
    bad = torch.tensor([-5, 100, 4096, 999999], dtype=torch.int32, device="cuda")
    out, lse = ra.ring_attn_decode(q, k, v, bad, P, cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    eff = [0, 100, 4096, 4096]           # clamped to [0, Smax]
    ref_o, ref_l = oracle_decode(q, k, v, eff, cfg.scale)
    for (b, h), ro in ref_o.items():
        if eff[b] == 0:
            assert np.isneginf(host(lse)[b, h]) and np.all(host(out)[b, h] == 0)
        else:
            margin("lse", abs(host(lse)[b, h] - ref_l[(b, h)]), TOL_BF16_LSE)
            margin("out", np.max(np.abs(host(out)[b, h] - ro)), TOL_BF16_OUT)


@pytest.mark.parametrize("cap,P,lens", [
    (1000, 4, (1000, 251, 250, 1)),     # chunks of 250 rows: stage boxes straddle chunk ends
    (20480, 1, (20480, 8192, 8193, 16385, 5000)),  # one chunk over 1, 2 or 3 of the kernel's 8192-row sub-splits
])
def test_decode_partials_odd_chunks(cap, P, lens):
    need_cuda()
    cfg = W.Decode("odd", len(lens), 4, 1, 128, cap, P, 152, fixed_lens=lens)
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    part, plse = ra.ring_attn_decode_partial(q, k, v, sl, P, cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    C = cap // P
    for p in range(P):
        ref_o, ref_l = oracle_decode(q, k, v, lens, cfg.scale, chunk=(p, C))
        for (b, h), ro in ref_o.items():
            rl = ref_l[(b, h)]
            if np.isneginf(rl):
                assert np.isneginf(host(plse)[b, h, p])
            else:
                margin("lse", abs(host(plse)[b, h, p] - rl), TOL_BF16_LSE)
                margin("out", np.max(np.abs(host(part)[b, h, p] - ro)), TOL_BF16_OUT)


def test_merge_single_part_is_identity():
    need_cuda()
    g = torch.Generator(device="cuda").manual_seed(161)
    part = torch.randn((2, 3, 1, 128), generator=g, device="cuda")
    plse = torch.randn((2, 3, 1), generator=g, device="cuda")
    out, lse = ra.ring_attn_merge(part, plse, dtype=torch.float32)
    ro, rl = omerge.merge(host(part), host(plse))
    margin("out", np.max(np.abs(host(out) - ro)), TOL_FP32)
    margin("lse", np.max(np.abs(host(lse) - rl)), TOL_FP32)
    np.testing.assert_allclose(host(out), host(part)[:, :, 0], atol=TOL_FP32)
