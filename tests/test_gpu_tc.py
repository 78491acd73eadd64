"""GPU parity of the tensor-core (tcgen05) ring attention against the fp64
oracle: small shapes on every row, the full-size workloads on the rows the
oracle can afford (every row of the contiguous S=8192 workload; 256 sampled
rows per head at S=32768 and S=131072), the S=131072 workload through the
step API (sampled rows against the oracle, every row against the fused
ring), device work counters against the oracle's schedule enumeration, and
the SIMT cross-check."""
import dataclasses

import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import workloads as W
from oracle import schedule as sch
from tests.helpers import margin, TOL_BF16_LSE, TOL_BF16_OUT, check_rows, host, need_cuda, oracle_rows
from tests.test_gpu_simt import ring_by_steps

pytestmark = pytest.mark.gpu

SMALL = [
    W.Prefill("noncausal_P1", "bf16", False, "contiguous", 1, 2, 2, 256, 128, 1, 101),
    W.Prefill("causal_contig_P2", "bf16", True, "contiguous", 1, 2, 2, 512, 128, 2, 102),
    W.Prefill("zigzag_gqa_P4", "bf16", True, "zigzag", 1, 8, 2, 2048, 128, 4, 103),
    W.Prefill("zigzag_mha_keysx8", "bf16", True, "zigzag", 2, 4, 4, 4096, 128, 4, 104, keys_x8=True),
    W.Prefill("contig_gqa_d64", "bf16", True, "contiguous", 1, 4, 2, 1024, 64, 4, 105),
    W.Prefill("ragged_chunks_200", "bf16", True, "zigzag", 1, 3, 3, 1200, 128, 3, 106),
    W.Prefill("ragged_noncausal_odd_group", "bf16", False, "zigzag", 2, 6, 2, 1400, 128, 7, 107),
    W.Prefill("tiny_S48", "bf16", True, "zigzag", 1, 2, 1, 48, 128, 2, 108),
]


def run(cfg, rows=None, fn=ra.ring_attn_fwd):
    need_cuda()
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = fn(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    rows = W.sample_rows(cfg) if rows is None else rows
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, cfg.causal)
    return check_rows(out, lse, rows, ref_out, ref_lse, TOL_BF16_OUT, TOL_BF16_LSE, cfg.name)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_every_row(cfg):
    run(cfg, rows=W.sample_rows(cfg, 0))


def test_against_simt_every_row():
    # GPU vs GPU on every row of a mid-size zig-zag GQA case (independent kernels, same inputs)
    need_cuda()
    cfg = W.Prefill("mid", "bf16", True, "zigzag", 1, 16, 4, 16384, 128, 8, 111)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    o1, l1 = ra.ring_attn_fwd(q, k, v, cfg.P, True, "zigzag", cfg.scale)
    o2, l2 = ra.ring_attn_fwd_simt(q, k, v, cfg.P, True, "zigzag", cfg.scale)
    torch.cuda.synchronize()
    margin("out", (o1.float() - o2.float()).abs().max().item(), TOL_BF16_OUT)
    margin("lse", (l1 - l2).abs().max().item(), TOL_BF16_LSE)


def test_cfg2_full_size_every_row():
    # causal contiguous split, B1 H8 S8192 D128 P8 (rank i does i+1 chunk pairs)
    run(W.CFG2, rows=W.sample_rows(W.CFG2, 0))


def test_cfg3_full_size_sampled():
    # causal zig-zag, B2 H16 S32768 D128 P8, 1% of key rows x8
    run(W.CFG3)


def test_cfg4_full_size_sampled():
    # causal zig-zag GQA, B1 Hq32 Hkv8 S131072 D128 P16: the timed workload
    run(W.CFG4)


def test_cfg4_full_size_through_the_step_api():
    # the timed workload as 16 ranks x 16 hops of ring_attn_step (state in HBM): sampled rows
    # against the oracle, and every row against the fused ring of the same inputs
    need_cuda()
    cfg = W.CFG4
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = ring_by_steps(q, k, v, cfg.P, cfg.layout, cfg.causal, cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    rows = W.sample_rows(cfg, 2)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, cfg.causal)
    check_rows(out, lse, rows, ref_out, ref_lse, TOL_BF16_OUT, TOL_BF16_LSE, "steps")
    fo, fl = ra.ring_attn_fwd(q, k, v, cfg.P, causal=True, layout=cfg.layout, scale=cfg.scale)
    torch.cuda.synchronize()
    margin("out", (out.float() - fo.float()).abs().max().item(), TOL_BF16_OUT, "steps vs fused, every row")
    margin("lse", (lse - fl).abs().max().item(), TOL_BF16_LSE, "steps vs fused, every row")


@pytest.mark.parametrize("cfg", [W.CFG2, W.CFG3, W.CFG4,
                                 W.Prefill("ragged_counts", "bf16", True, "zigzag", 1, 3, 3, 1200, 128, 3, 106),
                                 W.Prefill("noncausal_counts", "bf16", False, "contiguous", 1, 2, 2, 1024, 128, 4, 7)],
                         ids=lambda c: c.name)
def test_device_counters_equal_schedule_enumeration(cfg):
    need_cuda()
    q, k, v = W.prefill_inputs(dataclasses.replace(cfg, S=cfg.S), "cuda")
    _, _, cnt = ra.ring_attn_fwd_counted(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    torch.cuda.synchronize()
    cnt = host(cnt).astype(np.int64) if cnt.dtype != torch.int64 else cnt.cpu().numpy()
    full, partial, _, _ = sch.tile_classes(cfg.S, cfg.P, cfg.layout, cfg.causal, 128, 128)
    heads = cfg.B * cfg.Hq
    assert int(cnt[0]) == full * heads and int(cnt[1]) == partial * heads
    pairs = sch.per_rank_pairs(cfg.P, cfg.layout, cfg.causal)
    assert [int(x) for x in cnt[2:]] == [p_ * heads for p_ in pairs]
    if cfg.causal and cfg.layout == "contiguous":
        assert pairs == [r + 1 for r in range(cfg.P)]
    if cfg.causal and cfg.layout == "zigzag":
        assert pairs == [2 * cfg.P + 1] * cfg.P


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_ring_steps_bf16(layout):
    need_cuda()
    cfg = W.Prefill("steps", "bf16", True, layout, 1, 4, 2, 2048, 128, 4, 121)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = ring_by_steps(q, k, v, cfg.P, layout, True, cfg.scale)
    rows = W.sample_rows(cfg, 0)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, True)
    check_rows(out, lse, rows, ref_out, ref_lse, TOL_BF16_OUT, TOL_BF16_LSE, "bf16 steps")


def test_ring_steps_bf16_shuffled_and_checkpoint():
    need_cuda()
    import random
    cfg = W.Prefill("steps_shuf", "bf16", False, "zigzag", 2, 2, 2, 1024, 64, 4, 122)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    rng = random.Random(3)
    out, lse = ring_by_steps(q, k, v, cfg.P, "zigzag", False, cfg.scale,
                             order_fn=lambda s: rng.sample(s, len(s)), checkpoint_at=2)
    rows = W.sample_rows(cfg, 0)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, False)
    check_rows(out, lse, rows, ref_out, ref_lse, TOL_BF16_OUT, TOL_BF16_LSE, "bf16 shuffled steps")


def test_p_independence():
    # the result does not depend on how many virtual ranks share the work
    need_cuda()
    base = W.Prefill("pind", "bf16", True, "zigzag", 1, 4, 4, 8192, 128, 1, 131)
    q, k, v = W.prefill_inputs(base, "cuda")
    outs = []
    for P in (1, 2, 4, 8, 16):
        o, l = ra.ring_attn_fwd(q, k, v, P, True, "zigzag", base.scale)
        outs.append((o.float(), l))
    oc, lc = ra.ring_attn_fwd(q, k, v, 8, True, "contiguous", base.scale)
    outs.append((oc.float(), lc))
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        margin("out", (o - outs[0][0]).abs().max().item(), TOL_BF16_OUT)
        margin("lse", (l - outs[0][1]).abs().max().item(), TOL_BF16_LSE)


# D = 128 runs on CTA pairs (tcgen05 cta_group::2) by default; RING_ATTN_TC_KERNEL=single selects
# the one-CTA kernel.  Both are checked against the oracle on the item shapes the pair kernel
# forms differently: four heads (group 4), two heads at two row tiles (group 2), four row tiles
# (group 1 and 3), ragged chunks, the striped split, and the step API.
BOTH = [
    W.Prefill("pair_group4_zigzag", "bf16", True, "zigzag", 1, 8, 2, 2048, 128, 4, 131),
    W.Prefill("pair_group2_ragged", "bf16", True, "zigzag", 2, 4, 2, 1200, 128, 3, 132),
    W.Prefill("pair_group1_keysx8", "bf16", True, "zigzag", 1, 2, 2, 4096, 128, 4, 133, keys_x8=True),
    W.Prefill("pair_group3_noncausal", "bf16", False, "contiguous", 1, 6, 2, 1024, 128, 2, 134),
    W.Prefill("pair_striped_group4", "bf16", True, "striped", 1, 8, 2, 1536, 128, 3, 135),
    W.Prefill("pair_tail_S200", "bf16", True, "zigzag", 1, 4, 1, 200, 128, 1, 136),
]


@pytest.mark.parametrize("kernel", ["pair", "single"])
@pytest.mark.parametrize("cfg", BOTH, ids=lambda c: c.name)
def test_both_tensor_core_kernels_every_row(cfg, kernel, monkeypatch):
    monkeypatch.setenv("RING_ATTN_TC_KERNEL", kernel)
    run(cfg, rows=W.sample_rows(cfg, 0))


@pytest.mark.parametrize("kernel", ["pair", "single"])
@pytest.mark.parametrize("layout", ["zigzag", "striped"])
def test_both_tensor_core_kernels_through_the_step_api(layout, kernel, monkeypatch):
    monkeypatch.setenv("RING_ATTN_TC_KERNEL", kernel)
    need_cuda()
    cfg = W.Prefill("pair_steps", "bf16", True, layout, 1, 8, 2, 1536, 128, 3, 137)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = ring_by_steps(q, k, v, cfg.P, layout, True, cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    rows = W.sample_rows(cfg, 0)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, True)
    check_rows(out, lse, rows, ref_out, ref_lse, TOL_BF16_OUT, TOL_BF16_LSE, f"{kernel} {layout} steps")
