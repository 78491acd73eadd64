"""Split variants on the GPU against the fp64 oracle: zig-zag with k chunks
per rank (the code exercise of "Lesson 8: Context Parallelism"), the
sequential k-per-rank split of its worked example, and the striped split
(token t on rank t mod P), through the fused tensor-core path, the CUDA-core
path and the step API; the device's work counters against the schedule
enumeration of the oracle."""
import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import workloads as W
from oracle import schedule as sch
from tests.helpers import (margin, TOL_BF16_LSE, TOL_BF16_OUT, TOL_FP32, check_rows, need_cuda, oracle_rows)
from tests.test_gpu_simt import ring_by_steps

pytestmark = pytest.mark.gpu

TC_CASES = [
    W.Prefill("zigzag4_gqa", "bf16", True, "zigzag4", 1, 8, 2, 8192, 128, 4, 201, sample_rows=96),
    W.Prefill("zigzag3_ragged_chunks", "bf16", True, "zigzag3", 1, 4, 4, 3000, 128, 2, 202),
    W.Prefill("zigzag8_P2", "bf16", True, "zigzag8", 1, 2, 1, 4096, 128, 2, 203),
    W.Prefill("contiguous2", "bf16", True, "contiguous2", 1, 4, 1, 4096, 128, 4, 204),
    W.Prefill("striped_gqa", "bf16", True, "striped", 1, 8, 2, 8192, 128, 8, 205, sample_rows=96),
    W.Prefill("striped_ragged_d64", "bf16", True, "striped", 2, 4, 4, 6000, 64, 4, 206, sample_rows=96),
    W.Prefill("striped_noncausal", "bf16", False, "striped", 1, 4, 2, 4096, 128, 4, 207, sample_rows=96),
    W.Prefill("striped_odd_group", "bf16", True, "striped", 1, 3, 1, 2048, 128, 8, 208),
    W.Prefill("striped_keysx8", "bf16", True, "striped", 1, 4, 4, 4096, 128, 16, 209, keys_x8=True, sample_rows=96),
    W.Prefill("striped_P1", "bf16", True, "striped", 1, 2, 2, 1024, 128, 1, 210),
]


def _check_fwd(cfg, fn, tol_o, tol_l):
    need_cuda()
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = fn(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    rows = W.sample_rows(cfg)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, cfg.causal)
    return check_rows(out, lse, rows, ref_out, ref_lse, tol_o, tol_l, cfg.name)


@pytest.mark.parametrize("cfg", TC_CASES, ids=lambda c: c.name)
def test_tc_split_variants(cfg):
    _check_fwd(cfg, ra.ring_attn_fwd, TOL_BF16_OUT, TOL_BF16_LSE)


@pytest.mark.parametrize("cfg", [
    W.Prefill("fp32_striped", "fp32", True, "striped", 1, 2, 2, 1024, 64, 4, 211),
    W.Prefill("fp32_striped_ragged", "fp32", True, "striped", 1, 2, 1, 900, 128, 3, 212),
    W.Prefill("fp32_zigzag3", "fp32", True, "zigzag3", 1, 2, 2, 960, 64, 4, 213),
    W.Prefill("fp32_contiguous3", "fp32", True, "contiguous3", 1, 2, 2, 768, 64, 2, 214),
], ids=lambda c: c.name)
def test_simt_fp32_split_variants(cfg):
    _check_fwd(cfg, ra.ring_attn_fwd, TOL_FP32, TOL_FP32)


@pytest.mark.parametrize("layout", ["striped", "zigzag4", "zigzag3"])
def test_tc_matches_simt(layout):
    # two independent kernels on the same bf16 inputs
    need_cuda()
    cfg = W.Prefill("x", "bf16", True, layout, 1, 4, 2, 6144, 128, 4, 215)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    o1, l1 = ra.ring_attn_fwd(q, k, v, cfg.P, True, layout, cfg.scale)
    o2, l2 = ra.ring_attn_fwd_simt(q, k, v, cfg.P, True, layout, cfg.scale)
    torch.cuda.synchronize()
    margin("out", (o1.float() - o2.float()).abs().max().item(), TOL_BF16_OUT)
    margin("lse", (l1 - l2).abs().max().item(), TOL_BF16_LSE)


@pytest.mark.parametrize("dtype,layout,S,P,tol_o,tol_l", [
    ("bf16", "striped", 2048, 4, TOL_BF16_OUT, TOL_BF16_LSE),
    ("bf16", "zigzag4", 2048, 2, TOL_BF16_OUT, TOL_BF16_LSE),
    ("bf16", "striped", 1800, 3, TOL_BF16_OUT, TOL_BF16_LSE),
    ("fp32", "striped", 1024, 4, TOL_FP32, TOL_FP32),
    ("fp32", "zigzag3", 768, 2, TOL_FP32, TOL_FP32),
])
def test_steps_split_variants(dtype, layout, S, P, tol_o, tol_l):
    need_cuda()
    cfg = W.Prefill("steps", dtype, True, layout, 1, 4, 2, S, 128, P, 216)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = ring_by_steps(q, k, v, P, layout, True, cfg.scale)
    rows = W.sample_rows(cfg, 0)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, True)
    check_rows(out, lse, rows, ref_out, ref_lse, tol_o, tol_l, f"{dtype} {layout} steps")


@pytest.mark.parametrize("cfg", [
    W.Prefill("cnt_striped", "bf16", True, "striped", 1, 4, 4, 16384, 128, 8, 217),
    W.Prefill("cnt_striped_ragged", "bf16", True, "striped", 1, 2, 2, 6000, 128, 4, 218),
    W.Prefill("cnt_zigzag4", "bf16", True, "zigzag4", 1, 4, 2, 16384, 128, 4, 219),
    W.Prefill("cnt_zigzag3", "bf16", True, "zigzag3", 1, 2, 2, 3000, 128, 2, 220),
], ids=lambda c: c.name)
def test_device_counters_split_variants(cfg):
    need_cuda()
    q, k, v = W.prefill_inputs(cfg, "cuda")
    _, _, cnt = ra.ring_attn_fwd_counted(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    torch.cuda.synchronize()
    cnt = cnt.cpu().numpy().astype(np.int64)
    full, partial, _, _ = sch.tile_classes(cfg.S, cfg.P, cfg.layout, cfg.causal, 128, 128)
    heads = cfg.B * cfg.Hq
    assert int(cnt[0]) == full * heads and int(cnt[1]) == partial * heads
    pairs = sch.per_rank_pairs(cfg.P, cfg.layout, cfg.causal, cfg.S)
    assert [int(x) for x in cnt[2:]] == [p_ * heads for p_ in pairs]


def test_split_does_not_change_the_result():
    # exact attention: every split gives the same output up to rounding order
    need_cuda()
    cfg = W.Prefill("same", "bf16", True, "zigzag", 1, 4, 4, 6144, 128, 4, 221)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    ref_o, ref_l = ra.ring_attn_fwd(q, k, v, 4, True, "contiguous", cfg.scale)
    for layout in ("zigzag", "zigzag4", "zigzag3", "contiguous2", "striped"):
        o, l = ra.ring_attn_fwd(q, k, v, 4, True, layout, cfg.scale)
        torch.cuda.synchronize()
        margin("out", (o.float() - ref_o.float()).abs().max().item(), TOL_BF16_OUT, str(layout))
        margin("lse", (l - ref_l).abs().max().item(), TOL_BF16_LSE, str(layout))
