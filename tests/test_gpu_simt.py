"""GPU parity of the CUDA-core path (float32 and bf16 inputs) and of the
ring-step API against the fp64 oracle, on the same seeded inputs."""
import dataclasses
import random

import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import oracle
import workloads as W
from oracle import schedule as sch
from tests.helpers import (TOL_BF16_LSE, TOL_BF16_OUT, TOL_FP32, check_rows, host, need_cuda, oracle_rows)

pytestmark = pytest.mark.gpu


def run_fwd_and_check(cfg, fn, tol_out, tol_lse, rows=None):
    need_cuda()
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = fn(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    rows = W.sample_rows(cfg) if rows is None else rows
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, cfg.causal)
    return check_rows(out, lse, rows, ref_out, ref_lse, tol_out, tol_lse, cfg.name)


def test_cfg1_fp32_fused_ring():
    # fp32, non-causal, B1 H2 S256 D64 P4: every row, max abs err <= 1e-5
    run_fwd_and_check(W.CFG1, ra.ring_attn_fwd, TOL_FP32, TOL_FP32)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("P", [1, 2, 4])
def test_fp32_layouts(layout, causal, P):
    cfg = dataclasses.replace(W.CFG1, causal=causal, layout=layout, P=P, seed=11)
    run_fwd_and_check(cfg, ra.ring_attn_fwd, TOL_FP32, TOL_FP32)


def test_fp32_ragged_gqa_d128():
    # chunks of 50 rows (not a multiple of the 64-row tile), GQA group 3, D = 128
    cfg = W.Prefill("ragged", "fp32", True, "zigzag", 2, 6, 2, 300, 128, 3, 12)
    run_fwd_and_check(cfg, ra.ring_attn_fwd, TOL_FP32, TOL_FP32)


@pytest.mark.parametrize("cfg", [
    W.Prefill("bf16_contig_small", "bf16", True, "contiguous", 1, 4, 4, 1024, 128, 8, 21),
    W.Prefill("bf16_zigzag_small_keysx8", "bf16", True, "zigzag", 2, 2, 2, 2048, 128, 4, 22, keys_x8=True),
    W.Prefill("bf16_gqa_small", "bf16", True, "zigzag", 1, 8, 2, 1024, 128, 2, 23),
    W.Prefill("bf16_noncausal_d64", "bf16", False, "contiguous", 1, 2, 1, 640, 64, 5, 24),
], ids=lambda c: c.name)
def test_bf16_simt(cfg):
    run_fwd_and_check(cfg, ra.ring_attn_fwd_simt, TOL_BF16_OUT, TOL_BF16_LSE, rows=W.sample_rows(cfg, 0))


def ring_by_steps(q, k, v, P, layout, causal, scale, order_fn=None, checkpoint_at=None):
    """Drive ring_attn_step rank by rank; returns (out, lse) in natural order.
    Each rank's shard is gathered from its chunks (its stripe when striped)."""
    B, S, Hq, D = q.shape
    own = sch.layout_assignment(P, layout)
    pos = sch.chunk_positions(S, P, layout)
    C = sch.chunk_len(S, P, layout)
    stripes = P if layout.startswith("striped") else 0
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), device=q.device, dtype=torch.float32)
    for r in range(P):
        qc = own[r]
        rows = torch.tensor([t for c in qc for t in pos[c]], device=q.device)
        qs = q[:, rows].contiguous()
        m, l, O = ra.new_state(B, Hq, len(rows), D)
        srcs = sch.block_sources(P, r)
        if order_fn is not None:
            srcs = order_fn(srcs)
        for t, src in enumerate(srcs):
            kc = own[src]
            krows = torch.tensor([t_ for c in kc for t_ in pos[c]], device=q.device)
            ra.ring_attn_step(qs, k[:, krows].contiguous(), v[:, krows].contiguous(), m, l, O, qc, kc, C,
                              causal=causal, scale=scale, stripes=stripes)
            if checkpoint_at is not None and t == checkpoint_at:
                # checkpoint / resume: the state is the only thing carried between steps
                saved = [x.cpu().clone() for x in (m, l, O)]
                m, l, O = (x.cuda() for x in saved)
        o_r, lse_r = ra.ring_attn_state_finalize(m, l, O, dtype=q.dtype)
        out[:, rows] = o_r
        lse[:, :, rows] = lse_r
    return out, lse


@pytest.mark.parametrize("shuffle", [False, True])
def test_cfg1_fp32_ring_steps(shuffle):
    need_cuda()
    cfg = W.CFG1
    q, k, v = W.prefill_inputs(cfg, "cuda")
    rng = random.Random(5)
    order = (lambda s: rng.sample(s, len(s))) if shuffle else None
    out, lse = ring_by_steps(q, k, v, cfg.P, cfg.layout, cfg.causal, cfg.scale, order_fn=order)
    rows = W.sample_rows(cfg, 0)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, cfg.causal)
    check_rows(out, lse, rows, ref_out, ref_lse, TOL_FP32, TOL_FP32, "steps")


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_fp32_causal_steps_checkpoint(layout):
    need_cuda()
    cfg = dataclasses.replace(W.CFG1, causal=True, layout=layout, seed=31)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    out, lse = ring_by_steps(q, k, v, cfg.P, cfg.layout, True, cfg.scale, checkpoint_at=1)
    rows = W.sample_rows(cfg, 0)
    ref_out, ref_lse = oracle_rows(q, k, v, rows, cfg.scale, True)
    check_rows(out, lse, rows, ref_out, ref_lse, TOL_FP32, TOL_FP32, "steps+checkpoint")


def test_step_state_is_attention_over_seen_keys():
    # after each step: m = max score over keys seen so far, l = sum exp(s - m), O normalised
    need_cuda()
    cfg = dataclasses.replace(W.CFG1, causal=False, seed=41)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    C = cfg.chunk
    r = 1
    rows = np.arange(r * C, (r + 1) * C)
    qs = q[:, rows].contiguous()
    m, l, O = ra.new_state(cfg.B, cfg.Hq, C, cfg.D)
    seen = []
    for src in sch.block_sources(cfg.P, r):
        krows = np.arange(src * C, (src + 1) * C)
        ra.ring_attn_step(qs, k[:, krows].contiguous(), v[:, krows].contiguous(), m, l, O, [r], [src], C,
                          causal=False, scale=cfg.scale)
        seen.extend(krows)
        sk = np.array(sorted(seen))
        ks, vs = host(k)[:, sk], host(v)[:, sk]
        req = [(0, h, i) for h in range(cfg.Hq) for i in range(C)]
        ref_o, ref_lse = oracle.attention_rows(host(qs), ks, vs, req, scale=cfg.scale, causal=False)
        s_full = np.einsum("id,jd->ij", host(qs)[0, :, 0].astype(np.float64), ks[0, :, 0].astype(np.float64)) * cfg.scale
        np.testing.assert_allclose(host(m)[0, 0], s_full.max(1), atol=1e-5)
        got_lse = host(m) + np.log(host(l))
        np.testing.assert_allclose(got_lse.reshape(-1), ref_lse, atol=TOL_FP32)
        np.testing.assert_allclose(host(O).transpose(0, 2, 1, 3).reshape(-1, cfg.D), ref_o, atol=TOL_FP32)


def test_step_fully_masked_block_keeps_state():
    # a K/V chunk entirely after the query chunk (causal) must leave the state untouched
    need_cuda()
    cfg = dataclasses.replace(W.CFG1, causal=True, seed=51)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    C = cfg.chunk
    qs = q[:, :C].contiguous()
    m, l, O = ra.new_state(cfg.B, cfg.Hq, C, cfg.D)
    ra.ring_attn_step(qs, k[:, :C].contiguous(), v[:, :C].contiguous(), m, l, O, [0], [0], C, True, cfg.scale)
    before = [x.clone() for x in (m, l, O)]
    ra.ring_attn_step(qs, k[:, 2 * C:3 * C].contiguous(), v[:, 2 * C:3 * C].contiguous(), m, l, O, [0], [2], C,
                      True, cfg.scale)
    for a, b in zip(before, (m, l, O)):
        assert torch.equal(a, b)


def test_bounded_wait_reports_timeout():
    need_cuda()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    ra.ring_attn_selftest_wait(2000)
    st, where = ra.ring_attn_device_error()
    assert st == ra.RING_ETIMEOUT and where == 11
    assert ra.ring_attn_device_error()[0] == ra.RING_OK     # read-and-clear
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
