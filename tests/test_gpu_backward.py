"""Backward of the ring on the GPU against the fp64 oracle (oracle.attention_bwd):
the fused ring backward for every split, float32 and bf16, and the step API
driven hop by hop (dK, dV travelling with their block).  The forward's own
out and lse feed the backward, as in training."""
import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import oracle
import workloads as W
from oracle import schedule as sch
from tests.helpers import margin, host, need_cuda

pytestmark = pytest.mark.gpu

# max |gpu - oracle| <= TOL * max(1, max |oracle|) per gradient.  float32: sums of at most S
# float32 products and expf (a few ulp) -- measured 3.5e-6; bf16: the bf16 rounding of each
# gradient (2^-9 of its size) plus that of the forward output inside delta -- measured 4.0e-3
TOL_BWD_FP32 = 2e-5
TOL_BWD_BF16 = 1e-2


def _dout(cfg, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dt = torch.float32 if cfg.dtype == "fp32" else torch.bfloat16
    return torch.randn((cfg.B, cfg.S, cfg.Hq, cfg.D), generator=g, device="cuda").to(dt)


def _check(grads, refs, tol, what):
    for name, x, r in zip(("dq", "dk", "dv"), grads, refs):
        err = float(np.max(np.abs(host(x) - r)))
        bound = tol * max(1.0, float(np.max(np.abs(r))))
        assert np.all(np.isfinite(host(x))), f"{what} {name}"
        margin(name, err, bound, what)


CASES = [
    W.Prefill("fp32_noncausal_P1", "fp32", False, "contiguous", 1, 2, 2, 256, 64, 1, 601),
    W.Prefill("fp32_zigzag_gqa", "fp32", True, "zigzag", 1, 4, 2, 1024, 128, 4, 602),
    W.Prefill("fp32_striped_ragged", "fp32", True, "striped", 1, 2, 1, 768, 64, 3, 603),
    W.Prefill("bf16_zigzag_gqa", "bf16", True, "zigzag", 1, 8, 2, 2048, 128, 4, 604),
    W.Prefill("bf16_ragged_chunks", "bf16", True, "zigzag", 2, 3, 3, 1200, 128, 3, 605),
    W.Prefill("bf16_zigzag4_d64", "bf16", True, "zigzag4", 1, 4, 1, 2048, 64, 2, 606),
    W.Prefill("bf16_contiguous_noncausal", "bf16", False, "contiguous", 1, 2, 2, 1024, 128, 4, 607),
    W.Prefill("bf16_odd_group_zigzag3", "bf16", True, "zigzag3", 1, 6, 2, 1536, 128, 2, 611),
    W.Prefill("bf16_striped_ragged_gqa", "bf16", True, "striped", 1, 8, 2, 2700, 64, 3, 612),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_ring_backward_against_oracle(cfg):
    need_cuda()
    q, k, v = W.prefill_inputs(cfg, "cuda")
    dout = _dout(cfg, cfg.seed + 1)
    out, lse = ra.ring_attn_fwd(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    dq, dk, dv = ra.ring_attn_bwd(q, k, v, out, lse, dout, cfg.P, causal=cfg.causal, layout=cfg.layout,
                                  scale=cfg.scale)
    torch.cuda.synchronize()
    refs = oracle.attention_bwd(host(q), host(k), host(v), host(dout), scale=cfg.scale, causal=cfg.causal)
    _check((dq, dk, dv), refs, TOL_BWD_FP32 if cfg.dtype == "fp32" else TOL_BWD_BF16, cfg.name)


def test_backward_same_for_every_split():
    # exact gradients: the split only changes the order of the sums
    need_cuda()
    cfg = W.Prefill("splits", "fp32", True, "zigzag", 1, 2, 2, 768, 64, 2, 608)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    dout = _dout(cfg, 9)
    ref = None
    for layout in ("contiguous", "zigzag", "zigzag3", "striped", "contiguous2"):
        out, lse = ra.ring_attn_fwd(q, k, v, 2, True, layout, cfg.scale)
        g = ra.ring_attn_bwd(q, k, v, out, lse, dout, 2, True, layout, cfg.scale)
        torch.cuda.synchronize()
        if ref is None:
            ref = [x.clone() for x in g]
        else:
            for x, r in zip(g, ref):
                assert (x - r).abs().max().item() <= 1e-5, layout


def test_backward_delta():
    need_cuda()
    g = torch.Generator(device="cuda").manual_seed(5)
    out = torch.randn((2, 100, 3, 128), generator=g, device="cuda").to(torch.bfloat16)
    dout = torch.randn((2, 100, 3, 128), generator=g, device="cuda").to(torch.bfloat16)
    delta = ra.ring_attn_bwd_delta(out, dout)
    ref = np.einsum("bihd,bihd->bhi", host(out).astype(np.float64), host(dout).astype(np.float64))
    assert np.max(np.abs(host(delta) - ref)) <= 1e-4


@pytest.mark.parametrize("dtype,layout,S,P", [("fp32", "zigzag", 1024, 4), ("bf16", "striped", 1536, 3),
                                              ("fp32", "contiguous", 512, 4)])
def test_step_backward_ring(dtype, layout, S, P):
    # every rank meets every block; dK, dV of a block are summed wherever it is met
    need_cuda()
    cfg = W.Prefill("stepbwd", dtype, True, layout, 1, 4, 2, S, 64, P, 609)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    dout = _dout(cfg, 10)
    out, lse = ra.ring_attn_fwd(q, k, v, P, True, layout, cfg.scale)
    delta = ra.ring_attn_bwd_delta(out, dout)
    own = sch.layout_assignment(P, layout)
    pos = sch.chunk_positions(S, P, layout)
    C = sch.chunk_len(S, P, layout)
    stripes = P if layout == "striped" else 0
    rows = {r: torch.tensor([t for c in own[r] for t in pos[c]], device="cuda") for r in range(P)}
    B, Hq, Hkv, D = 1, 4, 2, 64
    dq = torch.zeros((B, S, Hq, D), device="cuda")
    dk_acc = {s: torch.zeros((B, len(rows[s]), Hkv, D), device="cuda") for s in range(P)}
    dv_acc = {s: torch.zeros((B, len(rows[s]), Hkv, D), device="cuda") for s in range(P)}
    for r in range(P):
        rr = rows[r]
        qs, ds = q[:, rr].contiguous(), dout[:, rr].contiguous()
        ls, dl = lse[:, :, rr].contiguous(), delta[:, :, rr].contiguous()
        dq_r = torch.zeros((B, len(rr), Hq, D), device="cuda")
        for src in sch.block_sources(P, r):
            kr = rows[src]
            ra.ring_attn_step_bwd(qs, k[:, kr].contiguous(), v[:, kr].contiguous(), ds, ls, dl, dq_r, dk_acc[src],
                                  dv_acc[src], own[r], own[src], C, causal=True, scale=cfg.scale, stripes=stripes)
        dq[:, rr] = dq_r
    dk = torch.zeros((B, S, Hkv, D), device="cuda")
    dv = torch.zeros((B, S, Hkv, D), device="cuda")
    for s in range(P):
        dk[:, rows[s]] = dk_acc[s]
        dv[:, rows[s]] = dv_acc[s]
    torch.cuda.synchronize()
    refs = oracle.attention_bwd(host(q), host(k), host(v), host(dout), scale=cfg.scale, causal=True)
    # float32 accumulators on both sides of the bf16 rounding: the bf16 case keeps the bf16 input error only
    _check((dq, dk, dv), refs, TOL_BWD_FP32 if dtype == "fp32" else 5e-3, f"steps {dtype} {layout}")


@pytest.mark.parametrize("layout,S,P,Hq,Hkv,D", [("zigzag", 4096, 4, 8, 2, 128), ("striped", 3072, 3, 4, 4, 128),
                                                 ("contiguous", 2048, 2, 4, 1, 64), ("zigzag4", 4096, 2, 6, 2, 128)])
def test_tensor_core_backward_matches_cuda_cores(layout, S, P, Hq, Hkv, D):
    # two independent implementations on the same bf16 inputs and forward results
    need_cuda()
    cfg = W.Prefill("tcsimt", "bf16", True, layout, 1, Hq, Hkv, S, D, P, 610)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    dout = _dout(cfg, 11)
    out, lse = ra.ring_attn_fwd(q, k, v, P, True, layout, cfg.scale)
    g1 = ra.ring_attn_bwd(q, k, v, out, lse, dout, P, True, layout, cfg.scale)
    g2 = ra.ring_attn_bwd_simt(q, k, v, out, lse, dout, P, True, layout, cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    for name, a, b in zip(("dq", "dk", "dv"), g1, g2):
        scale_ = max(1.0, b.float().abs().max().item())
        margin(str(name), (a.float() - b.float()).abs().max().item(), TOL_BWD_BF16 * scale_)


def test_full_size_backward_sampled_rows_and_invariants():
    # causal zig-zag GQA, B1 Hq32 Hkv8 S131072 D128 P16 (the timed forward workload): dq on
    # sampled rows of four heads against the row-at-a-time fp64 oracle; dk and dv through
    # properties that hold at any size: shifting every key by one vector leaves the output
    # unchanged (sum_j dk_j = 0 per kv head) and the weights of a row sum to one
    # (sum_j dv_j = sum over the group's rows of dout)
    need_cuda()
    cfg = W.CFG4
    q, k, v = W.prefill_inputs(cfg, "cuda")
    dout = _dout(cfg, 12)
    out, lse = ra.ring_attn_fwd(q, k, v, cfg.P, True, cfg.layout, cfg.scale)
    dq, dk, dv = ra.ring_attn_bwd(q, k, v, out, lse, dout, cfg.P, True, cfg.layout, cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    rows = np.array([r for r in W.sample_rows(cfg, 24) if r[1] in (0, 9, 22, 31)], dtype=np.int32)
    ref = oracle.attention_bwd_dq_rows(host(q), host(k), host(v), host(dout), rows, scale=cfg.scale, causal=True)
    got = host(dq)[rows[:, 0], rows[:, 2], rows[:, 1]]
    margin("dq", np.max(np.abs(got - ref)), TOL_BWD_BF16 * max(1.0, float(np.max(np.abs(ref)))))
    G = cfg.Hq // cfg.Hkv
    dk64 = dk.double().sum(dim=1).cpu().numpy()                                  # [B, Hkv, D]
    dv64 = dv.double().sum(dim=1).cpu().numpy()
    do64 = dout.double().sum(dim=1).reshape(cfg.B, cfg.Hkv, G, cfg.D).sum(2).cpu().numpy()
    # Two roundings break the identities by random walks: each summed bf16 element (2^-9 of its
    # size, over S rows), and the bf16 P and dS inside the products -- a query row's bf16 weights
    # sum to 1 only within about 2^-9, which walks over the S*G rows of dout (or q) of the group
    walk = lambda x: 8.0 * np.sqrt(cfg.S) * 2.0 ** -9 * float(x.float().pow(2).mean().sqrt().item())
    rows_walk = lambda y: 4.0 * np.sqrt(cfg.S * G) * 2.0 ** -9 * float(y.float().pow(2).mean().sqrt().item())
    assert np.max(np.abs(dk64)) <= walk(dk) + cfg.scale * rows_walk(q) * 8.0
    assert np.max(np.abs(dv64 - do64)) <= walk(dv) + rows_walk(dout)


@pytest.mark.parametrize("cfg", [
    W.Prefill("autograd_bf16_zigzag_gqa", "bf16", True, "zigzag", 1, 8, 2, 2048, 128, 4, 621),
    W.Prefill("autograd_bf16_striped_gqa", "bf16", True, "striped", 2, 4, 2, 1536, 128, 3, 622),
    W.Prefill("autograd_fp32_zigzag_gqa", "fp32", True, "zigzag", 1, 4, 2, 1024, 64, 4, 623),
    W.Prefill("autograd_fp32_striped", "fp32", True, "striped", 1, 2, 2, 768, 64, 3, 624),
], ids=lambda c: c.name)
def test_ring_attention_under_autograd_against_oracle(cfg):
    # the training entry point: out = ring_attention(q, k, v, P) on leaf tensors, loss = sum(out * dout),
    # loss.backward(); the leaves' gradients against the fp64 oracle
    need_cuda()
    q, k, v = W.prefill_inputs(cfg, "cuda")
    dout = _dout(cfg, cfg.seed + 1)
    lq, lk, lv = (x.clone().requires_grad_(True) for x in (q, k, v))
    out = ra.ring_attention(lq, lk, lv, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
    (out.float() * dout.float()).sum().backward()
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    assert lq.grad.dtype == q.dtype and lk.grad.shape == k.shape and lv.grad.shape == v.shape
    rows = oracle.all_rows(cfg.B, cfg.Hq, cfg.S)
    ro, _ = oracle.attention_rows(host(q), host(k), host(v), rows, scale=cfg.scale, causal=cfg.causal)
    ro = ro.reshape(cfg.B, cfg.Hq, cfg.S, cfg.D).transpose(0, 2, 1, 3)
    margin("out", np.max(np.abs(host(out) - ro)), 1e-5 if cfg.dtype == "fp32" else 2e-2)
    refs = oracle.attention_bwd(host(q), host(k), host(v), host(dout), scale=cfg.scale, causal=cfg.causal)
    _check((lq.grad, lk.grad, lv.grad), refs, TOL_BWD_FP32 if cfg.dtype == "fp32" else TOL_BWD_BF16, cfg.name)
