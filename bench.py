#!/usr/bin/env python
"""Benchmark of the ring-attention hot path on B200.

One "step" is one pass of the whole hot path on one batch of synthetic input:
  * prefill: the fused ring (all P virtual ranks) of the causal zig-zag GQA
    workload B1 Hq32 Hkv8 S131072 D128 P16 -- the headline metric,
    causal-adjusted TFLOP/s (4*B*Hq*S^2*D/2 per step);
  * decode: the split-KV single-token decode B8 Hq32 Hkv8 D128, 2^20-token
    capacity in 32 chunks, valid lengths U[0.5M, 1M] (partials + merge),
    reported in the same line as GB/s of algorithmic bytes.
Inputs are resident in HBM before the timed region (both workloads' inputs
exceed the 126 MB L2).  Times are CUDA events on the launching stream;
multi-GPU runs are independent replicas (no collective on the data path),
timed as the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload, on the host cores, with the same metric and config.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's published B200 figures: dense bf16 tensor throughput (half the 2:4-sparsity
# figure of the datasheet) and HBM3e bandwidth of the HGX part.  Reported beside the
# measured peaks so a reader can judge a fraction against either.
PUBLISHED = {"bf16_tflops": 2250.0, "hbm_gbs": 7700.0,
             "source": "NVIDIA B200 datasheet: 2.25 PFLOP/s dense bf16, 7.7 TB/s HBM3e (HGX)"}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- distributed plumbing
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        return dist, int(os.environ["RANK"]), world
    return None, 0, 1


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, x: float, device="cuda") -> float:
    """The largest x over all ranks (timings are taken as the max over ranks)."""
    if dist is None:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(work_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job rate of `world` independent replicas, each doing `steps` steps
    of `work_per_step`, timed as the max over ranks."""
    return work_per_step * steps * world / (max_ms / 1e3)


# --------------------------------------------------------------------------- the hot path
def decode_bytes(cfg, lens: np.ndarray) -> float:
    """Algorithmic bytes of one split-KV decode: every valid K and V row once,
    q, the partial results written and read back, the output and lse."""
    kv = float(lens.sum()) * cfg.Hkv * cfg.D * 2 * 2
    q = cfg.B * cfg.Hq * cfg.D * 2
    parts = cfg.B * cfg.Hq * cfg.P * (cfg.D + 1) * 4 * 2
    out = cfg.B * cfg.Hq * (cfg.D * 2 + 4)
    return kv + q + parts + out


def step_ring(ra, cfg, q, k, v, dev):
    """The whole ring of `cfg` through the step API: for each rank r, a fresh
    state, then P calls of ring_attn_step (hop t folds the block that started
    on rank (r - t) mod P), then the finalisation of the state.  The state
    (m, l, O fp32) is read and written in HBM by every call.  Returns the
    closure, the number of library launches per ring, and rank P-1's output
    with its token positions (for a check against the fused ring)."""
    from context_exact_attention_ring_b200 import ring
    P = cfg.P
    own = ring.split_chunks(P, cfg.layout)
    C = cfg.S // (P * len(own[0]))
    rows = [ring.shard_rows(cfg.S, P, cfg.layout, r).to(dev) for r in range(P)]
    qs = [q[:, rr].contiguous() for rr in rows]
    ks = [k[:, rr].contiguous() for rr in rows]
    vs = [v[:, rr].contiguous() for rr in rows]
    S_loc = int(rows[0].numel())
    m, l, O = ra.new_state(cfg.B, cfg.Hq, S_loc, cfg.D, dev)
    o_r = torch.empty((cfg.B, S_loc, cfg.Hq, cfg.D), device=dev, dtype=q.dtype)
    lse_r = torch.empty((cfg.B, cfg.Hq, S_loc), device=dev, dtype=torch.float32)

    def run():
        for r in range(P):
            ra.ring_attn_state_init(m, l, O)
            for t in range(P):
                src = (r - t) % P
                ra.ring_attn_step(qs[r], ks[src], vs[src], m, l, O, own[r], own[src], C, causal=cfg.causal,
                                  scale=cfg.scale)
            ra.ring_attn_state_finalize(m, l, O, dtype=q.dtype, out=o_r, lse=lse_r)

    return run, P * (P + 2), o_r, rows[P - 1]


def merge_bytes(mc) -> float:
    """Algorithmic bytes of one merge: the partials and their lse read once,
    the bf16 output and its lse written."""
    return float(mc.B * mc.Hq * (mc.P * (mc.D + 1) * 4 + mc.D * 2 + 4))


def time_merge_only(ra, dev, reps=24, sets=4):
    """ring_attn_merge alone on an HBM-bound shape (W.MERGE_ONLY), launched
    back to back on `sets` input sets (4 x 137 MB, four times the L2) taken in
    turn, so no launch finds its partials in L2.  CUDA events on the launching
    stream around all `reps` launches.  Returns (mean ms per launch, GB/s)."""
    mc = W.MERGE_ONLY
    ins = [W.merge_inputs(dataclasses.replace(mc, seed=mc.seed + i), dev) for i in range(sets)]
    out = torch.empty((mc.B, mc.Hq, mc.D), device=dev, dtype=torch.bfloat16)
    olse = torch.empty((mc.B, mc.Hq), device=dev, dtype=torch.float32)
    st = torch.cuda.current_stream()
    for i in range(2 * sets):
        ra.ring_attn_merge(*ins[i % sets], out=out, out_lse=olse)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for i in range(reps):
        ra.ring_attn_merge(*ins[i % sets], out=out, out_lse=olse)
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del ins
    return ms, merge_bytes(mc) / (ms / 1e3) / 1e9


def run_ours(args):
    import context_exact_attention_ring_b200 as ra

    dist, rank, world = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    st = torch.cuda.current_stream()
    pk, pk_kind = peaks()
    cfg, dcfg = W.CFG4, W.CFG5

    q, k, v = W.prefill_inputs(cfg, dev)
    out = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.S), device=dev, dtype=torch.float32)
    dq, dk, dv, dl = W.decode_inputs(dcfg, dev)
    lens = dl.cpu().numpy().astype(np.int64)
    part = torch.empty((dcfg.B, dcfg.Hq, dcfg.P, dcfg.D), device=dev, dtype=torch.float32)
    plse = torch.empty((dcfg.B, dcfg.Hq, dcfg.P), device=dev, dtype=torch.float32)
    dout = torch.empty((dcfg.B, dcfg.Hq, dcfg.D), device=dev, dtype=torch.bfloat16)
    dlse = torch.empty((dcfg.B, dcfg.Hq), device=dev, dtype=torch.float32)
    ws = ra.decode_workspace(dcfg.B, dcfg.Hq, dcfg.Hkv, dcfg.capacity, dcfg.D, dcfg.P, dev)
    torch.cuda.synchronize()

    def prefill():
        ra.ring_attn_fwd(q, k, v, cfg.P, causal=True, layout=cfg.layout, scale=cfg.scale, out=out, lse=lse)

    def decode():
        ra.ring_attn_decode(dq, dk, dv, dl, dcfg.P, dcfg.scale, partials=part, part_lse=plse, out=dout,
                            out_lse=dlse, workspace=ws)

    for _ in range(args.warmup):
        prefill()
        decode()
    torch.cuda.synchronize()
    st_err = ra.ring_attn_device_error()[0]
    if st_err != ra.RING_OK:
        raise RuntimeError(f"device error during warm-up: {st_err}")

    clocks = ClockSampler(torch.cuda.current_device())
    barrier(dist)
    torch.cuda.synchronize()
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(st)
    for e0, e1, e2 in ev:
        e0.record(st)
        prefill()
        e1.record(st)
        decode()
        e2.record(st)
    t_all1.record(st)
    torch.cuda.synchronize()
    barrier(dist)
    clk = clocks.stop()
    if ra.ring_attn_device_error()[0] != ra.RING_OK:
        raise RuntimeError("device error during the timed region")

    pre_ms = [a.elapsed_time(b) for a, b, _ in ev]
    dec_ms = [b.elapsed_time(c) for _, b, c in ev]
    total_ms = t_all0.elapsed_time(t_all1)
    total_ms = max_over_ranks(dist, total_ms)
    pre_sum = max_over_ranks(dist, sum(pre_ms))
    dec_sum = max_over_ranks(dist, sum(dec_ms))

    flops = cfg.flops()
    value = replica_throughput(flops, args.steps, world, pre_sum) / 1e12     # causal-adjusted TFLOP/s, all ranks
    dbytes = decode_bytes(dcfg, lens)
    dvalue = replica_throughput(dbytes, args.steps, world, dec_sum) / 1e9    # GB/s, all ranks

    # ---------------------------------------------------------------- end to end (host buffers)
    # Every step copies its inputs from pinned host memory, runs ring_attn_fwd and copies out and
    # lse back to pinned host memory.  Steps are pipelined the way a serving loop uses the
    # asynchronous API: two device slots and three streams, so the host-to-device copy of step
    # i+1 and the device-to-host copy of step i-1 run while step i computes.
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hv = v.cpu().pin_memory()
        hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        hlse = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
        slots = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), o=torch.empty_like(out),
                      l=torch.empty_like(lse)) for _ in range(2)]
        s_in, s_c, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        inputs_free = [torch.cuda.Event() for _ in range(2)]    # compute of the slot's last step is done
        inputs_ready = [torch.cuda.Event() for _ in range(2)]
        outputs_free = [torch.cuda.Event() for _ in range(2)]   # the slot's last outputs are on the host
        computed = [torch.cuda.Event() for _ in range(2)]
        e2e_steps = max(2, args.steps)

        def e2e_step(i):
            sl, s_ = slots[i % 2], i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(inputs_free[s_])
                sl["q"].copy_(hq, non_blocking=True)
                sl["k"].copy_(hk, non_blocking=True)
                sl["v"].copy_(hv, non_blocking=True)
                inputs_ready[s_].record(s_in)
            with torch.cuda.stream(s_c):
                s_c.wait_event(inputs_ready[s_])
                if i >= 2:
                    s_c.wait_event(outputs_free[s_])
                ra.ring_attn_fwd(sl["q"], sl["k"], sl["v"], cfg.P, causal=True, layout=cfg.layout, scale=cfg.scale,
                                 out=sl["o"], lse=sl["l"])
                computed[s_].record(s_c)
                inputs_free[s_].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[s_])
                hout[s_].copy_(sl["o"], non_blocking=True)
                hlse[s_].copy_(sl["l"], non_blocking=True)
                outputs_free[s_].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(dist)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(s_in)
        for i in range(e2e_steps):
            e2e_step(i)
        s_in.wait_stream(s_out)
        a1.record(s_in)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(dist, a0.elapsed_time(a1))
        # the result really came back: the last step's output on the host equals the device result
        assert torch.equal(hout[(e2e_steps - 1) % 2][0, :4].to(dev), out[0, :4])
        h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
        d2h = hout[0].numel() * 2 + hlse[0].numel() * 4
        e2e = {"value": round(flops * e2e_steps * world / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms / e2e_steps, 3), "steps": e2e_steps,
               "path": "pinned host -> ring_attn_fwd -> pinned host; 2 device slots, copy-in / compute / copy-out "
                       "streams overlapping consecutive steps"}

    # ---------------------------------------------------------------- backward of the same ring
    # Timed after the main region on the same inputs (the forward's out and lse), outside the
    # step; the usual convention counts 2.5x the forward's FLOPs for dQ, dK, dV.
    bwd = None
    if not args.no_bwd:
        g = torch.Generator(device=dev).manual_seed(cfg.seed + 7)
        gout = torch.randn(q.shape, generator=g, device=dev).to(q.dtype)
        gq, gk, gv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(int(ra.lib().ring_attn_bwd_workspace_bytes(cfg.B, cfg.Hq, cfg.S)), device=dev,
                         dtype=torch.uint8)
        bfn = lambda: ra.ring_attn_bwd(q, k, v, out, lse, gout, cfg.P, causal=True, layout=cfg.layout,
                                       scale=cfg.scale, dq=gq, dk=gk, dv=gv, workspace=ws)
        bfn()
        torch.cuda.synchronize()
        barrier(dist)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(st)
        for _ in range(2):
            bfn()
        b1.record(st)
        torch.cuda.synchronize()
        bwd_ms = max_over_ranks(dist, b0.elapsed_time(b1)) / 2
        bwd_tf = 2.5 * flops * world / (bwd_ms / 1e3) / 1e12
        bwd = {"metric": "causal-adjusted backward TFLOP/s (2.5x the forward FLOPs)", "value": round(bwd_tf, 1),
               "unit": "TFLOP/s", "ms_per_call": round(bwd_ms, 3), "launches_per_call": 3,
               "kernels": "bwd_delta_kernel + attn_bwd_tc_kernel<128,true> (dK, dV) + <128,false> (dQ)"}
        del gout, gq, gk, gv, ws

    # ---------------------------------------------------------------- the same ring through the step API
    # P ranks x P hops of ring_attn_step with the state in HBM (what a multi-GPU ring runs per rank),
    # timed after the main region; its output is checked against the fused ring's.
    step_api = None
    if not args.no_step:
        srun, slaunch, so, srows = step_ring(ra, cfg, q, k, v, dev)
        srun()
        torch.cuda.synchronize()
        diff = float((so.float() - out[:, srows].float()).abs().max())
        if not diff <= 2e-2:
            raise RuntimeError(f"step API result differs from the fused ring by {diff}")
        barrier(dist)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(st)
        for _ in range(2):
            srun()
        c1.record(st)
        torch.cuda.synchronize()
        if ra.ring_attn_device_error()[0] != ra.RING_OK:
            raise RuntimeError("device error in the step API timing")
        step_ms = max_over_ranks(dist, c0.elapsed_time(c1)) / 2
        step_tf = flops * world / (step_ms / 1e3) / 1e12
        peak_s = pk.get("bf16_tflops_sustained") or pk["bf16_tflops"]
        step_api = {"metric": "causal-adjusted TFLOP/s of the same ring through ring_attn_step "
                              "(P ranks x P hops, state read and written in HBM by every call)",
                    "value": round(step_tf, 1), "unit": "TFLOP/s", "ms_per_ring": round(step_ms, 3),
                    "calls_per_ring": cfg.P * cfg.P, "launches_per_ring": slaunch,
                    "frac": round(step_tf / world / peak_s, 4), "max_abs_diff_vs_fused_out": round(diff, 5)}
        del srun, so

    # ---------------------------------------------------------------- the merge alone, HBM-bound
    merge_only = None
    if not args.no_merge:
        barrier(dist)
        m_ms, m_gbs = time_merge_only(ra, dev)
        m_ms = max_over_ranks(dist, m_ms)
        m_gbs = merge_bytes(W.MERGE_ONLY) / (m_ms / 1e3) / 1e9
        merge_only = {"metric": "ring_attn_merge GB/s of algorithmic bytes; back-to-back launches over 4 input "
                                "sets of 137 MB taken in turn (no launch finds its input in L2)",
                      "workload": W.MERGE_ONLY.name, "value": round(m_gbs * world, 1), "unit": "GB/s",
                      "ms_per_launch": round(m_ms, 4), "bytes_per_launch": merge_bytes(W.MERGE_ONLY),
                      "roofline": {"bound": "hbm", "achieved": round(m_gbs, 1), "peak": pk["hbm_gbs"],
                                   "unit": "GB/s", "frac": round(m_gbs / pk["hbm_gbs"], 4),
                                   "traffic": load_traffic().get("merge"),
                                   "kernel": "merge_kernel<bf16>", "peak_kind": f"{pk_kind} HBM copy",
                                   "frac_of_published": round(m_gbs / PUBLISHED["hbm_gbs"], 4)}}

    # ---------------------------------------------------------------- roofline of the dominant kernel
    pre_avg = statistics.mean(pre_ms)
    achieved_tf = flops / (pre_avg / 1e3) / 1e12
    peak_tf = pk.get("bf16_tflops_sustained") or pk["bf16_tflops"]
    dec_avg = statistics.mean(dec_ms)
    achieved_gb = dbytes / (dec_avg / 1e3) / 1e9
    traffic = load_traffic()

    line = {
        "metric": "causal-adjusted attention TFLOP/s at S=128k (1 GPU); split-KV decode GB/s",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), bf16; no dataset)",
        "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "S": cfg.S, "D": cfg.D,
                   "P": cfg.P, "layout": cfg.layout, "causal": True,
                   "flops_per_step": flops, "l2": "inputs larger than L2 (q 1.07 GB, k+v 0.54 GB)",
                   "decode_workload": dcfg.name, "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "tensor", "achieved": round(achieved_tf, 1), "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": round(achieved_tf / peak_tf, 4), "traffic": traffic.get("attn_tc_pair"),
                     "kernel": "attn_tc_pair_kernel (tcgen05 cta_group::2)",
                     "peak_kind": f"{pk_kind} bf16 dense, sustained",
                     "frac_of_burst": round(achieved_tf / pk["bf16_tflops"], 4),
                     "frac_of_published": round(achieved_tf / PUBLISHED["bf16_tflops"], 4),
                     "published_peak": PUBLISHED["bf16_tflops"], "published_source": PUBLISHED["source"]},
        "decode": {"metric": "split-KV decode GB/s", "value": round(dvalue, 1), "unit": "GB/s",
                   "ms_per_step": round(dec_avg, 3), "bytes_per_step": dbytes,
                   "roofline": {"bound": "hbm", "achieved": round(achieved_gb, 1), "peak": pk["hbm_gbs"],
                                "unit": "GB/s", "frac": round(achieved_gb / pk["hbm_gbs"], 4),
                                "traffic": traffic.get("decode"), "kernel": "decode_kernel<4, 128> + merge_kernel",
                                "peak_kind": f"{pk_kind} HBM copy",
                                "frac_of_published": round(achieved_gb / PUBLISHED["hbm_gbs"], 4),
                                "published_peak": PUBLISHED["hbm_gbs"]},
                   "merge_only": merge_only},
        "prefill_ms_per_step": round(pre_avg, 3),
        "e2e": e2e,
        "backward": bwd,
        "step_api": step_api,
        "gpu_launches": args.steps * 3,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(cfg, q, k, v, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def load_traffic():
    """DRAM bytes per launch of each kernel from the committed ncu summary
    (profiles/traffic.json).  An entry whose kernel sources changed since the
    counters were taken is reported as None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        d = json.load(f)
    out = {}
    for k, e in d.items():
        if not isinstance(e, dict):
            continue
        m = hashlib.sha256()
        try:
            for src in e["sources"]:
                with open(os.path.join(ROOT, src), "rb") as g:
                    m.update(g.read())
        except OSError:
            continue
        out[k] = e["bytes"] if m.hexdigest()[:16] == e["source_sha256"] else None
    return out


# --------------------------------------------------------------------------- oracle on the host cores
def cpu_baseline(cfg, q=None, k=None, v=None, seconds=15.0):
    """fp64 oracle on a bounded sample of the workload's query rows, on every
    host core; value in causal-adjusted TFLOP/s of the rows processed."""
    import oracle
    if q is None:
        q, k, v = W.prefill_inputs(cfg, "cpu")
    hq = q.float().cpu().numpy()
    hk = k.float().cpu().numpy()
    hv = v.float().cpu().numpy()
    rng = np.random.default_rng(cfg.seed + 7)
    cores = oracle.cores()
    # calibrate on a small batch, then size the sample to about `seconds`
    def rows_of(n):
        b = rng.integers(0, cfg.B, n)
        h = rng.integers(0, cfg.Hq, n)
        i = rng.integers(0, cfg.S, n)
        return np.stack([b, h, i], 1).astype(np.int32)
    def flops_of(rows):
        return float(np.sum(4.0 * cfg.D * (rows[:, 2].astype(np.float64) + 1)))
    cal = rows_of(4 * cores)
    t0 = time.perf_counter()
    oracle.attention_rows(hq, hk, hv, cal, scale=cfg.scale, causal=True)
    dt = time.perf_counter() - t0
    rate = flops_of(cal) / max(dt, 1e-6)
    n = int(max(4 * cores, min(200000, seconds * rate / (4.0 * cfg.D * cfg.S / 2))))
    rows = rows_of(n)
    t0 = time.perf_counter()
    oracle.attention_rows(hq, hk, hv, rows, scale=cfg.scale, causal=True)
    dt = time.perf_counter() - t0
    rate = flops_of(rows) / dt
    return {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} uniformly drawn query rows of {cfg.name} (causal fp64 rows, all allowed keys), "
                      f"{dt:.1f} s", "seconds": round(dt, 2),
            "extrapolated_full_problem_s": round(cfg.flops() / rate, 1)}


def run_reference(args):
    """The reference arm: the oracle as it stands, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = W.CFG4
    q, k, v = W.prefill_inputs(cfg, "cpu")
    for _ in range(args.warmup):
        cpu_baseline(cfg, q, k, v, seconds=1.0)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(cfg, q, k, v, seconds=args.cpu_seconds / max(1, args.steps)))
    wall = time.perf_counter() - t0
    value = statistics.mean(v_["value"] for v_ in vals)
    line = {"impl": "reference", "metric": "causal-adjusted attention TFLOP/s at S=128k (1 GPU); split-KV decode GB/s",
            "value": value, "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall * 1e3 / args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1), bf16 values read exactly)",
            "config": {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "S": cfg.S, "D": cfg.D,
                       "P": cfg.P, "layout": cfg.layout, "causal": True},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- profiling cases
PROFILE_CASES = {
    # tensor-core ring, causal zig-zag MHA with 1% of keys x8: q/k/v 268 MB each (> L2), one launch ~11 ms
    "tc": W.CFG3,
    # the timed S=128k GQA workload (only for single-pass ncu metrics)
    "tc_full": W.CFG4,
    # the same causal zig-zag GQA ring (group 4: the CTA-pair kernel) at S=32k, P=16: 1/16 of the
    # S=128k work, q 268 MB (> L2); a small case for full captures
    "tc_gqa": W.Prefill("ring_bf16_causal_zigzag_gqa_B1_Hq32_Hkv8_S32768_D128_P16", "bf16", True, "zigzag",
                        1, 32, 8, 32768, 128, 16, 4),
    # one kv head (4 query heads) of the S=128k GQA workload: the same K/V per kv head (67 MB) and the
    # same walk as the timed workload, whose 8 kv heads run one after another; 1/8 of its work
    "tc_gqa_1head": W.Prefill("ring_bf16_causal_zigzag_gqa_B1_Hq4_Hkv1_S131072_D128_P16", "bf16", True, "zigzag",
                              1, 4, 1, 131072, 128, 16, 4),
    # the same S=128k GQA workload under the other splits (same FLOPs, different tiles and order)
    "tc_full_contiguous": dataclasses.replace(W.CFG4, layout="contiguous",
                                              name="ring_bf16_causal_contiguous_gqa_B1_Hq32_Hkv8_S131072_D128_P16"),
    "tc_full_zigzag4": dataclasses.replace(W.CFG4, layout="zigzag4",
                                           name="ring_bf16_causal_zigzag4_gqa_B1_Hq32_Hkv8_S131072_D128_P16"),
    "tc_full_striped": dataclasses.replace(W.CFG4, layout="striped",
                                           name="ring_bf16_causal_striped_gqa_B1_Hq32_Hkv8_S131072_D128_P16"),
    # the S=128k GQA workload as P x P calls of ring_attn_step (state in HBM)
    "step_full": W.CFG4,
    # backward of the S=128k GQA workload (tensor cores: K/V-major then Q-major launch)
    "bwd_full": W.CFG4,
    # backward of the causal zig-zag MHA workload with 1% of keys x8 (a small case for ncu)
    "bwd": W.CFG3,
    # backward of one kv head (4 query heads) of the S=128k GQA workload: the same walk per kv
    # head as the timed backward, 1/8 of its work (a small case for ncu)
    "bwd_gqa_1head": W.Prefill("ring_bf16_causal_zigzag_gqa_B1_Hq4_Hkv1_S131072_D128_P16", "bf16", True, "zigzag",
                               1, 4, 1, 131072, 128, 16, 4),
    # split-KV decode on 4 x 65536-token sequences (K+V 1.07 GB > L2, lengths U[32k, 64k])
    "decode": W.Decode("decode_B4_Hq32_Hkv8_D128_ctx64k_P2", 4, 32, 8, 128, 1 << 16, 2, 5),
    "decode_fused": W.Decode("decode_B4_Hq32_Hkv8_D128_ctx64k_P2", 4, 32, 8, 128, 1 << 16, 2, 5),
    "decode_full": W.CFG5,
    # the same decode in one launch (partials plus the last-CTA merge)
    "decode_full_fused": W.CFG5,
    # the merge alone: B*Hq = 8192 rows of 32 float32 partials of 128 dims (134 MB > L2)
    "merge": W.MERGE_ONLY,
}


def run_profile(args):
    """Launch one kernel of the hot path `--steps` times after `--warmup`
    launches, for ncu captures (-k <kernel> -s <warmup>).  Prints the mean
    CUDA-event time per launch."""
    import context_exact_attention_ring_b200 as ra
    name = args.profile
    cfg = PROFILE_CASES[name]
    dev = torch.device("cuda", 0)
    if isinstance(cfg, W.Prefill) and name.startswith("bwd"):
        q, k, v = W.prefill_inputs(cfg, dev)
        g = torch.Generator(device=dev).manual_seed(cfg.seed + 7)
        dout = torch.randn(q.shape, generator=g, device=dev).to(q.dtype)
        out, lse = ra.ring_attn_fwd(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(int(ra.lib().ring_attn_bwd_workspace_bytes(cfg.B, cfg.Hq, cfg.S)), device=dev,
                         dtype=torch.uint8)
        fn = lambda: ra.ring_attn_bwd(q, k, v, out, lse, dout, cfg.P, causal=cfg.causal, layout=cfg.layout,
                                      scale=cfg.scale, dq=dq, dk=dk, dv=dv, workspace=ws)
        # the usual backward convention: 2.5x the forward's FLOPs (the two launches compute 3.5x)
        work, unit = 2.5 * cfg.flops() / 1e12, "TFLOP/s"
    elif isinstance(cfg, W.Prefill) and name.startswith("step"):
        q, k, v = W.prefill_inputs(cfg, dev)
        fn, _, _, _ = step_ring(ra, cfg, q, k, v, dev)
        work, unit = cfg.flops() / 1e12, "TFLOP/s"
    elif isinstance(cfg, W.Prefill):
        q, k, v = W.prefill_inputs(cfg, dev)
        out = torch.empty_like(q)
        lse = torch.empty((cfg.B, cfg.Hq, cfg.S), device=dev, dtype=torch.float32)
        fn = lambda: ra.ring_attn_fwd(q, k, v, cfg.P, causal=cfg.causal, layout=cfg.layout, scale=cfg.scale,
                                      out=out, lse=lse)
        work, unit = cfg.flops() / 1e12, "TFLOP/s"
    elif isinstance(cfg, W.Merge):
        part, plse = W.merge_inputs(cfg, dev)
        out = torch.empty((cfg.B, cfg.Hq, cfg.D), device=dev, dtype=torch.bfloat16)
        olse = torch.empty((cfg.B, cfg.Hq), device=dev, dtype=torch.float32)
        fn = lambda: ra.ring_attn_merge(part, plse, out=out, out_lse=olse)
        work, unit = merge_bytes(cfg) / 1e9, "GB/s"
    else:
        q, k, v, sl = W.decode_inputs(cfg, dev)
        lens = sl.cpu().numpy().astype(np.int64)
        ws = ra.decode_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.capacity, cfg.D, cfg.P, dev)
        part = torch.empty((cfg.B, cfg.Hq, cfg.P, cfg.D), device=dev, dtype=torch.float32)
        plse = torch.empty((cfg.B, cfg.Hq, cfg.P), device=dev, dtype=torch.float32)
        if name.endswith("_fused"):
            out = torch.empty((cfg.B, cfg.Hq, cfg.D), device=dev, dtype=torch.bfloat16)
            olse = torch.empty((cfg.B, cfg.Hq), device=dev, dtype=torch.float32)
            fn = lambda: ra.ring_attn_decode_fused(q, k, v, cfg.P, seqlens=sl, scale=cfg.scale, partials=part,
                                                   part_lse=plse, out=out, out_lse=olse, workspace=ws)
        else:
            fn = lambda: ra.ring_attn_decode_partial(q, k, v, sl, cfg.P, cfg.scale, partials=part, part_lse=plse,
                                                     workspace=ws)
        work, unit = decode_bytes(cfg, lens) / 1e9, "GB/s"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    print(json.dumps({"profile": name, "workload": cfg.name, "ms_per_launch": round(ms, 3),
                      "rate": round(work / (ms / 1e3), 1), "unit": unit}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile", choices=sorted(PROFILE_CASES), default=None,
                    help="launch one kernel of the hot path on a profiling workload (for ncu)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward timing after the main region")
    ap.add_argument("--no-step", action="store_true", help="skip the step-API timing after the main region")
    ap.add_argument("--no-merge", action="store_true", help="skip the merge-only timing after the main region")
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
        return
    if args.warmup < 3:
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
