"""The cross-GPU loops of ring.py with P = 2..4 ranks on one GPU, through the
library's own kernels (no stand-ins), against the fp64 oracle.

Each rank is a process of its own on cuda:0.  Ranks that share a GPU cannot
use NCCL, so the neighbour exchange (HostRing below) moves each block through
host memory over gloo: the send is copied to the host, crosses by gloo P2P and
is copied into the receiving rank's device buffer when the receive is waited
on.  Every wait is on the host; no kernel waits on another rank.  Per rank:

  * ring_forward: out and lse of the rank's shard against the oracle's rows;
  * ring_backward on the forward's own out and lse: dq, dk, dv of the shard
    (dK, dV travel with their block and come home) against oracle.attention_bwd;
  * RingAttention under torch autograd: loss = sum(out * dout), backward(),
    the leaf gradients against the same oracle;
  * helix_decode over KV shards filled round-robin block by block (the
    placement of ring_attn_kv_append), against attention over every valid key.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from context_exact_attention_ring_b200 import ring as R

pytestmark = pytest.mark.gpu

# tolerances of tests/helpers.py and tests/test_gpu_backward.py
TOL = {"bf16": (2e-2, 1e-3, 1e-2), "fp32": (1e-5, 1e-5, 2e-5)}   # out, lse, gradients (x max(1, |ref|))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _CopyBack:
    """Request of HostRing.shift: waits for the gloo transfers, then copies
    the received host buffers into the device tensors."""

    def __init__(self, reqs, host, dev):
        self.reqs, self.host, self.dev = reqs, host, dev

    def wait(self):
        for r in self.reqs:
            r.wait()
        for h, d in zip(self.host, self.dev):
            d.copy_(h.view(d.dtype) if h.dtype != d.dtype else h)


class HostRing(R.Ring):
    """ring.Ring for ranks that share one GPU: the block crosses through host
    memory over gloo instead of NCCL (bf16 travels as int16 bits)."""

    def shift(self, send, recv):
        if self.world == 1:
            return []
        nxt, prv = (self.rank + 1) % self.world, (self.rank - 1) % self.world
        wire = lambda t: t.view(torch.int16) if t.dtype == torch.bfloat16 else t
        hs = [wire(t).cpu() for t in send]
        hr = [torch.empty(t.shape, dtype=wire(t).dtype) for t in recv]
        ops = [dist.P2POp(dist.isend, h, nxt) for h in hs] + [dist.P2POp(dist.irecv, h, prv) for h in hr]
        return [_CopyBack(dist.batch_isend_irecv(ops), hr, recv)]


def _host_gather(t):
    """helix_decode's exchange over gloo: every rank's t, in rank order, on t's device."""
    h = t.cpu()
    got = [torch.empty_like(h) for _ in range(dist.get_world_size())]
    dist.all_gather(got, h)
    return [g.to(t.device) for g in got]


# (P, split, dtype, D, S, Hq, Hkv): ragged chunks (160 and 300 rows) and a GQA group of 4 included
CASES = [(2, "zigzag", "bf16", 128, 1024, 4, 2), (3, "striped", "bf16", 128, 1536, 4, 2),
         (4, "contiguous2", "bf16", 64, 1024, 4, 2), (4, "zigzag", "bf16", 128, 2048, 8, 2),
         (3, "zigzag", "fp32", 64, 960, 4, 2), (2, "striped", "fp32", 64, 600, 2, 1)]


def _prefill_case(P, layout, dtype, D, S, Hq, Hkv):
    import workloads as W
    return W.Prefill(f"ring_{layout}_P{P}_{dtype}", dtype, True, layout, 1, Hq, Hkv, S, D, P, 700 + P)


def _rank_prefill(rank, P, port, case, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=P, timeout=datetime.timedelta(seconds=120))
    try:
        import workloads as W
        cfg = _prefill_case(*case)
        layout = cfg.layout
        q, k, v = W.prefill_inputs(cfg, "cuda")             # every rank draws the whole problem, keeps its shard
        g = torch.Generator(device="cuda").manual_seed(cfg.seed + 1)
        dout = torch.randn(q.shape, generator=g, device="cuda").to(q.dtype)
        rows = R.shard_rows(cfg.S, P, layout, rank).cuda()
        qs, ks, vs, ds = (x[:, rows].contiguous() for x in (q, k, v, dout))
        ring = HostRing()
        out, lse = R.ring_forward(qs, ks, vs, layout=layout, scale=cfg.scale, ring=ring)
        dq, dk, dv = R.ring_backward(qs, ks, vs, out, lse, ds, layout=layout, scale=cfg.scale, ring=ring)
        # the same two loops under autograd
        lq, lk, lv = (x.clone().requires_grad_(True) for x in (qs, ks, vs))
        o2 = R.ring_attention(lq, lk, lv, layout=layout, scale=cfg.scale, ring=ring)
        (o2.float() * ds.float()).sum().backward()
        torch.cuda.synchronize()
        f = lambda t: t.detach().float().cpu().numpy()
        q_out.put((rank, rows.cpu().numpy(), f(out), f(lse), f(dq), f(dk), f(dv), f(o2), f(lq.grad), f(lk.grad),
                   f(lv.grad)))
    finally:
        dist.destroy_process_group()


def _spawn(target, P, *args):
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, P, port, *args, qq)) for r in range(P)]
    for p in procs:
        p.start()
    try:
        res = sorted((qq.get(timeout=600) for _ in range(P)), key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(120)
            if p.is_alive():
                p.kill()                      # this test's own child, by its handle
                p.join(10)
    assert all(p.exitcode == 0 for p in procs)
    return res


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"P{c[0]}-{c[1]}-{c[2]}-D{c[3]}-S{c[4]}-G{c[5] // c[6]}")
def test_ring_loops_on_P_ranks_of_one_gpu_against_the_oracle(case):
    import oracle
    import workloads as W
    from tests.helpers import margin, need_cuda
    need_cuda()
    cfg = _prefill_case(*case)
    P, dtype = cfg.P, cfg.dtype
    res = _spawn(_rank_prefill, P, case)
    q, k, v = W.prefill_inputs(cfg, "cuda")
    g = torch.Generator(device="cuda").manual_seed(cfg.seed + 1)
    dout = torch.randn(q.shape, generator=g, device="cuda").to(q.dtype)
    hq, hk, hv, hd = (x.float().cpu().numpy() for x in (q, k, v, dout))
    ro, rl = oracle.attention_rows(hq, hk, hv, oracle.all_rows(cfg.B, cfg.Hq, cfg.S), scale=cfg.scale, causal=True)
    ro = ro.reshape(cfg.B, cfg.Hq, cfg.S, cfg.D).transpose(0, 2, 1, 3)
    rl = rl.reshape(cfg.B, cfg.Hq, cfg.S)
    refs = oracle.attention_bwd(hq, hk, hv, hd, scale=cfg.scale, causal=True)
    t_out, t_lse, t_g = TOL[dtype]
    seen = np.zeros(cfg.S, dtype=int)
    for rank, rows, out, lse, dq, dk, dv, o2, gq, gk, gv in res:
        seen[rows] += 1
        margin("out", np.max(np.abs(out - ro[:, rows])), t_out)
        margin("lse", np.max(np.abs(lse - rl[:, :, rows])), t_lse)
        margin("out", np.max(np.abs(o2 - ro[:, rows])), t_out, "autograd")
        for name, got, auto, ref in (("dq", dq, gq, refs[0]), ("dk", dk, gk, refs[1]), ("dv", dv, gv, refs[2])):
            bound = t_g * max(1.0, float(np.max(np.abs(ref[:, rows]))))
            margin(name, np.max(np.abs(got - ref[:, rows])), bound)
            margin(name, np.max(np.abs(auto - ref[:, rows])), bound, "autograd")
    assert np.all(seen == 1)                 # the shards partition the sequence


def _rank_helix(rank, P, port, block, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=P, timeout=datetime.timedelta(seconds=120))
    try:
        import workloads as W
        cfg = W.Decode("helix_ranks", 3, 16, 4, 128, 4096 * P, P, 800 + P, fixed_lens=(1000, 37, 0))
        q, k, v, _ = W.decode_inputs(cfg, "cuda")
        # round-robin placement: append index n of a sequence goes to shard (n // block) % P
        lens = [1000, 37, 0]
        C = cfg.capacity // P
        ks = torch.zeros((cfg.B, C, cfg.Hkv, cfg.D), device="cuda", dtype=k.dtype)
        vs = torch.zeros_like(ks)
        fill = torch.zeros(cfg.B, dtype=torch.int32)
        for b, n in enumerate(lens):
            mine = [t for t in range(n) if (t // block) % P == rank]
            fill[b] = len(mine)
            if mine:
                ks[b, :len(mine)] = k[b, mine]
                vs[b, :len(mine)] = v[b, mine]
        out, lse = R.helix_decode(q, ks, vs, fill.cuda(), scale=cfg.scale, gather=_host_gather)
        torch.cuda.synchronize()
        q_out.put((rank, out.float().cpu().numpy(), lse.cpu().numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("P,block", [(2, 1), (3, 16), (4, 64)])
def test_helix_decode_on_P_ranks_of_one_gpu_against_the_oracle(P, block):
    import oracle
    import workloads as W
    from tests.helpers import margin, need_cuda
    need_cuda()
    res = _spawn(_rank_helix, P, block)
    cfg = W.Decode("helix_ranks", 3, 16, 4, 128, 4096 * P, P, 800 + P, fixed_lens=(1000, 37, 0))
    q, k, v, _ = W.decode_inputs(cfg, "cuda")
    hq, hk, hv = (x.float().cpu().numpy() for x in (q, k, v))
    G = cfg.Hq // cfg.Hkv
    for b, n in enumerate((1000, 37, 0)):
        for gk in range(cfg.Hkv):
            if n == 0:
                for rank, out, lse in res:
                    assert np.all(np.isneginf(lse[b])) and np.all(out[b] == 0)
                continue
            rows = [(0, h, 0) for h in range(G)]
            o, l = oracle.attention_rows(hq[b:b + 1, None, gk * G:(gk + 1) * G], hk[b:b + 1, :, gk:gk + 1],
                                         hv[b:b + 1, :, gk:gk + 1], rows, scale=cfg.scale, causal=False,
                                         kv_len=np.array([n]))
            for rank, out, lse in res:
                margin("out", np.max(np.abs(out[b, gk * G:(gk + 1) * G] - o)), 2e-2)
                margin("lse", np.max(np.abs(lse[b, gk * G:(gk + 1) * G] - l)), 1e-3)
