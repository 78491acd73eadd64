"""The library's calls inside a CUDA graph: a prefill ring and a split-KV
decode are captured once and replayed.  Every call is asynchronous on the
current stream and allocates nothing, so a replay must give exactly the eager
results (the kernels fix their summation order), also after the inputs are
overwritten in place (the graph reads the buffers, not values captured with
it)."""
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import workloads as W
from tests.helpers import need_cuda

pytestmark = pytest.mark.gpu


def test_prefill_and_decode_replay_in_a_cuda_graph():
    need_cuda()
    pcfg = W.Prefill("graph_prefill", "bf16", True, "zigzag", 1, 8, 4, 4096, 128, 4, 21)
    q, k, v = W.prefill_inputs(pcfg, "cuda")
    dcfg = W.Decode("graph_decode", 3, 16, 4, 128, 16384, 4, 22, fixed_lens=(16384, 9000, 77))
    dq, dk, dv, sl = W.decode_inputs(dcfg, "cuda")
    ws = ra.decode_workspace(dcfg.B, dcfg.Hq, dcfg.Hkv, dcfg.capacity, dcfg.D, dcfg.P)

    def buffers():
        return dict(out=torch.empty_like(q), lse=torch.empty((pcfg.B, pcfg.Hq, pcfg.S), device="cuda"),
                    part=torch.empty((dcfg.B, dcfg.Hq, dcfg.P, dcfg.D), device="cuda"),
                    plse=torch.empty((dcfg.B, dcfg.Hq, dcfg.P), device="cuda"),
                    dout=torch.empty((dcfg.B, dcfg.Hq, dcfg.D), device="cuda", dtype=torch.bfloat16),
                    dlse=torch.empty((dcfg.B, dcfg.Hq), device="cuda"))

    def step(b):
        ra.ring_attn_fwd(q, k, v, pcfg.P, causal=True, layout=pcfg.layout, scale=pcfg.scale, out=b["out"],
                         lse=b["lse"])
        ra.ring_attn_decode(dq, dk, dv, sl, dcfg.P, dcfg.scale, partials=b["part"], part_lse=b["plse"],
                            out=b["dout"], out_lse=b["dlse"], workspace=ws)

    eager, graphed = buffers(), buffers()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(graphed)                       # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(graphed)

    for round_ in range(2):
        if round_ == 1:                     # new inputs, same buffers
            gen = torch.Generator(device="cuda").manual_seed(23)
            q.copy_(torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype))
            dq.copy_(torch.randn(dq.shape, generator=gen, device="cuda").to(dq.dtype))
        step(eager)
        g.replay()
        torch.cuda.synchronize()
        assert ra.ring_attn_device_error()[0] == ra.RING_OK
        for name in eager:
            assert torch.equal(eager[name], graphed[name]), (round_, name)
