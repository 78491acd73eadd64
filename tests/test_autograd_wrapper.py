"""The autograd wrapper of the binding (ring_attention / RingAttnFunction) on
the CPU: stand-ins for ring_attn_fwd and ring_attn_bwd (float64 attention
and its gradients from torch) check the wrapper's plumbing. P, the mask, the
split and the scale must pass through unchanged; the backward must receive
the forward's own out and lse; the gradients must return in (q, k, v) order
and equal torch autograd of the same attention.  Without stand-ins, host
tensors are refused as by every compute call."""
import pytest
import torch

import context_exact_attention_ring_b200 as ra


def _attn(q, k, v, causal, scale):
    G = q.shape[2] // k.shape[2]
    tq = q.transpose(1, 2)
    tk = k.repeat_interleave(G, dim=2).transpose(1, 2)
    tv = v.repeat_interleave(G, dim=2).transpose(1, 2)
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                            scale=scale).transpose(1, 2)


def test_gradients_flow_through_the_two_calls(monkeypatch):
    calls = {}

    def fake_fwd(q, k, v, P, causal=True, layout="zigzag", scale=None, out=None, lse=None):
        calls["fwd"] = (P, causal, layout, scale)
        with torch.no_grad():
            o = _attn(q, k, v, causal, scale)
        l = torch.zeros(q.shape[0], q.shape[2], q.shape[1], dtype=torch.float64)
        calls["saved"] = (o, l)
        return o, l

    def fake_bwd(q, k, v, out, lse, dout, P, causal=True, layout="zigzag", scale=None, **kw):
        calls["bwd"] = (P, causal, layout, scale)
        # the forward's own tensors (autograd returns saved outputs as new objects on the same storage)
        assert out.data_ptr() == calls["saved"][0].data_ptr() and lse.data_ptr() == calls["saved"][1].data_ptr()
        assert dout.is_contiguous() and dout.dtype == q.dtype
        with torch.enable_grad():                     # a backward runs with gradient recording off
            qq, kk, vv = (x.detach().clone().requires_grad_() for x in (q, k, v))
            _attn(qq, kk, vv, causal, scale).backward(dout)
        return qq.grad, kk.grad, vv.grad

    monkeypatch.setattr(ra, "ring_attn_fwd", fake_fwd)
    monkeypatch.setattr(ra, "ring_attn_bwd", fake_bwd)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(2, 48, 4, 16, generator=g, dtype=torch.float64, requires_grad=True)
    k = torch.randn(2, 48, 2, 16, generator=g, dtype=torch.float64, requires_grad=True)
    v = torch.randn(2, 48, 2, 16, generator=g, dtype=torch.float64, requires_grad=True)
    w = torch.randn(2, 48, 4, 16, generator=g, dtype=torch.float64)
    out = ra.ring_attention(q, k, v, 4, True, "zigzag4", 0.3)
    (out * w).sum().backward()
    assert calls["fwd"] == calls["bwd"] == (4, True, "zigzag4", 0.3)
    q2, k2, v2 = (x.detach().clone().requires_grad_() for x in (q, k, v))
    (_attn(q2, k2, v2, True, 0.3) * w).sum().backward()
    for a, b in ((q.grad, q2.grad), (k.grad, k2.grad), (v.grad, v2.grad)):
        torch.testing.assert_close(a, b, rtol=0, atol=1e-12)


def test_views_reach_the_library_as_contiguous_tensors(monkeypatch):
    seen = []

    def fake_fwd(q, k, v, P, causal=True, layout="zigzag", scale=None, out=None, lse=None):
        seen.extend(x.is_contiguous() for x in (q, k, v))
        with torch.no_grad():
            return _attn(q, k, v, causal, scale), torch.zeros(q.shape[0], q.shape[2], q.shape[1], dtype=q.dtype)

    monkeypatch.setattr(ra, "ring_attn_fwd", fake_fwd)
    base = torch.randn(2, 4, 48, 16, dtype=torch.float64)
    q = base.transpose(1, 2)                                  # [B, S, H, D] view, not contiguous
    assert not q.is_contiguous()
    ra.ring_attention(q, q, q, 4, True)
    assert seen == [True, True, True]


def test_host_tensors_are_refused():
    q = torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16, requires_grad=True)
    k = torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        ra.ring_attention(q, k, k, 2)
