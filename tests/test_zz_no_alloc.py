"""The allocation-free decode entry point, ring_attn_decode_partial_noalloc.

Some callers cannot call cudaMalloc or hand the library a workspace -- a host
program whose own allocator owns all device memory, or code on a latency-
critical path where an allocation (which may synchronise the device) is not
acceptable.  For them the library keeps its decode scratch in one fixed
device array.  This test calls that entry point through the C ABI twice in a
row (the array keeps the previous call's contents, so the second call checks
that stale data does not leak into the result) and compares each result with
the workspace-based ring_attn_decode_partial, within the decode tolerances
used by the other tests.  It also checks that sizes needing more scratch than
the array holds are refused before anything is launched.

This file is collected last so that a run stopping at the first failure has
already run every other test; it passes alone or after them.
"""
import ctypes

import numpy as np
import pytest
import torch

import context_exact_attention_ring_b200 as ra
import workloads as W
from tests.helpers import TOL_BF16_LSE, TOL_BF16_OUT, host, need_cuda

pytestmark = pytest.mark.gpu

SCRATCH_MAX = 40 << 20


def call_noalloc(q, k, v, sl, partials, part_lse, P, scale):
    B, Hq, D = q.shape
    _, Smax, Hkv, _ = k.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return ra.lib().ring_attn_decode_partial_noalloc(
        p(q), p(k), p(v), p(sl), p(partials), p(part_lse), B, Hq, Hkv, Smax, D, P, scale, ra.RING_BF16,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def compare(part, plse, ref_part, ref_plse):
    a, b = host(plse), host(ref_plse)
    assert np.array_equal(np.isneginf(a), np.isneginf(b))
    fin = np.isfinite(b)
    assert np.all(np.isfinite(a[fin]))
    assert np.max(np.abs(a[fin] - b[fin])) <= TOL_BF16_LSE
    assert np.max(np.abs(host(part) - host(ref_part))) <= TOL_BF16_OUT


@pytest.mark.parametrize("Hq,Hkv,lens,cap,P", [
    (8, 2, (0, 1, 5000, 8192, 8193, 32768, 12345, 20000), 32768, 4),
    (32, 8, (70000, 131072, 65537, 100), 131072, 8),
])
def test_noalloc_decode_matches_workspace_entry_point(Hq, Hkv, lens, cap, P):
    need_cuda()
    cfg = W.Decode("noalloc", len(lens), Hq, Hkv, 128, cap, P, 91, fixed_lens=tuple(lens))
    q, k, v, sl = W.decode_inputs(cfg, "cuda")
    ref_part, ref_plse = ra.ring_attn_decode_partial(q, k, v, sl, P, cfg.scale)
    torch.cuda.synchronize()
    assert ra.ring_attn_device_error()[0] == ra.RING_OK
    for _ in range(2):
        part = torch.full_like(ref_part, float("nan"))
        plse = torch.full_like(ref_plse, float("nan"))
        assert call_noalloc(q, k, v, sl, part, plse, P, cfg.scale) == ra.RING_OK
        torch.cuda.synchronize()
        assert ra.ring_attn_device_error()[0] == ra.RING_OK
        compare(part, plse, ref_part, ref_plse)
    # the merged results agree as well
    o1, l1 = ra.ring_attn_merge(part, plse)
    o2, l2 = ra.ring_attn_merge(ref_part, ref_plse)
    assert (o1.float() - o2.float()).abs().max().item() <= TOL_BF16_OUT


def test_noalloc_rejects_sizes_beyond_its_scratch():
    need_cuda()
    # B=64, Hq=32, Hkv=8, 2^20 tokens in 32 chunks needs far more than the fixed scratch
    B, Hq, Hkv, Smax, D, P = 64, 32, 8, 1 << 20, 128, 32
    assert ra.ring_attn_decode_workspace_bytes(B, Hq, Hkv, Smax, D, P) > SCRATCH_MAX
    dummy = torch.empty(64, device="cuda", dtype=torch.float32)
    p = ctypes.c_void_p(dummy.data_ptr())
    st = ra.lib().ring_attn_decode_partial_noalloc(p, p, p, p, p, p, B, Hq, Hkv, Smax, D, P, 0.088, ra.RING_BF16,
                                                   None)
    assert st == ra.RING_EINVAL
    # and the full-size 1M-token decode of the benchmark fits
    assert ra.ring_attn_decode_workspace_bytes(8, 32, 8, 1 << 20, 128, 32) <= SCRATCH_MAX
