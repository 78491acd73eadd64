"""Exact ring attention on one B200 (sm_100a), emulating P virtual ranks.

A thin ctypes binding over ``libringattn_sm100a.so`` (C ABI in
``include/ring_attn.h``).  It only marshals arguments: torch tensors are
passed by device pointer and the current torch CUDA stream; every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback --
importing works without a GPU (for the host-side helpers), but every compute
call raises if the library or a CUDA device is missing.

Names follow the C ABI:
  ring_attn_fwd, ring_attn_fwd_counted, ring_attn_fwd_simt,
  ring_attn_state_init, ring_attn_step, ring_attn_state_finalize,
  ring_attn_decode_partial, ring_attn_merge, ring_attn_decode,
  ring_attn_decode_workspace_bytes, ring_attn_decode_fused,
  ring_attn_kv_append, ring_attn_sched_stats, ring_attn_device_error;
and ring_attention (RingAttnFunction), the forward and backward under autograd.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libringattn_sm100a.so")

RING_OK, RING_EINVAL, RING_EUNSUPPORTED, RING_ECUDA, RING_ETIMEOUT, RING_ECAPACITY = 0, -1, -2, -3, -4, -5
RING_CONTIGUOUS, RING_ZIGZAG, RING_STRIPED = 0, 1, 2
RING_MAX_CHUNKS_PER_RANK = 8
RING_BF16, RING_FP32 = 0, 1
LAYOUTS = {"contiguous": RING_CONTIGUOUS, "zigzag": RING_ZIGZAG, "striped": RING_STRIPED}


def ring_split(split: str, k: int = 0) -> int:
    """The C ABI's split code RING_SPLIT(split, k): k chunks per rank (0 = the split's default)."""
    return LAYOUTS[split] | (int(k) << 8)

EXPORTED = (
    "ring_attn_fwd", "ring_attn_fwd_counted", "ring_attn_fwd_simt", "ring_attn_state_init", "ring_attn_step",
    "ring_attn_state_finalize", "ring_attn_decode_partial", "ring_attn_decode_workspace_bytes", "ring_attn_decode",
    "ring_attn_merge", "ring_attn_sched_stats", "ring_attn_device_error", "ring_attn_strerror",
    "ring_attn_version", "ring_attn_built_arch", "ring_attn_selftest_wait", "ring_attn_decode_partial_noalloc",
    "ring_attn_decode_fused", "ring_attn_kv_append", "ring_attn_bwd", "ring_attn_bwd_delta",
    "ring_attn_bwd_workspace_bytes", "ring_attn_step_bwd", "ring_attn_bwd_simt",
)


class RingError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} ({status})")


class ChunkIds(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int32), ("q", ctypes.c_int32 * RING_MAX_CHUNKS_PER_RANK),
                ("n_kv", ctypes.c_int32), ("kv", ctypes.c_int32 * RING_MAX_CHUNKS_PER_RANK),
                ("chunk_len", ctypes.c_int32), ("causal", ctypes.c_int32), ("stripes", ctypes.c_int32)]


_lib = None


def lib():
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m context_exact_attention_ring_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    prefill = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32]
    sig = {
        "ring_attn_fwd": prefill + [vp],
        "ring_attn_fwd_counted": prefill + [vp, vp],
        "ring_attn_fwd_simt": prefill + [vp],
        "ring_attn_state_init": [vp, vp, vp, i32, i32, i32, i32, vp],
        "ring_attn_step": [vp, vp, vp, vp, vp, vp, ctypes.POINTER(ChunkIds), i32, i32, i32, i32, f32, i32, vp],
        "ring_attn_state_finalize": [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp],
        "ring_attn_decode_partial": [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, sz, vp],
        "ring_attn_decode": [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, sz, vp],
        "ring_attn_decode_partial_noalloc": [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp],
        "ring_attn_decode_fused": [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, sz,
                                   vp],
        "ring_attn_kv_append": [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp],
        "ring_attn_bwd": [vp] * 9 + [i32] * 8 + [f32, i32, vp, sz, vp],
        "ring_attn_bwd_simt": [vp] * 9 + [i32] * 8 + [f32, i32, vp, sz, vp],
        "ring_attn_bwd_delta": [vp, vp, vp, i32, i32, i32, i32, i32, vp],
        "ring_attn_step_bwd": [vp] * 9 + [ctypes.POINTER(ChunkIds), i32, i32, i32, i32, f32, i32, vp],
        "ring_attn_merge": [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp],
        "ring_attn_sched_stats": [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp],
        "ring_attn_device_error": [ctypes.POINTER(ctypes.c_int)],
        "ring_attn_strerror": [i32],
        "ring_attn_version": [],
        "ring_attn_selftest_wait": [i32, vp],
        "ring_attn_built_arch": [],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.ring_attn_strerror.restype = ctypes.c_char_p
    L.ring_attn_decode_workspace_bytes.argtypes = [i32] * 6
    L.ring_attn_decode_workspace_bytes.restype = sz
    L.ring_attn_bwd_workspace_bytes.argtypes = [i32] * 3
    L.ring_attn_bwd_workspace_bytes.restype = sz
    _lib = L
    return L


def strerror(status: int) -> str:
    try:
        return lib().ring_attn_strerror(int(status)).decode()
    except RuntimeError:
        return str(status)


def _check(status: int, what: str):
    if status != RING_OK:
        raise RingError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return RING_BF16
    if t.dtype == torch.float32:
        return RING_FP32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _layout(layout) -> int:
    """A split code from 'contiguous' | 'zigzag' | 'striped', optionally with the
    chunks per rank appended ('zigzag4', 'contiguous2'), or an int code."""
    if not isinstance(layout, str):
        return int(layout)
    name = layout.rstrip("0123456789")
    k = layout[len(name):]
    if name not in LAYOUTS:
        raise ValueError(f"unknown split {layout!r}")
    return ring_split(name, int(k) if k else 0)


def _prefill(name, q, k, v, P, causal, layout, scale, out, lse, extra=()):
    _cuda(q, k, v, out, lse)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, S, Hkv, D) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q [B,S,Hq,D], k/v [B,S,Hkv,D] of one dtype expected")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, S), device=q.device, dtype=torch.float32)
    st = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, S, D, int(P),
                               int(bool(causal)), _layout(layout), scale, _dtype_code(q), *extra, _stream())
    _check(st, name)
    return out, lse


def ring_attn_fwd(q, k, v, P, causal=True, layout="zigzag", scale=None, out=None, lse=None):
    """Whole ring (all P virtual ranks) in one launch.  Returns (out, lse)."""
    return _prefill("ring_attn_fwd", q, k, v, P, causal, layout, scale, out, lse)


def ring_attn_fwd_counted(q, k, v, P, causal=True, layout="zigzag", scale=None, out=None, lse=None, counters=None):
    """ring_attn_fwd plus the device-side work counters [full, partial, pairs of rank 0..P-1]."""
    if counters is None:
        counters = torch.zeros(2 + int(P), device=q.device, dtype=torch.int64)
    out, lse = _prefill("ring_attn_fwd_counted", q, k, v, P, causal, layout, scale, out, lse,
                        extra=(_ptr(counters),))
    return out, lse, counters


def ring_attn_fwd_simt(q, k, v, P, causal=True, layout="zigzag", scale=None, out=None, lse=None):
    """The CUDA-core cross-check path of ring_attn_fwd."""
    return _prefill("ring_attn_fwd_simt", q, k, v, P, causal, layout, scale, out, lse)


def ring_attn_bwd_delta(out, dout, delta=None):
    """delta [B,Hq,S] = rowsum(dout * out) for out, dout [B,S,Hq,D]."""
    _cuda(out, dout, delta)
    B, S, Hq, D = out.shape
    if delta is None:
        delta = torch.empty((B, Hq, S), device=out.device, dtype=torch.float32)
    _check(lib().ring_attn_bwd_delta(_ptr(out), _ptr(dout), _ptr(delta), B, Hq, S, D, _dtype_code(out), _stream()),
           "ring_attn_bwd_delta")
    return delta


def ring_attn_bwd(q, k, v, out, lse, dout, P, causal=True, layout="zigzag", scale=None, dq=None, dk=None, dv=None,
                  workspace=None, _name="ring_attn_bwd"):
    """Gradients (dq, dk, dv) of the whole ring for the output gradient dout."""
    _cuda(q, k, v, out, lse, dout, dq, dk, dv, workspace)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if out.shape != q.shape or dout.shape != q.shape or dout.dtype != q.dtype or out.dtype != q.dtype:
        raise ValueError("out and dout must match q")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(int(lib().ring_attn_bwd_workspace_bytes(B, Hq, S)), device=q.device,
                                dtype=torch.uint8)
    st = getattr(lib(), _name)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, Hq, Hkv, S, D, int(P), int(bool(causal)), _layout(layout), scale,
                               _dtype_code(q), _ptr(workspace), workspace.numel(), _stream())
    _check(st, _name)
    return dq, dk, dv


def ring_attn_bwd_simt(q, k, v, out, lse, dout, P, causal=True, layout="zigzag", scale=None, dq=None, dk=None,
                       dv=None, workspace=None):
    """The CUDA-core cross-check path of ring_attn_bwd."""
    return ring_attn_bwd(q, k, v, out, lse, dout, P, causal, layout, scale, dq, dk, dv, workspace,
                         _name="ring_attn_bwd_simt")


def ring_attn_step_bwd(q_shard, kchunk, vchunk, dout_shard, lse, delta, dq_acc, dk_acc, dv_acc, q_ids, kv_ids,
                       chunk_len, causal=True, scale=None, stripes=0):
    """One backward hop: add this block's share to dq_acc and the shard's share
    to dk_acc, dv_acc (float32, in place)."""
    _cuda(q_shard, kchunk, vchunk, dout_shard, lse, delta, dq_acc, dk_acc, dv_acc)
    B, Sq, Hq, D = q_shard.shape
    Hkv = kchunk.shape[2]
    ids = _chunk_ids(q_ids, kv_ids, chunk_len, causal, stripes)
    if Sq != len(q_ids) * chunk_len or kchunk.shape[1] != len(kv_ids) * chunk_len:
        raise ValueError("shard / chunk buffers do not match the chunk ids")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = lib().ring_attn_step_bwd(_ptr(q_shard), _ptr(kchunk), _ptr(vchunk), _ptr(dout_shard), _ptr(lse),
                                  _ptr(delta), _ptr(dq_acc), _ptr(dk_acc), _ptr(dv_acc), ctypes.byref(ids), B, Hq,
                                  Hkv, D, scale, _dtype_code(q_shard), _stream())
    _check(st, "ring_attn_step_bwd")


def _chunk_ids(q_ids, kv_ids, chunk_len, causal, stripes):
    if not (1 <= len(q_ids) <= RING_MAX_CHUNKS_PER_RANK and 1 <= len(kv_ids) <= RING_MAX_CHUNKS_PER_RANK):
        raise ValueError(f"1..{RING_MAX_CHUNKS_PER_RANK} chunk ids expected")
    ids = ChunkIds()
    ids.n_q = len(q_ids)
    ids.n_kv = len(kv_ids)
    for i, c in enumerate(q_ids):
        ids.q[i] = int(c)
    for i, c in enumerate(kv_ids):
        ids.kv[i] = int(c)
    ids.chunk_len = int(chunk_len)
    ids.causal = int(bool(causal))
    ids.stripes = int(stripes)
    return ids


def ring_attn_state_init(m, l, O):
    _cuda(m, l, O)
    B, Hq, S = m.shape
    _check(lib().ring_attn_state_init(_ptr(m), _ptr(l), _ptr(O), B, Hq, S, O.shape[-1], _stream()),
           "ring_attn_state_init")


def new_state(B, Hq, S_loc, D, device="cuda"):
    """Allocate (with torch) and initialise a ring state (m, l, O)."""
    m = torch.empty((B, Hq, S_loc), device=device, dtype=torch.float32)
    l = torch.empty_like(m)
    O = torch.empty((B, S_loc, Hq, D), device=device, dtype=torch.float32)
    ring_attn_state_init(m, l, O)
    return m, l, O


def ring_attn_step(q_shard, kchunk, vchunk, m, l, O, q_ids, kv_ids, chunk_len, causal=True, scale=None, stripes=0):
    """One ring hop: fold the held K/V chunks (global ids kv_ids) into the
    state of the query shard (global chunk ids q_ids), in place.  With
    stripes=P the shard and the block are stripes of the striped split and
    q_ids / kv_ids hold the two ranks."""
    _cuda(q_shard, kchunk, vchunk, m, l, O)
    B, Sq, Hq, D = q_shard.shape
    Hkv = kchunk.shape[2]
    ids = _chunk_ids(q_ids, kv_ids, chunk_len, causal, stripes)
    if Sq != len(q_ids) * chunk_len or kchunk.shape[1] != len(kv_ids) * chunk_len:
        raise ValueError("shard / chunk buffers do not match the chunk ids")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = lib().ring_attn_step(_ptr(q_shard), _ptr(kchunk), _ptr(vchunk), _ptr(m), _ptr(l), _ptr(O),
                              ctypes.byref(ids), B, Hq, Hkv, D, scale, _dtype_code(q_shard), _stream())
    _check(st, "ring_attn_step")


def ring_attn_state_finalize(m, l, O, dtype=torch.bfloat16, out=None, lse=None):
    _cuda(m, l, O)
    B, S, Hq, D = O.shape
    if out is None:
        out = torch.empty((B, S, Hq, D), device=O.device, dtype=dtype)
    if lse is None:
        lse = torch.empty((B, Hq, S), device=O.device, dtype=torch.float32)
    st = lib().ring_attn_state_finalize(_ptr(m), _ptr(l), _ptr(O), _ptr(out), _ptr(lse), B, Hq, S, D,
                                        _dtype_code(out), _stream())
    _check(st, "ring_attn_state_finalize")
    return out, lse


def ring_attn_decode_workspace_bytes(B, Hq, Hkv, Smax, D, P) -> int:
    return int(lib().ring_attn_decode_workspace_bytes(B, Hq, Hkv, Smax, D, P))


def decode_workspace(B, Hq, Hkv, Smax, D, P, device="cuda"):
    """A zeroed workspace for the decode calls (allocated with torch)."""
    n = ring_attn_decode_workspace_bytes(B, Hq, Hkv, Smax, D, P)
    if n == 0:
        raise ValueError("bad decode sizes")
    return torch.zeros(n, device=device, dtype=torch.uint8)


def _decode_shapes(q, k, seqlens, P):
    B, Hq, D = q.shape
    _, Smax, Hkv, _ = k.shape
    if seqlens.dtype != torch.int32 or seqlens.shape != (B,):
        raise ValueError("seqlens must be int32 [B]")
    return B, Hq, Hkv, Smax, D


def ring_attn_decode_partial(q, k, v, seqlens, P, scale=None, partials=None, part_lse=None, workspace=None):
    _cuda(q, k, v, seqlens, partials, part_lse, workspace)
    B, Hq, Hkv, Smax, D = _decode_shapes(q, k, seqlens, P)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if partials is None:
        partials = torch.empty((B, Hq, P, D), device=q.device, dtype=torch.float32)
    if part_lse is None:
        part_lse = torch.empty((B, Hq, P), device=q.device, dtype=torch.float32)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, Smax, D, P, q.device)
    st = lib().ring_attn_decode_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), _ptr(partials), _ptr(part_lse),
                                        B, Hq, Hkv, Smax, D, int(P), scale, _dtype_code(q), _ptr(workspace),
                                        workspace.numel(), _stream())
    _check(st, "ring_attn_decode_partial")
    return partials, part_lse


def ring_attn_decode_partial_noalloc(q, k, v, seqlens, P, scale=None, partials=None, part_lse=None):
    """ring_attn_decode_partial using the library's fixed scratch array (no
    workspace, no allocation inside the call; see include/ring_attn.h).
    Pass preallocated `partials` and `part_lse` to avoid torch allocations."""
    _cuda(q, k, v, seqlens, partials, part_lse)
    B, Hq, Hkv, Smax, D = _decode_shapes(q, k, seqlens, P)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if partials is None:
        partials = torch.empty((B, Hq, P, D), device=q.device, dtype=torch.float32)
    if part_lse is None:
        part_lse = torch.empty((B, Hq, P), device=q.device, dtype=torch.float32)
    st = lib().ring_attn_decode_partial_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), _ptr(partials),
                                                _ptr(part_lse), B, Hq, Hkv, Smax, D, int(P), scale, _dtype_code(q),
                                                _stream())
    _check(st, "ring_attn_decode_partial_noalloc")
    return partials, part_lse


def ring_attn_merge(partials, part_lse, out=None, out_lse=None, dtype=torch.bfloat16):
    _cuda(partials, part_lse, out, out_lse)
    B, Hq, P, D = partials.shape
    if out is None:
        out = torch.empty((B, Hq, D), device=partials.device, dtype=dtype)
    if out_lse is None:
        out_lse = torch.empty((B, Hq), device=partials.device, dtype=torch.float32)
    st = lib().ring_attn_merge(_ptr(partials), _ptr(part_lse), _ptr(out), _ptr(out_lse), B, Hq, P, D,
                               _dtype_code(out), _stream())
    _check(st, "ring_attn_merge")
    return out, out_lse


def ring_attn_decode(q, k, v, seqlens, P, scale=None, partials=None, part_lse=None, out=None, out_lse=None,
                     workspace=None):
    """Split-KV decode (per-chunk partials, then the merge).  Returns (out, out_lse)."""
    _cuda(q, k, v, seqlens, partials, part_lse, out, out_lse, workspace)
    B, Hq, Hkv, Smax, D = _decode_shapes(q, k, seqlens, P)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dev = q.device
    if partials is None:
        partials = torch.empty((B, Hq, P, D), device=dev, dtype=torch.float32)
    if part_lse is None:
        part_lse = torch.empty((B, Hq, P), device=dev, dtype=torch.float32)
    if out is None:
        out = torch.empty((B, Hq, D), device=dev, dtype=torch.bfloat16)
    if out_lse is None:
        out_lse = torch.empty((B, Hq), device=dev, dtype=torch.float32)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, Smax, D, P, dev)
    st = lib().ring_attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), _ptr(partials), _ptr(part_lse), _ptr(out),
                                _ptr(out_lse), B, Hq, Hkv, Smax, D, int(P), scale, _dtype_code(q), _ptr(workspace),
                                workspace.numel(), _stream())
    _check(st, "ring_attn_decode")
    return out, out_lse


def ring_attn_decode_fused(q, k, v, P, seqlens=None, shard_lens=None, scale=None, partials=None, part_lse=None,
                           out=None, out_lse=None, workspace=None):
    """Split-KV decode in one launch (partials plus the last-CTA merge).  Valid
    rows come from `seqlens` [B] (whole-cache lengths) or `shard_lens` [B,P]
    (per-chunk fill counts, e.g. after ring_attn_kv_append).  Returns (out, out_lse)."""
    if (seqlens is None) == (shard_lens is None):
        raise ValueError("give exactly one of seqlens / shard_lens")
    _cuda(q, k, v, seqlens, shard_lens, partials, part_lse, out, out_lse, workspace)
    B, Hq, D = q.shape
    _, Smax, Hkv, _ = k.shape
    lens = seqlens if seqlens is not None else shard_lens
    if lens.dtype != torch.int32 or lens.shape != ((B,) if seqlens is not None else (B, int(P))):
        raise ValueError("seqlens must be int32 [B], shard_lens int32 [B,P]")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dev = q.device
    if partials is None:
        partials = torch.empty((B, Hq, P, D), device=dev, dtype=torch.float32)
    if part_lse is None:
        part_lse = torch.empty((B, Hq, P), device=dev, dtype=torch.float32)
    if out is None:
        out = torch.empty((B, Hq, D), device=dev, dtype=torch.bfloat16)
    if out_lse is None:
        out_lse = torch.empty((B, Hq), device=dev, dtype=torch.float32)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, Smax, D, P, dev)
    st = lib().ring_attn_decode_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(seqlens), _ptr(shard_lens), _ptr(partials),
                                      _ptr(part_lse), _ptr(out), _ptr(out_lse), B, Hq, Hkv, Smax, D, int(P), scale,
                                      _dtype_code(q), _ptr(workspace), workspace.numel(), _stream())
    _check(st, "ring_attn_decode_fused")
    return out, out_lse


def ring_attn_kv_append(k_cache, v_cache, k_new, v_new, shard_lens, n_appended, P, block):
    """Append k_new / v_new [B,T,Hkv,D] to the P-way sharded cache [B,Smax,Hkv,D],
    round-robin by blocks of `block` tokens; shard_lens [B,P] and n_appended [B]
    (int32, device) advance in place."""
    _cuda(k_cache, v_cache, k_new, v_new, shard_lens, n_appended)
    B, Smax, Hkv, D = k_cache.shape
    T = k_new.shape[1]
    if k_new.shape != (B, T, Hkv, D) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("k_new/v_new [B,T,Hkv,D] and caches [B,Smax,Hkv,D] expected")
    if k_new.dtype != k_cache.dtype or v_new.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise ValueError("one dtype for caches and new tokens")
    if shard_lens.dtype != torch.int32 or shard_lens.shape != (B, int(P)):
        raise ValueError("shard_lens must be int32 [B,P]")
    if n_appended.dtype != torch.int32 or n_appended.shape != (B,):
        raise ValueError("n_appended must be int32 [B]")
    st = lib().ring_attn_kv_append(_ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new), _ptr(shard_lens),
                                   _ptr(n_appended), B, T, Hkv, Smax, D, int(P), int(block),
                                   _dtype_code(k_cache), _stream())
    _check(st, "ring_attn_kv_append")


class RingAttnFunction(torch.autograd.Function):
    """Autograd over the whole ring: forward is ring_attn_fwd, backward is
    ring_attn_bwd on the saved q, k, v, out and lse.  Only marshalling: both
    passes run in the library's kernels."""

    @staticmethod
    def forward(ctx, q, k, v, P, causal=True, layout="zigzag", scale=None):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()   # views (e.g. transposes) are copied once
        out, lse = ring_attn_fwd(q, k, v, P, causal, layout, scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.cfg = (P, causal, layout, scale)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        P, causal, layout, scale = ctx.cfg
        dq, dk, dv = ring_attn_bwd(q, k, v, out, lse, dout.to(q.dtype).contiguous(), P, causal, layout, scale)
        return dq, dk, dv, None, None, None, None


def ring_attention(q, k, v, P, causal=True, layout="zigzag", scale=None):
    """out = ring attention of q, k, v that autograd can differentiate
    (RingAttnFunction)."""
    return RingAttnFunction.apply(q, k, v, P, causal, layout, scale)


def ring_attn_sched_stats(S, P, causal, layout, tile_q=128, tile_k=128):
    """Host-side scheduler counts: (per_rank_pairs[P], full, partial, skipped)."""
    per = (ctypes.c_int64 * int(P))()
    f, pa, sk = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    st = lib().ring_attn_sched_stats(int(S), int(P), int(bool(causal)), _layout(layout), int(tile_q), int(tile_k),
                                     ctypes.cast(per, ctypes.c_void_p), ctypes.byref(f), ctypes.byref(pa),
                                     ctypes.byref(sk))
    _check(st, "ring_attn_sched_stats")
    return list(per), f.value, pa.value, sk.value


def ring_attn_selftest_wait(limit_us=1000):
    """Run the bounded-wait self test (see the header); check with ring_attn_device_error()."""
    _check(lib().ring_attn_selftest_wait(int(limit_us), _stream()), "ring_attn_selftest_wait")


def ring_attn_device_error():
    """Synchronise and return (status, site) of the device error word (cleared)."""
    where = ctypes.c_int(0)
    st = lib().ring_attn_device_error(ctypes.byref(where))
    return st, where.value
