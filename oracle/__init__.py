"""Oracle for the ring-attention hot path: plain, slow, fp64, CPU only.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``context_exact_attention_ring_b200``) never
imports it, and it imports nothing from the product: the two share no code.

Contents
  attn_fp64.c   the definition of (causal / GQA / variable-length) attention
                in fp64, threaded over query rows          -> ``attention_rows``;
                and its gradients (the calculus of that
                definition; the pages give no backward)    -> ``attention_bwd``,
                ``attention_bwd_dq_rows`` (sampled rows)
  brute.py      a second, independent numpy fp64 oracle that materialises the
                whole score matrix (tiny shapes only)     -> ``brute``
  schedule.py   the chunk assignment / ring rotation / causal workload
                enumerators and the tile classifier       -> ``schedule``
  streaming.py  the online-softmax recurrence of "Lesson 8: Context
                Parallelism" section 3, in fp64, used only to pin that the
                blockwise recurrence reaches the oracle's value.
  merge.py      the direct formula for combining normalised partial
                attention results (O_p, lse_p).
  helix.py      the round-robin placement of appended KV tokens across
                KV-parallel ranks ("NVIDIA unveils Helix Parallelism"),
                simulated one token at a time.

Parity pins for every function live in ``tests/test_oracle_*.py``; none of
them is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_fp64.c")
_LIB = os.path.join(_HERE, "liboracle_fp64.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_fp64.c with gcc (plain -O2, no fast-math: the oracle keeps
    IEEE double semantics).  Returns the path of the shared library.

    Plumbing (builds the C oracle); no passage.
    """
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-D_GNU_SOURCE",
             "-shared", "-fPIC", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_attn_rows.restype = ctypes.c_int
        lib.oracle_attn_rows.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.oracle_cores.restype = ctypes.c_int
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.oracle_attn_bwd_dq_rows.restype = ctypes.c_int
        lib.oracle_attn_bwd_dq_rows.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int]
        _lib = lib
    return _lib


def cores() -> int:
    """Host cores available to the oracle's threads.

    Plumbing; no passage.
    """
    return int(_load().oracle_cores())


def _f32(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.float32:
        a = a.astype(np.float32)
    return np.ascontiguousarray(a)


def attention_rows(q, k, v, rows, *, scale: float, causal: bool,
                   qpos=None, kpos=None, kv_len=None, threads: int = 0):
    """fp64 attention for the requested query rows.

    q [B,Sq,Hq,D], k/v [B,Skv,Hkv,D] (any float dtype; read as float32, which
    holds bf16 values exactly).  ``rows`` is an int array [n,3] of (b, h, i).
    ``qpos``/``kpos`` give global token positions (default: the row index),
    ``kv_len`` [B] limits the keys of each batch entry.
    Returns (out [n,D] float64, lse [n] float64); lse is the natural log.

    Follows the definition of attention in "Lesson 8: Context Parallelism",
    section 1, with the causal rule of section 4 (attn_fp64.c).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Sq, Hq, D = q.shape
    Bk, Skv, Hkv, Dk = k.shape
    assert Bk == B and Dk == D and v.shape == k.shape and Hq % Hkv == 0
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    keep = []

    def ptr(a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(np.asarray(a, dtype=dt))
        keep.append(a)
        return a.ctypes.data

    rc = _load().oracle_attn_rows(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Sq, Skv, Hq, Hkv, D,
        ptr(qpos, np.int64), ptr(kpos, np.int64), int(bool(causal)), ptr(kv_len, np.int64),
        float(scale), rows.ctypes.data, n, out.ctypes.data, lse.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError(f"oracle_attn_rows failed with code {rc}")
    return out, lse


def attention_bwd(q, k, v, dout, *, scale: float, causal: bool, qpos=None, kpos=None, threads: int = 0):
    """fp64 gradients of L = sum(dout * out) with respect to q, k, v (the
    calculus of the attention definition; see attn_fp64.c).

    q, dout [B,Sq,Hq,D], k/v [B,Skv,Hkv,D] (read as float32).  Returns
    (dq [B,Sq,Hq,D], dk [B,Skv,Hkv,D], dv [B,Skv,Hkv,D]) float64.

    The pages give no backward: this is the calculus of the definition of
    "Lesson 8", section 1 (attn_fp64.c).
    """
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, Sq, Hq, D = q.shape
    Bk, Skv, Hkv, Dk = k.shape
    assert Bk == B and Dk == D and v.shape == k.shape and dout.shape == q.shape and Hq % Hkv == 0
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(k.shape, dtype=np.float64)
    keep = []

    def ptr(a):
        if a is None:
            return None
        a = np.ascontiguousarray(np.asarray(a, dtype=np.int64))
        keep.append(a)
        return a.ctypes.data

    rc = _load().oracle_attn_bwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, B, Sq, Skv, Hq,
                                 Hkv, D, ptr(qpos), ptr(kpos), int(bool(causal)), float(scale), dq.ctypes.data,
                                 dk.ctypes.data, dv.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd failed with code {rc}")
    return dq, dk, dv


def attention_bwd_dq_rows(q, k, v, dout, rows, *, scale: float, causal: bool, threads: int = 0):
    """fp64 dq of the requested query rows (b, h, i) only: each row needs just
    its own scores, so large problems can be sampled.  Returns [n, D] float64.

    The pages give no backward: the calculus of "Lesson 8", section 1, one
    query row at a time (attn_fp64.c).
    """
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, S, Hq, D = q.shape
    _, Sk, Hkv, _ = k.shape
    assert Sk == S and v.shape == k.shape and dout.shape == q.shape and Hq % Hkv == 0
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    dq = np.zeros((rows.shape[0], D), dtype=np.float64)
    rc = _load().oracle_attn_bwd_dq_rows(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, B, S, Hq,
                                         Hkv, D, int(bool(causal)), float(scale), rows.ctypes.data, rows.shape[0],
                                         dq.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd_dq_rows failed with code {rc}")
    return dq


def all_rows(B: int, H: int, S: int) -> np.ndarray:
    """Every (b, h, i) triple, in (b, h, i) order.

    Plumbing; no passage.
    """
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(S), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1).astype(np.int32)


def attention_full(q, k, v, *, scale: float, causal: bool, qpos=None, kpos=None,
                   kv_len=None, threads: int = 0):
    """fp64 attention for every query row.
    Returns out [B,Sq,Hq,D] and lse [B,Hq,Sq] (float64).

    As attention_rows ("Lesson 8", sections 1 and 4), for every row.
    """
    B, Sq, Hq, D = np.asarray(q).shape
    rows = all_rows(B, Hq, Sq)
    out, lse = attention_rows(q, k, v, rows, scale=scale, causal=causal, qpos=qpos,
                              kpos=kpos, kv_len=kv_len, threads=threads)
    out = out.reshape(B, Hq, Sq, D).transpose(0, 2, 1, 3).copy()
    lse = lse.reshape(B, Hq, Sq)
    return out, lse


from . import brute, merge, schedule, streaming  # noqa: E402,F401
