"""Second oracle: numpy fp64 attention over the whole S x S score matrix.

TEST INFRASTRUCTURE (see the package docstring).  Written independently of
attn_fp64.c so the two can pin each other: this one builds the full score
tensor with einsum, masks it, and uses the max-shifted softmax along the key
axis -- the formula of "Lesson 8: Context Parallelism", section 1, with the
causal rule of section 4 (query i sees keys j <= i).  Tiny shapes only.
"""
from __future__ import annotations

import numpy as np


def brute(q, k, v, *, scale: float, causal: bool, qpos=None, kpos=None, kv_len=None):
    """Returns (out [B,Sq,Hq,D], lse [B,Hq,Sq]) in float64.

    Follows "Lesson 8: Context Parallelism", section 1, with the causal rule of
    section 4.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Sq, Hq, D = q.shape
    _, Skv, Hkv, _ = k.shape
    G = Hq // Hkv
    # expand K/V heads so query head h reads KV head h // G
    kh = np.repeat(k, G, axis=2)                      # [B,Skv,Hq,D]
    vh = np.repeat(v, G, axis=2)
    s = np.einsum("bihd,bjhd->bhij", q, kh) * scale   # [B,Hq,Sq,Skv]
    allowed = np.ones((B, 1, Sq, Skv), dtype=bool)
    qp = np.arange(Sq) if qpos is None else np.asarray(qpos)
    kp = np.arange(Skv) if kpos is None else np.asarray(kpos)
    if causal:
        allowed &= (kp[None, :] <= qp[:, None])[None, None]
    if kv_len is not None:
        kl = np.asarray(kv_len)
        allowed &= (np.arange(Skv)[None, :] < kl[:, None])[:, None, None, :]
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    any_key = np.isfinite(m)
    m_safe = np.where(any_key, m, 0.0)
    p = np.exp(s - m_safe)                            # masked entries -> 0
    z = p.sum(axis=-1, keepdims=True)
    z_safe = np.where(z > 0, z, 1.0)
    out = np.einsum("bhij,bjhd->bihd", p / z_safe, vh)
    lse = np.where(any_key[..., 0], m[..., 0] + np.log(z_safe[..., 0]), -np.inf)
    return out, lse
