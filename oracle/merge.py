"""Direct formula for combining partial attention results, in fp64.

TEST INFRASTRUCTURE (see the package docstring).

When the keys of one query are split into disjoint parts p (the KV cache
sharded along the sequence: "NVIDIA unveils Helix Parallelism", Phase 1,
KV parallelism), each part yields a normalised partial output O_p and its
log-sum-exp lse_p = m_p + ln l_p.  Attention over the union of the parts is

    lse = ln sum_p exp(lse_p)
    out = sum_p exp(lse_p - lse) * O_p ,

which is what the online-softmax update of "Lesson 8: Context Parallelism",
section 3, gives when whole partial states are folded one after another.
Parts with no key (lse_p = -inf) contribute nothing; if every part is empty,
out = 0 and lse = -inf.
"""
from __future__ import annotations

import numpy as np


def merge(partials, part_lse):
    """partials [..., P, D], part_lse [..., P] -> (out [..., D], lse [...]).

    The update of "Lesson 8: Context Parallelism", section 3, applied to
    whole partial states (the merge of "NVIDIA unveils Helix Parallelism",
    Phase 1).
    """
    O = np.asarray(partials, dtype=np.float64)
    L = np.asarray(part_lse, dtype=np.float64)
    m = L.max(axis=-1, keepdims=True)
    live = np.isfinite(m)
    m_safe = np.where(live, m, 0.0)
    w = np.exp(L - m_safe)                       # exp(-inf) = 0 for empty parts
    z = w.sum(axis=-1, keepdims=True)
    z_safe = np.where(z > 0, z, 1.0)
    out = (w[..., None] * O).sum(axis=-2) / z_safe
    lse = np.where(live[..., 0], m[..., 0] + np.log(z_safe[..., 0]), -np.inf)
    out = np.where(live, out, 0.0)
    return out, lse
