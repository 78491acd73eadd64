"""The online-softmax recurrence of the ring loop, in fp64.

TEST INFRASTRUCTURE (see the package docstring).  Used only to pin that the
blockwise recurrence reaches the plain definition computed by attn_fp64.c
(after a full loop the result is exact attention: "Sequence parallelism and
ring attention", FAQ; "Lesson 8: Context Parallelism", section 3).

The update follows "Lesson 8", section 3, in its notation: when a new K/V
block arrives with scores S_new,
    m~     = max(m, max S_new)
    l'     = l * exp(m - m~) + sum exp(S_new - m~)
    O'     = O * exp(m - m~) * l / l' + exp(S_new - m~) V_new / l'
and m takes the value m~ (the section defines m~ but leaves the assignment
implicit; it is the only consistent reading).  The state starts at
m = -inf, l = 0, O = 0; a block in which a row has no allowed key leaves that
row's state unchanged.
"""
from __future__ import annotations

import numpy as np


def init_state(n_rows: int, D: int):
    """The starting state of "Lesson 8", section 3: m = -inf, l = 0, O = 0.
    """
    return (np.full(n_rows, -np.inf), np.zeros(n_rows), np.zeros((n_rows, D)))


def update(state, s_new: np.ndarray, v_new: np.ndarray):
    """One ring step for a set of query rows.

    s_new [n, Lk] scaled scores of the new block (-inf where masked),
    v_new [Lk, D] its value rows.  Returns the new (m, l, O) with O normalised.

    The update of "Lesson 8", section 3.
    """
    m, l, O = state
    blk_max = s_new.max(axis=1) if s_new.shape[1] else np.full(s_new.shape[0], -np.inf)
    m_t = np.maximum(m, blk_max)
    live = np.isfinite(m_t)
    m_safe = np.where(live, m_t, 0.0)
    alpha = np.where(np.isfinite(m), np.exp(m - m_safe), 0.0)
    p = np.exp(s_new - m_safe[:, None])               # exp(-inf) = 0 on masked entries
    l_new = l * alpha + p.sum(axis=1)
    l_div = np.where(l_new > 0, l_new, 1.0)
    O_new = O * (alpha * l / l_div)[:, None] + (p @ v_new) / l_div[:, None]
    m_out = np.where(live, m_t, m)
    l_out = np.where(live, l_new, l)
    O_out = np.where(live[:, None], O_new, O)
    return m_out, l_out, O_out


def ring_attention_rows(q, k, v, *, scale: float, causal: bool, chunks_in_order, chunk_len: int,
                        q_rows, qpos, h: int, b: int = 0):
    """Run the recurrence for query rows ``q_rows`` (positions ``qpos``) of head
    h over the K/V chunks given in visiting order.  q [B,S,Hq,D], k/v
    [B,S,Hkv,D].  Returns (out, lse, m, l) per row.

    The ring loop of "Lesson 8", sections 2 and 3.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    G = q.shape[2] // k.shape[2]
    g = h // G
    qq = q[b, q_rows, h, :]
    qpos = np.asarray(qpos)
    st = init_state(len(q_rows), q.shape[3])
    for c in chunks_in_order:
        ks = np.arange(c * chunk_len, (c + 1) * chunk_len)
        s = (qq @ k[b, ks, g, :].T) * scale
        if causal:
            s = np.where(ks[None, :] <= qpos[:, None], s, -np.inf)
        st = update(st, s, v[b, ks, g, :])
    m, l, O = st
    lse = m + np.log(l)
    return O, lse, m, l
