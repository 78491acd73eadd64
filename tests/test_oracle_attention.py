"""Pins for the fp64 attention oracle (oracle/attn_fp64.c) and its
independent twin (oracle/brute.py), the recurrence (oracle/streaming.py) and
the partial-merge formula (oracle/merge.py).

Pins used, none of which re-types the oracle's own formula:
  * closed forms: identical keys give the mean of the allowed value rows and
    lse = s + ln|J|; constant value rows give that constant; one dominant
    score selects its value row within (|J|-1) e^-gap;
  * a library routine: torch's scaled_dot_product_attention in float64;
  * brute force: the numpy full-matrix oracle, written separately;
  * invariants: key permutation (non-causal), split / rotation independence of
    the ring recurrence (exact after a full loop: "Sequence parallelism and
    ring attention", FAQ; "Lesson 8: Context Parallelism", section 3).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute, merge, schedule, streaming


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def test_identical_keys_give_prefix_mean():
    B, S, H, D = 1, 37, 2, 16
    q = rnd((B, S, H, D), 1)
    k = np.broadcast_to(rnd((1, 1, H, D), 2), (B, S, H, D)).copy()
    v = rnd((B, S, H, D), 3)
    out, lse = oracle.attention_full(q, k, v, scale=0.3, causal=True)
    for h in range(H):
        for i in range(S):
            np.testing.assert_allclose(out[0, i, h], v[0, : i + 1, h].astype(np.float64).mean(0), atol=1e-12)
            s = 0.3 * float(np.dot(q[0, i, h].astype(np.float64), k[0, 0, h].astype(np.float64)))
            assert abs(lse[0, h, i] - (s + math.log(i + 1))) < 1e-12
    out_nc, lse_nc = oracle.attention_full(q, k, v, scale=0.3, causal=False)
    np.testing.assert_allclose(out_nc[0, 5], v[0].astype(np.float64).mean(0), atol=1e-12)


def test_zero_query_gives_mean_noncausal():
    B, S, H, D = 2, 20, 3, 8
    q = np.zeros((B, S, H, D), np.float32)
    k, v = rnd((B, S, H, D), 4), rnd((B, S, H, D), 5)
    out, lse = oracle.attention_full(q, k, v, scale=1.0, causal=False)
    np.testing.assert_allclose(out, np.broadcast_to(v.astype(np.float64).mean(1, keepdims=True), out.shape), atol=1e-12)
    np.testing.assert_allclose(lse, math.log(S), atol=1e-12)


def test_constant_values():
    B, S, H, D = 1, 29, 2, 8
    q, k = rnd((B, S, H, D), 6), rnd((B, S, H, D), 7)
    c = rnd((D,), 8)
    v = np.broadcast_to(c, (B, S, H, D)).copy()
    for causal in (False, True):
        out, _ = oracle.attention_full(q, k, v, scale=0.7, causal=causal)
        np.testing.assert_allclose(out, np.broadcast_to(c.astype(np.float64), out.shape), atol=1e-12)


def test_dominant_score_selects_row():
    B, S, H, D = 1, 16, 1, 8
    q = rnd((B, S, H, D), 9)
    k = rnd((B, S, H, D), 10) * 0.01
    v = rnd((B, S, H, D), 11)
    i, j, lam = 12, 5, 40.0
    k[0, j, 0] = lam * q[0, i, 0]
    out, _ = oracle.attention_rows(q, k, v, [(0, 0, i)], scale=1.0, causal=True)
    s = (q[0, i, 0].astype(np.float64) @ k[0, : i + 1, 0].astype(np.float64).T)
    gap = s[j] - np.max(np.delete(s, j))
    bound = i * math.exp(-gap) * 2 * np.abs(v).max()
    assert gap > 30
    assert np.max(np.abs(out[0] - v[0, j, 0])) <= bound + 1e-15


def test_single_key_is_that_value():
    q, k, v = rnd((1, 4, 1, 8), 12), rnd((1, 4, 1, 8), 13), rnd((1, 4, 1, 8), 14)
    out, lse = oracle.attention_rows(q, k, v, [(0, 0, 0)], scale=0.5, causal=True)
    np.testing.assert_allclose(out[0], v[0, 0, 0], atol=1e-15)
    assert abs(lse[0] - 0.5 * float(q[0, 0, 0].astype(np.float64) @ k[0, 0, 0].astype(np.float64))) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,S,Hq,Hkv,D", [(1, 64, 2, 2, 16), (2, 97, 4, 2, 32), (1, 130, 8, 2, 64)])
def test_matches_torch_sdpa_float64(causal, B, S, Hq, Hkv, D):
    q, k, v = rnd((B, S, Hq, D), 20), rnd((B, S, Hkv, D), 21), rnd((B, S, Hkv, D), 22)
    scale = 1 / math.sqrt(D)
    out, _ = oracle.attention_full(q, k, v, scale=scale, causal=causal)
    G = Hq // Hkv
    tq = torch.from_numpy(q).double().permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    tv = torch.from_numpy(v).double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_c_oracle_matches_numpy_brute(causal):
    B, S, Hq, Hkv, D = 2, 77, 6, 3, 24
    q, k, v = rnd((B, S, Hq, D), 30), rnd((B, S, Hkv, D), 31), rnd((B, S, Hkv, D), 32)
    a_out, a_lse = oracle.attention_full(q, k, v, scale=0.2, causal=causal)
    b_out, b_lse = brute.brute(q, k, v, scale=0.2, causal=causal)
    np.testing.assert_allclose(a_out, b_out, atol=1e-12, rtol=0)
    np.testing.assert_allclose(a_lse, b_lse, atol=1e-12, rtol=0)


def test_c_oracle_matches_brute_with_positions_and_lengths():
    B, Sq, Skv, Hq, Hkv, D = 3, 10, 50, 4, 1, 16
    q, k, v = rnd((B, Sq, Hq, D), 33), rnd((B, Skv, Hkv, D), 34), rnd((B, Skv, Hkv, D), 35)
    qpos = np.array([3, 7, 11, 19, 23, 29, 31, 37, 41, 49])
    kpos = np.arange(Skv)[::-1].copy()
    kv_len = np.array([50, 17, 1])
    a = oracle.attention_full(q, k, v, scale=0.4, causal=True, qpos=qpos, kpos=kpos, kv_len=kv_len)
    b = brute.brute(q, k, v, scale=0.4, causal=True, qpos=qpos, kpos=kpos, kv_len=kv_len)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)


def test_empty_key_set():
    q, k, v = rnd((1, 2, 1, 4), 36), rnd((1, 3, 1, 4), 37), rnd((1, 3, 1, 4), 38)
    out, lse = oracle.attention_rows(q, k, v, [(0, 0, 0)], scale=1.0, causal=False, kv_len=[0])
    assert np.all(out == 0) and lse[0] == -np.inf


def test_key_permutation_invariance_noncausal():
    B, S, H, D = 1, 45, 2, 16
    q, k, v = rnd((B, S, H, D), 40), rnd((B, S, H, D), 41), rnd((B, S, H, D), 42)
    perm = np.random.default_rng(43).permutation(S)
    a = oracle.attention_full(q, k, v, scale=0.25, causal=False)
    b = oracle.attention_full(q, k[:, perm], v[:, perm], scale=0.25, causal=False)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_ring_recurrence_equals_oracle(layout, causal, P):
    # the section-3 recurrence over the ring's visiting order reaches the definition
    S, Hq, Hkv, D = 256, 2, 1, 16
    q, k, v = rnd((1, S, Hq, D), 50), rnd((1, S, Hkv, D), 51), rnd((1, S, Hkv, D), 52)
    ref_out, ref_lse = oracle.attention_full(q, k, v, scale=0.25, causal=causal)
    C = schedule.chunk_len(S, P, layout)
    own = schedule.layout_assignment(P, layout)
    for r in range(P):
        rows = np.concatenate([np.arange(c * C, (c + 1) * C) for c in own[r]])
        order = schedule.kv_visit_order(P, layout, r)
        if causal:
            order = order  # masked pairs contribute nothing; they are kept to exercise the -inf path
        for h in range(Hq):
            O, lse, m, l = streaming.ring_attention_rows(q, k, v, scale=0.25, causal=causal, chunks_in_order=order,
                                                         chunk_len=C, q_rows=rows, qpos=rows, h=h)
            np.testing.assert_allclose(O, ref_out[0, rows, h], atol=1e-12)
            np.testing.assert_allclose(lse, ref_lse[0, h, rows], atol=1e-12)


def test_ring_recurrence_any_rotation_order():
    S, H, D, P = 96, 1, 8, 6
    q, k, v = rnd((1, S, H, D), 60), rnd((1, S, H, D), 61), rnd((1, S, H, D), 62)
    ref_out, ref_lse = oracle.attention_full(q, k, v, scale=0.3, causal=True)
    rows = np.arange(S)
    for order in itertools.islice(itertools.permutations(range(P)), 0, 720, 37):
        O, lse, _, _ = streaming.ring_attention_rows(q, k, v, scale=0.3, causal=True, chunks_in_order=order,
                                                     chunk_len=S // P, q_rows=rows, qpos=rows, h=0)
        np.testing.assert_allclose(O, ref_out[0, :, 0], atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse[0, 0], atol=1e-12)


def test_merge_of_part_results_equals_whole():
    # Helix phase 1: keys sharded along the sequence; merging the per-shard
    # results must give attention over all keys
    B, Skv, Hq, Hkv, D, P = 2, 120, 4, 2, 16, 5
    q, k, v = rnd((B, 1, Hq, D), 70), rnd((B, Skv, Hkv, D), 71), rnd((B, Skv, Hkv, D), 72)
    lens = np.array([120, 37])
    whole_out, whole_lse = oracle.attention_full(q, k, v, scale=0.3, causal=False, kv_len=lens)
    C = Skv // P
    parts = np.zeros((B, Hq, P, D))
    plse = np.full((B, Hq, P), -np.inf)
    for p in range(P):
        sl = slice(p * C, (p + 1) * C)
        lp = np.clip(lens - p * C, 0, C)
        o, l = oracle.attention_full(q, k[:, sl], v[:, sl], scale=0.3, causal=False, kv_len=lp)
        parts[:, :, p] = o[:, 0]
        plse[:, :, p] = l[:, :, 0]
    out, lse = merge.merge(parts, plse)
    assert np.isneginf(plse[1, :, 2:]).all()       # empty shards of the short sequence
    np.testing.assert_allclose(out, whole_out[:, 0], atol=1e-12)
    np.testing.assert_allclose(lse, whole_lse[:, :, 0], atol=1e-12)


def test_merge_all_empty():
    out, lse = merge.merge(np.ones((3, 4, 8)), np.full((3, 4), -np.inf))
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_streaming_state_matches_definition_after_each_step():
    # after t steps the state (m, l, O) is attention over the keys seen so far:
    # m is their max score, l = sum exp(s - m), O normalised
    S, D, P = 64, 8, 4
    q, k, v = rnd((1, S, 1, D), 80), rnd((1, S, 1, D), 81), rnd((1, S, 1, D), 82)
    rows = np.arange(S)
    C = S // P
    st = streaming.init_state(S, D)
    seen = []
    for c in (2, 0, 3, 1):
        ks = np.arange(c * C, (c + 1) * C)
        s = q[0, :, 0].astype(np.float64) @ k[0, ks, 0].astype(np.float64).T * 0.5
        st = streaming.update(st, s, v[0, ks, 0].astype(np.float64))
        seen.extend(ks)
        sk = np.array(sorted(seen))
        out, lse = oracle.attention_rows(q, k[:, sk], v[:, sk], [(0, 0, i) for i in rows], scale=0.5, causal=False)
        full_s = q[0, :, 0].astype(np.float64) @ k[0, sk, 0].astype(np.float64).T * 0.5
        np.testing.assert_allclose(st[0], full_s.max(1), atol=1e-13)
        np.testing.assert_allclose(st[0] + np.log(st[1]), lse, atol=1e-12)
        np.testing.assert_allclose(st[2], out, atol=1e-12)
