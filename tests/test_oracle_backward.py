"""Pins for the fp64 backward of the oracle (oracle.attention_bwd).

The pages give no backward; the oracle writes out the calculus of the
attention definition.  It is pinned to things outside itself:
  * central finite differences of the forward, L = sum(dout * out), computed
    with the independent numpy oracle (oracle/brute.py) in float64;
  * a library routine: torch autograd through scaled_dot_product_attention in
    float64;
  * closed forms and invariants: identical keys give dq = 0 and dv the
    prefix-averaged dout; constant values give dq = dk = 0; shifting every key
    by one vector leaves the output unchanged, so the dk of each head group
    sums to zero; the softmax weights of a row sum to one, so the dv sum to
    the dout sum.
A wrong sign, a dropped delta term, a transposed operand or a missing GQA
sum fails at least one of these.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.brute import brute


def _inputs(B, S, Hq, Hkv, D, seed):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return f(B, S, Hq, D), f(B, S, Hkv, D), f(B, S, Hkv, D), f(B, S, Hq, D)


def _loss(q, k, v, dout, scale, causal):
    out, _ = brute(q, k, v, scale=scale, causal=causal)
    return float(np.sum(out * np.asarray(dout, dtype=np.float64)))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,S,Hq,Hkv,D", [(1, 5, 2, 1, 3), (2, 4, 2, 2, 4)])
def test_central_finite_differences(causal, B, S, Hq, Hkv, D):
    q, k, v, dout = _inputs(B, S, Hq, Hkv, D, 11 + S)
    scale = 0.7
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, scale=scale, causal=causal)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        x64 = x.astype(np.float64)
        for idx in np.ndindex(x.shape):
            xp, xm = x64.copy(), x64.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = dict(q=q, k=k, v=v)
            args_m = dict(q=q, k=k, v=v)
            args_p[name], args_m[name] = xp, xm
            fd = (_loss(args_p["q"], args_p["k"], args_p["v"], dout, scale, causal) -
                  _loss(args_m["q"], args_m["k"], args_m["v"], dout, scale, causal)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * (1 + abs(fd)), (name, idx, fd, g[idx])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,S,Hq,Hkv,D", [(1, 33, 4, 2, 16), (2, 20, 3, 1, 8), (1, 64, 2, 2, 32)])
def test_matches_torch_autograd_float64(causal, B, S, Hq, Hkv, D):
    q, k, v, dout = _inputs(B, S, Hq, Hkv, D, 7)
    scale = 1.0 / np.sqrt(D)
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, scale=scale, causal=causal)
    G = Hq // Hkv
    tq = torch.tensor(q, dtype=torch.float64).transpose(1, 2).requires_grad_()
    tk = torch.tensor(k, dtype=torch.float64).transpose(1, 2).requires_grad_()
    tv = torch.tensor(v, dtype=torch.float64).transpose(1, 2).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1),
                                                         is_causal=causal, scale=scale)
    o.backward(torch.tensor(dout, dtype=torch.float64).transpose(1, 2))
    np.testing.assert_allclose(dq, tq.grad.transpose(1, 2).numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dk, tk.grad.transpose(1, 2).numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dv, tv.grad.transpose(1, 2).numpy(), atol=1e-10, rtol=0)


def test_identical_keys_closed_form():
    # every score of a row is equal, so the softmax weights are uniform, p_ij = 1/(i+1) over
    # j <= i, and the softmax derivative reduces to centring:
    #   dv_j = sum_{i >= j} dout_i / (i+1)
    #   ds_ij = (dout_i.v_j - mean_{j' <= i} dout_i.v_j') / (i+1), which sums to zero over j,
    #   so dq_i = scale * k * sum_j ds_ij = 0 and dk_j = scale * sum_{i >= j} ds_ij q_i
    B, S, H, D = 1, 9, 2, 5
    scale = 0.4
    rng = np.random.default_rng(3)
    q = rng.standard_normal((B, S, H, D)).astype(np.float32)
    k = np.tile(rng.standard_normal((1, 1, H, D)).astype(np.float32), (B, S, 1, 1))
    v = rng.standard_normal((B, S, H, D)).astype(np.float32)
    dout = rng.standard_normal((B, S, H, D)).astype(np.float32)
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, scale=scale, causal=True)
    assert np.max(np.abs(dq)) < 1e-12
    q64, v64, o64 = (x.astype(np.float64) for x in (q, v, dout))
    e_dv = np.zeros((B, S, H, D))
    e_dk = np.zeros((B, S, H, D))
    for h in range(H):
        for i in range(S):
            dp = np.array([o64[0, i, h] @ v64[0, j, h] for j in range(i + 1)])
            ds = (dp - dp.mean()) / (i + 1)
            for j in range(i + 1):
                e_dv[0, j, h] += o64[0, i, h] / (i + 1)
                e_dk[0, j, h] += scale * ds[j] * q64[0, i, h]
    np.testing.assert_allclose(dv, e_dv, atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, e_dk, atol=1e-12, rtol=0)


def test_constant_values_give_no_q_or_k_gradient():
    q, k, _, dout = _inputs(1, 12, 4, 2, 6, 5)
    v = np.tile(np.arange(6, dtype=np.float32)[None, None, None, :], (1, 12, 2, 1))
    dq, dk, _ = oracle.attention_bwd(q, k, v, dout, scale=0.3, causal=True)
    assert np.max(np.abs(dq)) < 1e-12 and np.max(np.abs(dk)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance_and_value_weights(causal):
    # out is unchanged when every key moves by the same vector: sum_j dk_j = 0 per (b, kv head);
    # each row's weights sum to one: sum_j dv_j = sum over the group's rows of dout
    B, S, Hq, Hkv, D = 2, 40, 4, 2, 8
    q, k, v, dout = _inputs(B, S, Hq, Hkv, D, 9)
    dq, dk, dv = oracle.attention_bwd(q, k, v, dout, scale=0.35, causal=causal)
    assert np.max(np.abs(dk.sum(axis=1))) < 1e-10
    G = Hq // Hkv
    dsum = dout.astype(np.float64).reshape(B, S, Hkv, G, D).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), dsum, atol=1e-10, rtol=0)


def test_positions_select_the_same_keys_as_the_causal_rule():
    # explicit positions equal to the row indices reproduce the causal result; a shard with
    # later positions (a ring step) equals the matching slice of the whole problem's dq
    q, k, v, dout = _inputs(1, 16, 2, 1, 4, 13)
    a = oracle.attention_bwd(q, k, v, dout, scale=0.5, causal=True)
    b = oracle.attention_bwd(q, k, v, dout, scale=0.5, causal=True, qpos=np.arange(16), kpos=np.arange(16))
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    dq_part, _, _ = oracle.attention_bwd(q[:, 8:], k, v, dout[:, 8:], scale=0.5, causal=True,
                                         qpos=np.arange(8, 16))
    np.testing.assert_allclose(dq_part, a[0][:, 8:], atol=1e-13, rtol=0)



def test_keys_moved_with_their_positions_give_the_same_gradients():
    # the causal rule reads a key's position, not its row: permuting the key/value rows together
    # with their positions leaves dq unchanged and permutes dk, dv the same way
    q, k, v, dout = _inputs(1, 24, 4, 2, 8, 19)
    perm = np.random.default_rng(20).permutation(24)
    a = oracle.attention_bwd(q, k, v, dout, scale=0.5, causal=True)
    b = oracle.attention_bwd(q, k[:, perm], v[:, perm], dout, scale=0.5, causal=True, kpos=perm)
    np.testing.assert_allclose(b[0], a[0], atol=1e-13, rtol=0)
    np.testing.assert_allclose(b[1], a[1][:, perm], atol=1e-13, rtol=0)
    np.testing.assert_allclose(b[2], a[2][:, perm], atol=1e-13, rtol=0)

@pytest.mark.parametrize("causal", [False, True])
def test_sampled_dq_rows_equal_the_full_backward(causal):
    # the row-at-a-time dq (for large problems) against the full backward pinned above
    q, k, v, dout = _inputs(2, 50, 4, 2, 16, 17)
    dq, _, _ = oracle.attention_bwd(q, k, v, dout, scale=0.3, causal=causal)
    rows = oracle.all_rows(2, 4, 50)
    got = oracle.attention_bwd_dq_rows(q, k, v, dout, rows, scale=0.3, causal=causal)
    ref = dq.transpose(0, 2, 1, 3).reshape(-1, 16)
    np.testing.assert_allclose(got, ref, atol=1e-12, rtol=0)
