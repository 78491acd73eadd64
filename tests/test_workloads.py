"""The seeded input recipe (workloads/) does what its description says: the
same seed gives the same tensors; the x8 workload scales exactly
floor(0.01 S) distinct key rows per (batch, kv head) and nothing else; the
sampled rows include the first and last row of every chunk; decode lengths
fall in [capacity/2, capacity]; the FLOP convention is 4 B Hq S^2 D, halved
when causal."""
import math

import numpy as np
import torch

import workloads as W


def test_same_seed_same_tensors_other_seed_others():
    cfg = W.Prefill("t", "bf16", True, "zigzag", 1, 4, 2, 512, 64, 2, 11)
    a = W.prefill_inputs(cfg)
    b = W.prefill_inputs(cfg)
    c = W.prefill_inputs(W.Prefill("t", "bf16", True, "zigzag", 1, 4, 2, 512, 64, 2, 12))
    for x, y, z in zip(a, b, c):
        assert x.dtype == torch.bfloat16
        assert torch.equal(x, y) and not torch.equal(x, z)


def test_keys_x8_scales_one_percent_of_key_rows_per_kv_head():
    # an N(0,1) row of D = 128 has norm about sqrt(128) = 11.3; times 8 about 90: a norm above 40
    # tells the scaled rows apart
    cfg = W.Prefill("t", "bf16", True, "zigzag", 2, 4, 2, 4096, 128, 4, 13, keys_x8=True)
    q, k, v = W.prefill_inputs(cfg)
    n_big = math.floor(0.01 * cfg.S)
    kn = k.float().norm(dim=-1)                                 # [B, S, Hkv]
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            assert int((kn[b, :, g] > 40).sum()) == n_big
    assert float(v.float().norm(dim=-1).max()) < 40 and float(q.float().norm(dim=-1).max()) < 40
    # the rows differ between (b, g) pairs: a fresh permutation for each
    rows = [set(torch.nonzero(kn[b, :, g] > 40).flatten().tolist()) for b in range(cfg.B) for g in range(cfg.Hkv)]
    assert len({frozenset(r) for r in rows}) == len(rows)


def test_sampled_rows_hold_every_chunk_edge():
    cfg = W.CFG4
    rows = W.sample_rows(cfg, 256)
    assert rows.shape == (cfg.B * cfg.Hq * 256, 3)
    per_head = rows[(rows[:, 0] == 0) & (rows[:, 1] == 5)][:, 2]
    assert len(per_head) == 256 and len(set(per_head.tolist())) == 256
    for c in range(cfg.n_chunks):
        assert c * cfg.chunk in per_head and (c + 1) * cfg.chunk - 1 in per_head
    assert per_head.min() == 0 and per_head.max() == cfg.S - 1
    striped = W.Prefill("s", "bf16", True, "striped", 1, 2, 2, 4096, 128, 16, 3)
    srows = W.sample_rows(striped, 64)[:, 2]
    for t in list(range(16)) + list(range(4096 - 16, 4096)):
        assert t in srows
    full = W.sample_rows(W.CFG1, 0)
    assert len(full) == W.CFG1.B * W.CFG1.Hq * W.CFG1.S


def test_decode_lengths_in_range_and_seeded():
    cfg = W.CFG5
    a, b = W.decode_lengths(cfg), W.decode_lengths(cfg)
    assert torch.equal(a, b) and a.dtype == torch.int32 and a.shape == (cfg.B,)
    assert int(a.min()) >= cfg.capacity // 2 and int(a.max()) <= cfg.capacity
    fixed = W.Decode("f", 3, 8, 2, 64, 1024, 4, 1, fixed_lens=(1024, 7, 0))
    assert W.decode_lengths(fixed).tolist() == [1024, 7, 0]


def test_flop_convention():
    assert W.CFG4.flops() == 4 * 32 * 131072 ** 2 * 128 / 2
    assert abs(W.CFG4.flops() / 1e12 - 140.7) < 0.05
    assert W.CFG1.flops() == 4 * 2 * 256 ** 2 * 64          # non-causal: every pair
    assert np.isclose(W.CFG3.flops(), 4 * 2 * 16 * 32768 ** 2 * 128 / 2)
