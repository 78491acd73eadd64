"""Seeded synthetic inputs shared by the tests, the oracle checks and bench.py.

This module holds only shapes, seeds and random-number recipes: none of the
attention arithmetic.  Both the CUDA path and the oracle receive the tensors
made here (the oracle gets host copies of the very same values).

Recipe (every workload):
  * Q, K, V i.i.d. N(0, 1), drawn in float32 from ``torch.Generator`` seeded
    with the workload's seed on the device the tensors live on, then rounded
    to bfloat16 (round-to-nearest-even) for the bf16 workloads.
  * ``keys_x8`` workload: in every (batch, kv head), exactly floor(0.01 * S)
    distinct key rows, picked by a seeded permutation, are multiplied by 8 in
    float32 before the bf16 rounding; V is untouched.
  * decode: per-sequence valid lengths drawn uniformly from the integers in
    [capacity/2, capacity] with a CPU generator of the workload's seed.
  * scale = 1/sqrt(D).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Prefill:
    name: str
    dtype: str            # "fp32" | "bf16"
    causal: bool
    layout: str           # "contiguous" | "zigzag" | "striped", optionally + chunks per rank ("zigzag4")
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    P: int
    seed: int
    keys_x8: bool = False
    sample_rows: int = 0  # 0 = check every row against the oracle

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def n_chunks(self) -> int:
        """Chunks of the split (stripes for the striped split)."""
        name = self.layout.rstrip("0123456789")
        per_rank = int(self.layout[len(name):] or (2 if name == "zigzag" else 1))
        return self.P * per_rank

    @property
    def chunk(self) -> int:
        return self.S // self.n_chunks

    def flops(self) -> float:
        """Causal-adjusted attention FLOPs: 4*B*Hq*S^2*D, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.S * self.S * self.D
        return f / 2 if self.causal else f


@dataclass(frozen=True)
class Decode:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    capacity: int
    P: int
    seed: int
    min_len: int = 0      # lengths ~ U[min_len, capacity]; 0 means capacity // 2
    fixed_lens: tuple = field(default=())

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def chunk(self) -> int:
        return self.capacity // self.P


@dataclass(frozen=True)
class Merge:
    """The (O, lse) merge alone: B*Hq rows of P normalised partials of D dims."""
    name: str
    B: int
    Hq: int
    P: int
    D: int
    seed: int
    empty_frac: float = 0.0   # share of parts with lse = -inf (their O is filled with NaN)


# The five workloads of the hot path.
CFG1 = Prefill("ring_fp32_noncausal_B1_H2_S256_D64_P4", "fp32", False, "contiguous", 1, 2, 2, 256, 64, 4, 1)
CFG2 = Prefill("ring_bf16_causal_contiguous_B1_H8_S8192_D128_P8", "bf16", True, "contiguous", 1, 8, 8, 8192, 128, 8, 2)
CFG3 = Prefill("ring_bf16_causal_zigzag_B2_H16_S32768_D128_P8_keysx8", "bf16", True, "zigzag", 2, 16, 16, 32768, 128, 8, 3,
               keys_x8=True, sample_rows=256)
CFG4 = Prefill("ring_bf16_causal_zigzag_gqa_B1_Hq32_Hkv8_S131072_D128_P16", "bf16", True, "zigzag", 1, 32, 8, 131072, 128, 16, 4,
               sample_rows=256)
CFG5 = Decode("decode_splitkv_bf16_B8_Hq32_Hkv8_D128_ctx1M_P32", 8, 32, 8, 128, 1 << 20, 32, 5)
CONFIGS = {c.name: c for c in (CFG1, CFG2, CFG3, CFG4, CFG5)}
# The merge of workload 5's partials on its own, at a size that is HBM-bound
# (134 MB of partials, above the 126 MB L2): B*Hq = 8192 rows, P = 32, D = 128.
MERGE_ONLY = Merge("merge_fp32parts_bf16out_BHq8192_P32_D128", 256, 32, 32, 128, 6)


def _dtype(name: str):
    return torch.float32 if name == "fp32" else torch.bfloat16


def randn(shape, gen: torch.Generator, device, dtype) -> torch.Tensor:
    """N(0,1) float32 draws rounded to ``dtype``."""
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x.to(dtype)


def prefill_inputs(cfg: Prefill, device="cpu"):
    """q [B,S,Hq,D], k, v [B,S,Hkv,D] on ``device`` for a prefill workload."""
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed)
    dt = _dtype(cfg.dtype)
    q = randn((cfg.B, cfg.S, cfg.Hq, cfg.D), gen, device, dt)
    kf = torch.randn((cfg.B, cfg.S, cfg.Hkv, cfg.D), generator=gen, device=device, dtype=torch.float32)
    if cfg.keys_x8:
        n_big = int(math.floor(0.01 * cfg.S))
        for b in range(cfg.B):
            for g in range(cfg.Hkv):
                rows = torch.randperm(cfg.S, generator=gen, device=device)[:n_big]
                kf[b, rows, g, :] *= 8.0
    k = kf.to(dt)
    del kf
    v = randn((cfg.B, cfg.S, cfg.Hkv, cfg.D), gen, device, dt)
    return q, k, v


def sample_rows(cfg: Prefill, n: int | None = None, seed_offset: int = 1000) -> np.ndarray:
    """Query rows checked against the oracle at large S: for every (b, hq),
    rows 0 and S-1, the first and last row of every chunk (stripe), and seeded uniform
    rows up to ``n`` (default cfg.sample_rows) per head.  Returns [N,3] int32
    (b, h, i); with n == 0 every row."""
    n = cfg.sample_rows if n is None else n
    if not n:
        b, h, i = np.meshgrid(np.arange(cfg.B), np.arange(cfg.Hq), np.arange(cfg.S), indexing="ij")
        return np.stack([b.ravel(), h.ravel(), i.ravel()], 1).astype(np.int32)
    rng = np.random.default_rng(cfg.seed + seed_offset)
    fixed = {0, cfg.S - 1}
    if cfg.layout.startswith("striped"):
        # first and last token of every stripe (token t belongs to stripe t mod P)
        fixed.update(range(cfg.P))
        fixed.update(range(cfg.S - cfg.P, cfg.S))
    else:
        for c in range(cfg.n_chunks):
            fixed.add(c * cfg.chunk)
            fixed.add((c + 1) * cfg.chunk - 1)
    out = []
    for b in range(cfg.B):
        for h in range(cfg.Hq):
            rows = set(fixed)
            while len(rows) < n:
                rows.add(int(rng.integers(0, cfg.S)))
            for i in sorted(rows):
                out.append((b, h, i))
    return np.asarray(out, dtype=np.int32)


def decode_lengths(cfg: Decode) -> torch.Tensor:
    if cfg.fixed_lens:
        return torch.tensor(cfg.fixed_lens, dtype=torch.int32)
    gen = torch.Generator()
    gen.manual_seed(cfg.seed)
    lo = cfg.min_len if cfg.min_len else cfg.capacity // 2
    return torch.randint(lo, cfg.capacity + 1, (cfg.B,), generator=gen, dtype=torch.int64).to(torch.int32)


def decode_inputs(cfg: Decode, device="cpu"):
    """q [B,Hq,D], k/v [B,capacity,Hkv,D] (bf16) and lengths [B] (int32)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed)
    q = randn((cfg.B, cfg.Hq, cfg.D), gen, device, torch.bfloat16)
    k = torch.empty((cfg.B, cfg.capacity, cfg.Hkv, cfg.D), device=device, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(cfg.B):      # one batch entry at a time bounds the float32 temporary
        k[b] = randn((cfg.capacity, cfg.Hkv, cfg.D), gen, device, torch.bfloat16)
        v[b] = randn((cfg.capacity, cfg.Hkv, cfg.D), gen, device, torch.bfloat16)
    lens = decode_lengths(cfg).to(device)
    return q, k, v, lens


def merge_inputs(cfg: Merge, device="cpu"):
    """partials [B,Hq,P,D] float32 N(0,1) and part_lse [B,Hq,P] float32
    N(0,1)*4.  With empty_frac > 0 that share of parts (seeded) gets
    lse = -inf and an O of NaN: an empty part must contribute nothing,
    whatever its O holds."""
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed)
    part = torch.randn((cfg.B, cfg.Hq, cfg.P, cfg.D), generator=gen, device=device, dtype=torch.float32)
    plse = torch.randn((cfg.B, cfg.Hq, cfg.P), generator=gen, device=device, dtype=torch.float32) * 4
    if cfg.empty_frac > 0:
        empty = torch.rand((cfg.B, cfg.Hq, cfg.P), generator=gen, device=device) < cfg.empty_frac
        plse[empty] = float("-inf")
        part[empty] = float("nan")
    return part, plse
