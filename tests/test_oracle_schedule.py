"""Pins for the schedule enumerator (oracle/schedule.py).

Each pin comes from outside the enumerator: the values printed by
"Lesson 8: Context Parallelism" (tests/golden/lesson8_schedule.json), its
closed forms (2P+1 pairs per zig-zag rank, section 4B; i+1 pairs per
contiguous rank, section 4A), and the tile totals of a lower-triangular
matrix, which do not depend on how the sequence is split.
"""
import json
import os

import pytest

from oracle import schedule as sch

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "lesson8_schedule.json")))


def _keys_int(d):
    return {int(k): v for k, v in d.items()}


def test_printed_assignments():
    P = GOLD["P"]
    assert sch.sequential_assignment(P, 2) == _keys_int(GOLD["sequential_2_per_rank"])
    assert sch.zigzag_assignment(P, 2) == _keys_int(GOLD["zigzag"])


def test_printed_workloads():
    P = GOLD["P"]
    ws = sch.causal_workload(sch.sequential_assignment(P, 2))
    wz = sch.causal_workload(sch.zigzag_assignment(P, 2))
    assert ws == _keys_int(GOLD["sequential_workload"])
    assert wz == _keys_int(GOLD["zigzag_workload"])
    assert max(ws.values()) / min(ws.values()) == GOLD["sequential_max_over_min"]


def test_printed_rotation():
    assert sch.ring_rotation(GOLD["P"], 2, 2) == GOLD["rank2_rotation"]


@pytest.mark.parametrize("P", list(range(1, 33)))
def test_zigzag_closed_form(P):
    # section 4B: every rank does (r+1) + (2P-r) = 2P+1 causal chunk pairs
    assert sch.per_rank_pairs(P, "zigzag", True) == [2 * P + 1] * P
    assert list(sch.causal_workload(sch.zigzag_assignment(P, 2)).values()) == [2 * P + 1] * P


@pytest.mark.parametrize("P", list(range(1, 17)))
def test_contiguous_closed_form(P):
    # section 4A: with one chunk per rank, rank i computes i+1 chunk pairs
    assert sch.per_rank_pairs(P, "contiguous", True) == [i + 1 for i in range(P)]
    # the lockstep efficiency sum(w) / (P * max w) = (P+1)/(2P) -> about half wasted
    w = sch.per_rank_pairs(P, "contiguous", True)
    assert sum(w) * 2 * P == (P + 1) * P * max(w)


@pytest.mark.parametrize("P,layout", [(p, l) for p in (1, 2, 3, 4, 8) for l in ("contiguous", "zigzag")])
def test_noncausal_every_pair_full(P, layout):
    pairs = sch.ring_pairs(P, layout, False)
    n = P * (1 if layout == "contiguous" else 2)
    assert len(pairs) == n * n and all(p.kind == "full" for p in pairs)


@pytest.mark.parametrize("P", [1, 2, 3, 5, 8])
def test_zigzag_pair_split(P):
    # step 0: two diagonal pairs and one full pair; every later step: exactly two full pairs
    pairs = sch.ring_pairs(P, "zigzag", True)
    for r in range(P):
        for t in range(P):
            kinds = sorted(p.kind for p in pairs if p.rank == r and p.step == t and p.kind != "skip")
            assert kinds == (["diag", "diag", "full"] if t == 0 else ["full", "full"])


@pytest.mark.parametrize("P,layout,S,T", [(4, "contiguous", 1024, 128), (8, "contiguous", 8192, 128),
                                          (4, "zigzag", 2048, 128), (8, "zigzag", 32768, 128),
                                          (16, "zigzag", 131072, 128), (3, "zigzag", 1536, 64)])
def test_tile_totals_lower_triangle(P, layout, S, T):
    # chunks aligned to the tile: T(T-1)/2 full, T partial (the diagonal), T(T-1)/2 skipped tiles
    full, partial, skipped, per_rank = sch.tile_classes(S, P, layout, True, T, T)
    n = S // T
    assert (full, partial, skipped) == (n * (n - 1) // 2, n, n * (n - 1) // 2)
    assert sum(per_rank) == full + partial


def test_tile_totals_zigzag_balanced():
    # zig-zag balances processed tiles across ranks exactly when tiles align with chunks
    _, _, _, per_rank = sch.tile_classes(16 * 1024, 8, "zigzag", True, 128, 128)
    assert len(set(per_rank)) == 1


def test_kv_visit_order_covers_all_chunks_once():
    for P in (1, 2, 4, 7):
        for layout in ("contiguous", "zigzag"):
            n = P * (1 if layout == "contiguous" else 2)
            for r in range(P):
                order = sch.kv_visit_order(P, layout, r)
                assert sorted(order) == list(range(n))
                # step 0 is the rank's own K/V
                assert order[: n // P] == sch.layout_assignment(P, layout)[r]
