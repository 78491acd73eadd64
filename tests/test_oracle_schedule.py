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
    assert sch.layout_assignment(P, "contiguous2") == _keys_int(GOLD["sequential_2_per_rank"])
    assert sch.layout_assignment(P, "zigzag") == _keys_int(GOLD["zigzag"])
    # the owner of every chunk agrees with the printed assignment
    for r, cs in _keys_int(GOLD["zigzag"]).items():
        assert all(sch.chunk_owner(c, P, "zigzag") == r for c in cs)


def test_printed_workloads():
    # causal chunk pairs per rank, counted by walking each rank's ring loop
    P = GOLD["P"]
    ws = dict(enumerate(sch.per_rank_pairs(P, "contiguous2", True)))
    wz = dict(enumerate(sch.per_rank_pairs(P, "zigzag", True)))
    assert ws == _keys_int(GOLD["sequential_workload"])
    assert wz == _keys_int(GOLD["zigzag_workload"])
    assert max(ws.values()) / min(ws.values()) == GOLD["sequential_max_over_min"]


def test_printed_rotation():
    assert sch.block_sources(GOLD["P"], 2, 2) == GOLD["rank2_rotation"]


@pytest.mark.parametrize("P", list(range(1, 33)))
def test_zigzag_closed_form(P):
    # section 4B: every rank does (r+1) + (2P-r) = 2P+1 causal chunk pairs
    assert sch.per_rank_pairs(P, "zigzag", True) == [2 * P + 1] * P


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


# --------------------------------------------------------------------------- split variants
@pytest.mark.parametrize("P,k", [(p, k) for p in (1, 2, 3, 4, 8) for k in (2, 3, 4, 5, 8)])
def test_general_zigzag_is_a_partition(P, k):
    own = sch.layout_assignment(P, f"zigzag{k}")
    assert sorted(c for cs in own.values() for c in cs) == list(range(P * k))
    # the code exercise's slot rule, as printed: even slot 2i counts up from the front (chunk
    # iP + r), odd slot 2i+1 down from the back (chunk kP - 1 - iP - r); for k = 2 the section
    # 4B pair {r, 2P-1-r}
    for r in range(P):
        assert own[r] == [(j // 2) * P + r if j % 2 == 0 else P * k - 1 - (j // 2) * P - r for j in range(k)]


@pytest.mark.parametrize("P,k", [(p, k) for p in (1, 2, 3, 4, 8, 16) for k in (2, 4, 6, 8)])
def test_general_zigzag_even_k_balanced_closed_form(P, k):
    # slots 2i and 2i+1 hold chunks iP+r and (k-i)P-1-r: (iP+r+1) + ((k-i)P-r) = kP+1 pairs,
    # so each rank does (k/2)(kP+1) causal chunk pairs whatever its index
    expect = [(k // 2) * (k * P + 1)] * P
    assert sch.per_rank_pairs(P, f"zigzag{k}", True) == expect


@pytest.mark.parametrize("P,k", [(2, 3), (4, 3), (3, 5)])
def test_general_zigzag_odd_k_near_balanced(P, k):
    # odd k: the unpaired last slot (a front chunk) leaves a spread of at most P-1 pairs
    w = sch.per_rank_pairs(P, f"zigzag{k}", True)
    assert max(w) - min(w) == P - 1


@pytest.mark.parametrize("P,k", [(2, 2), (4, 3), (3, 4)])
def test_sequential_k_per_rank_pairs(P, k):
    # rank r holds chunks rk .. rk+k-1, chunk c meets c+1 chunks: sum = k(rk) + k(k+1)/2
    assert sch.per_rank_pairs(P, f"contiguous{k}", True) == [k * r * k + k * (k + 1) // 2 for r in range(P)]


@pytest.mark.parametrize("S,P", [(64, 4), (96, 3), (1024, 8)])
def test_striped_tokens_partition(S, P):
    st = sch.striped_tokens(S, P)
    assert sorted(t for ts in st.values() for t in ts) == list(range(S))
    assert all(t % P == r for r, ts in st.items() for t in ts)


@pytest.mark.parametrize("S,P", [(64, 4), (4096, 8), (8192, 16)])
def test_striped_every_pair_meets_keys(S, P):
    # every rank's stripe has keys before some query of every other stripe
    assert sch.per_rank_pairs(P, "striped", True, S) == [P] * P


@pytest.mark.parametrize("S,P,T", [(4096, 4, 128), (8192, 8, 128), (2048, 2, 64), (131072, 16, 128)])
def test_striped_tile_totals_closed_form(S, P, T):
    # stripes of n = S/(P*T) tiles: pair (r, s) keeps key tile b for query tile a iff b < a (full) or
    # b == a (partial: the diagonal, shifted by one row when s > r), so each of the P^2 pairs is a
    # lower triangle of n(n-1)/2 full, n partial, n(n-1)/2 skipped tiles
    full, partial, skipped, per_rank = sch.tile_classes(S, P, "striped", True, T, T)
    n = S // (P * T)
    assert (full, partial, skipped) == (P * P * n * (n - 1) // 2, P * P * n, P * P * n * (n - 1) // 2)
    assert len(set(per_rank)) == 1


def _brute_tile_classes(S, P, layout, tq, tk):
    """Element by element: a tile is full if every (query, key) pair is allowed, skipped if none is."""
    pos = sch.chunk_positions(S, P, layout)
    own = sch.layout_assignment(P, layout)
    out = [0, 0, 0]
    for r in range(P):
        for src in range(P):
            for qc in own[r]:
                for kc in own[src]:
                    qp, kp = pos[qc], pos[kc]
                    for a in range(0, len(qp), tq):
                        for b in range(0, len(kp), tk):
                            ok = [kk <= qq for qq in qp[a:a + tq] for kk in kp[b:b + tk]]
                            out[0 if all(ok) else 2 if not any(ok) else 1] += 1
    return tuple(out)


@pytest.mark.parametrize("S,P,layout,tq,tk", [
    (48, 3, "striped", 4, 4), (64, 4, "striped", 5, 3), (60, 2, "zigzag3", 4, 4), (64, 2, "zigzag4", 3, 5),
    (48, 4, "contiguous2", 4, 4), (40, 2, "zigzag", 4, 3), (30, 3, "contiguous", 4, 4),
])
def test_tile_classes_brute_force(S, P, layout, tq, tk):
    full, partial, skipped, _ = sch.tile_classes(S, P, layout, True, tq, tk)
    assert (full, partial, skipped) == _brute_tile_classes(S, P, layout, tq, tk)


def test_kv_visit_order_general_splits():
    for P in (1, 2, 3, 4):
        for layout in ("zigzag3", "zigzag4", "contiguous2", "striped"):
            k = sch.parse_layout(layout)[1]
            for r in range(P):
                order = sch.kv_visit_order(P, layout, r)
                assert sorted(order) == list(range(P * k))
                assert order[:k] == sch.layout_assignment(P, layout)[r]
