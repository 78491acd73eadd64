"""Pins for the round-robin KV append simulation (oracle/helix.py): the
placement the Helix page prints (first block to GPU 0, next to GPU 1), a
closed form for the fill counts, the even growth the page states, and
bookkeeping invariants."""
import json
import os

import pytest

from oracle import helix

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "helix_round_robin.json")))


@pytest.mark.parametrize("P,block", [(2, 1), (4, 16), (8, 128), (32, 64)])
def test_printed_first_blocks(P, block):
    # block i (tokens i*block .. i*block+block-1) goes to GPU i, for the blocks the page names
    for blk, gpu in GOLD["printed_first_blocks"]:
        for n in range(blk * block, (blk + 1) * block):
            assert helix.append_rank(n, block, P) == gpu
    # the rotation continues past the last rank: the deal starts again at rank 0
    assert helix.append_rank(P * block, block, P) == 0


def _closed_form_count(N, p, block, P):
    # tokens 0..N-1 form N // (block P) full rounds of `block` each per rank, then a partial round
    # in which rank p gets what is left of its block
    full, rem = divmod(N, block * P)
    return full * block + min(max(rem - p * block, 0), block)


@pytest.mark.parametrize("P,block,N", [(4, 3, 0), (4, 3, 11), (4, 3, 12), (4, 3, 50), (8, 16, 1000), (3, 1, 7)])
def test_fill_counts_closed_form(P, block, N):
    shards, n, placements, dropped = helix.simulate_appends([[] for _ in range(P)], 0, list(range(N)), block, P,
                                                            capacity=10 ** 9)
    assert n == N and dropped == 0
    assert [len(s) for s in shards] == [_closed_form_count(N, p, block, P) for p in range(P)]


@pytest.mark.parametrize("P,block", [(2, 1), (4, 8), (8, 64), (5, 7)])
def test_even_growth(P, block):
    # from equal shards, fill counts never differ by more than one block at any time
    shards = [[None] * 100 for _ in range(P)]
    for step in range(P * block * 3 + 5):
        shards, _, _, _ = helix.simulate_appends(shards, step, [step], block, P, capacity=10 ** 9)
        lens = [len(s) for s in shards]
        assert max(lens) - min(lens) <= block


def test_every_token_once_in_arrival_order():
    P, block = 4, 5
    shards, n, placements, _ = helix.simulate_appends([[] for _ in range(P)], 7, list(range(200)), block, P, 10 ** 9)
    flat = sorted(t for s in shards for t in s)
    assert flat == list(range(200)) and n == 207
    for s in shards:
        assert s == sorted(s)
    for tok, (p, row) in enumerate(placements):
        assert shards[p][row] == tok


def test_capacity_drops_and_keeps_order():
    P, block, cap = 2, 2, 3
    shards, n, placements, dropped = helix.simulate_appends([[], []], 0, list(range(10)), block, P, cap)
    # tokens 0,1 -> r0; 2,3 -> r1; 4,5 -> r0 (5 fills r0 to 3... 4 is row 2, 5 is dropped); 6,7 -> r1 (6 row 2, 7 dropped)
    assert shards == [[0, 1, 4], [2, 3, 6]]
    assert dropped == 4 and n == 10
    assert placements[5] is None and placements[4] == (0, 2)
