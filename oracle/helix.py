"""Round-robin placement of appended KV tokens across KV-parallel ranks.

TEST INFRASTRUCTURE (see the package docstring).

Source: "NVIDIA unveils Helix Parallelism", on growing the KV cache during
decoding.  To keep one GPU from becoming a memory hotspot, appended tokens
are placed in blocks that rotate over the KV-parallel GPUs (block 0 on GPU 0,
block 1 on GPU 1, continuing in turn), so every rank's share grows at the
same pace.

Reading: the rotation wraps after the last rank (block i goes to rank
i mod P), a block is `block` consecutive appended tokens of one sequence, and
inside a rank's shard tokens keep their arrival order.

Everything here is a step-by-step simulation (one token at a time); no closed
form is used, so the closed forms in the tests pin it.
"""
from __future__ import annotations


def append_rank(n: int, block: int, P: int) -> int:
    """Rank that receives the n-th appended token (n = 0, 1, ...): block
    n // block, dealt to the ranks in turn.

    Follows "NVIDIA unveils Helix Parallelism", on KV cache growth.
    """
    return (n // block) % P


def simulate_appends(shards: list[list], n_appended: int, tokens: list, block: int, P: int, capacity: int):
    """Append `tokens` one by one to `shards` (a list of P lists, each the
    shard's rows in order), starting at append index `n_appended`.

    A token whose shard already holds `capacity` rows is dropped.  Returns
    (shards, n_appended_after, placements, dropped), where placements[j] is
    (rank, row) for token j, or None if it was dropped.

    Follows "NVIDIA unveils Helix Parallelism", on KV cache growth.
    """
    shards = [list(s) for s in shards]
    placements, dropped = [], 0
    n = n_appended
    for tok in tokens:
        p = append_rank(n, block, P)
        if len(shards[p]) < capacity:
            placements.append((p, len(shards[p])))
            shards[p].append(tok)
        else:
            placements.append(None)
            dropped += 1
        n += 1
    return shards, n, placements, dropped
