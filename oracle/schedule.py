"""Schedule enumerator for the ring: chunk ownership, ring rotation, causal
chunk-pair counts and tile classes, all by brute-force enumeration.

TEST INFRASTRUCTURE (see the package docstring).

Sources (each function cites the passage it follows):
  * "Lesson 8: Context Parallelism", section 2: at step t rank r works on the
    K/V block that left rank (r - t) mod P; P steps per ring loop.
  * same lesson, section 4A: contiguous split, rank r owns chunk r.
  * same lesson, section 4B: zig-zag split into 2P chunks, rank r owns chunks
    r and 2P-1-r; the worked example also gives the sequential assignment of
    k consecutive chunks per rank.
  * same lesson, section 4 and the worked example: under the causal mask,
    query chunk q attends K/V chunks 0..q, so a rank's workload is the sum of
    (q + 1) over its query chunks.
  * same lesson, code exercise: the general zig-zag rule for k chunks per rank
    (even slots count up from the front, odd slots down from the back).

Nothing here is closed-form: the closed forms printed on the page (2P+1 pairs
per zig-zag rank, i+1 per contiguous rank) are *pins* checked against these
enumerations in tests/test_oracle_schedule.py.
"""
from __future__ import annotations

from dataclasses import dataclass


def sequential_assignment(P: int, chunks_per_rank: int) -> dict[int, list[int]]:
    """Rank r owns chunks r*k .. r*k + k - 1 (worked example, sequential)."""
    return {r: [r * chunks_per_rank + c for c in range(chunks_per_rank)] for r in range(P)}


def zigzag_assignment(P: int, chunks_per_rank: int = 2) -> dict[int, list[int]]:
    """Zig-zag ownership (section 4B; general k from the code exercise).

    Slot c of rank r: even c takes chunk (c/2)*P + r, counting from the front;
    odd c takes chunk total-1-(c//2)*P-r, counting from the back.  For k = 2
    this is {r, 2P-1-r}.
    """
    total = P * chunks_per_rank
    out = {}
    for r in range(P):
        owned = []
        for c in range(chunks_per_rank):
            if c % 2 == 0:
                owned.append((c // 2) * P + r)
            else:
                owned.append(total - 1 - (c // 2) * P - r)
        out[r] = owned
    return out


def layout_assignment(P: int, layout: str) -> dict[int, list[int]]:
    """The two splits of the hot path: 'contiguous' (one chunk per rank,
    section 4A) and 'zigzag' (two chunks per rank, section 4B)."""
    if layout == "contiguous":
        return sequential_assignment(P, 1)
    if layout == "zigzag":
        return zigzag_assignment(P, 2)
    raise ValueError(layout)


def causal_workload(assign: dict[int, list[int]]) -> dict[int, int]:
    """Causal chunk pairs per rank: query chunk q sees K/V chunks 0..q, so the
    rank's count is the number of (q, kv) chunk pairs with kv <= q (section 4).
    Enumerated pair by pair rather than summed in closed form."""
    n_chunks = sum(len(v) for v in assign.values())
    return {r: sum(1 for q in qs for kv in range(n_chunks) if kv <= q) for r, qs in assign.items()}


def ring_rotation(P: int, rank: int, start: int | None = None) -> list[int]:
    """Which rank's K/V block rank ``rank`` holds at steps t = 0..P-1: blocks
    move from rank r-1 to rank r each step, so at step t it is the block that
    started on rank (start - t) mod P (section 2; start defaults to rank)."""
    s = rank if start is None else start
    return [(s - t) % P for t in range(P)]


@dataclass(frozen=True)
class Pair:
    rank: int       # virtual rank holding the queries
    step: int       # ring step t
    q_chunk: int    # global chunk index of the query chunk
    kv_chunk: int   # global chunk index of the key/value chunk
    kind: str       # 'full' | 'diag' | 'skip'


def ring_pairs(P: int, layout: str, causal: bool) -> list[Pair]:
    """Every (rank, step, q chunk, kv chunk) the ring loop meets, classified
    under the causal rule (kv < q full, kv == q diagonal, kv > q skipped)."""
    own = layout_assignment(P, layout)
    out = []
    for r in range(P):
        for t, src in enumerate(ring_rotation(P, r)):
            for qc in own[r]:
                for kc in own[src]:
                    if not causal or kc < qc:
                        kind = "full"
                    elif kc == qc:
                        kind = "diag"
                    else:
                        kind = "skip"
                    out.append(Pair(r, t, qc, kc, kind))
    return out


def per_rank_pairs(P: int, layout: str, causal: bool) -> list[int]:
    """Unmasked chunk pairs per rank (a diagonal pair counts as one)."""
    cnt = [0] * P
    for p in ring_pairs(P, layout, causal):
        if p.kind != "skip":
            cnt[p.rank] += 1
    return cnt


def chunk_len(S: int, P: int, layout: str) -> int:
    n = P if layout == "contiguous" else 2 * P
    if S % n:
        raise ValueError("S must divide into the chunks")
    return S // n


def tile_classes(S: int, P: int, layout: str, causal: bool, tile_q: int, tile_k: int):
    """Tile classes for one (batch, head), enumerated tile by tile.

    Each chunk pair met by the ring is cut into tiles of tile_q query rows and
    tile_k keys (the last tile of a chunk may be shorter).  With global first
    and last positions [q0,q1] x [k0,k1] a tile is 'full' if k1 <= q0,
    'skip' if k0 > q1, else 'partial' (causal); all tiles are full otherwise.
    Returns (full, partial, skipped, per_rank_processed[P]) where processed
    counts full + partial tiles by the rank owning the queries.
    """
    C = chunk_len(S, P, layout)
    full = partial = skipped = 0
    per_rank = [0] * P
    for pr in ring_pairs(P, layout, causal):
        qbase, kbase = pr.q_chunk * C, pr.kv_chunk * C
        for qa in range(0, C, tile_q):
            q0, q1 = qbase + qa, qbase + min(qa + tile_q, C) - 1
            for ka in range(0, C, tile_k):
                k0, k1 = kbase + ka, kbase + min(ka + tile_k, C) - 1
                if not causal or k1 <= q0:
                    full += 1
                    per_rank[pr.rank] += 1
                elif k0 > q1:
                    skipped += 1
                else:
                    partial += 1
                    per_rank[pr.rank] += 1
    return full, partial, skipped, per_rank


def rank_of_chunk(P: int, layout: str) -> dict[int, int]:
    """Owner rank of each global chunk."""
    return {c: r for r, cs in layout_assignment(P, layout).items() for c in cs}


def kv_visit_order(P: int, layout: str, rank: int) -> list[int]:
    """Global K/V chunk indices in the order rank ``rank`` meets them during
    one ring loop (for zig-zag, both chunks of the source rank at each step,
    in the order that rank owns them)."""
    own = layout_assignment(P, layout)
    return [c for src in ring_rotation(P, rank) for c in own[src]]
