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
  * "Sequence parallelism and ring attention", outlook: names the striped
    variant; read here as token t belonging to rank t mod P.

Nothing here is closed-form: the closed forms printed on the page (2P+1 pairs
per zig-zag rank, i+1 per contiguous rank) are *pins* checked against these
enumerations in tests/test_oracle_schedule.py.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

_DEFAULT_K = {"contiguous": 1, "zigzag": 2, "striped": 1}


def parse_layout(layout: str) -> tuple[str, int]:
    """Split name and chunks per rank: 'contiguous' | 'zigzag' | 'striped',
    optionally followed by k ('zigzag4' = four chunks per rank).

    Plumbing (names the splits of "Lesson 8", sections 4A and 4B, and the
    striped variant); no arithmetic.
    """
    name = layout.rstrip("0123456789")
    if name not in _DEFAULT_K:
        raise ValueError(layout)
    k = int(layout[len(name):]) if layout != name else _DEFAULT_K[name]
    if (name == "zigzag" and k < 2) or (name == "striped" and k != 1) or k < 1:
        raise ValueError(layout)
    return name, k


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


def striped_tokens(S: int, P: int) -> dict[int, list[int]]:
    """Striped split: rank r holds tokens r, r+P, r+2P, ... in that order.

    Reading of the striped variant named in "Sequence parallelism and ring
    attention", outlook.
    """
    return {r: list(range(r, S, P)) for r in range(P)}


def layout_assignment(P: int, layout: str) -> dict[int, list[int]]:
    """Chunks owned by each rank: 'contiguous' (section 4A; with k chunks per
    rank the sequential assignment), 'zigzag' (section 4B; k per rank from the
    code exercise).  For 'striped' the one "chunk" of rank r is its stripe,
    numbered r."""
    name, k = parse_layout(layout)
    if name == "contiguous":
        return sequential_assignment(P, k)
    if name == "zigzag":
        return zigzag_assignment(P, k)
    return {r: [r] for r in range(P)}


def chunk_positions(S: int, P: int, layout: str) -> dict[int, list[int]]:
    """Global token positions of every chunk, in the chunk's row order.

    Chunks of "Lesson 8", sections 4A and 4B (stripes for the striped split).
    """
    name, _ = parse_layout(layout)
    if name == "striped":
        if S % P:
            raise ValueError("S must divide into the stripes")
        return striped_tokens(S, P)
    C = chunk_len(S, P, layout)
    n = S // C
    return {c: list(range(c * C, (c + 1) * C)) for c in range(n)}


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


def ring_pairs(P: int, layout: str, causal: bool, S: int | None = None) -> list[Pair]:
    """Every (rank, step, q chunk, kv chunk) the ring loop meets, classified
    under the causal rule.  Chunked splits: kv < q full, kv == q diagonal,
    kv > q skipped.  Striped split (S needed): from the token positions, full
    if every key precedes every query, skipped if none does, else 'diag'.

    Rotation of "Lesson 8", section 2; causal rule of section 4.
    """
    own = layout_assignment(P, layout)
    striped = parse_layout(layout)[0] == "striped"
    pos = chunk_positions(S, P, layout) if striped else None
    out = []
    for r in range(P):
        for t, src in enumerate(ring_rotation(P, r)):
            for qc in own[r]:
                for kc in own[src]:
                    if striped:
                        qp, kp = pos[qc], pos[kc]
                        if not causal or max(kp) <= min(qp):
                            kind = "full"
                        elif min(kp) > max(qp):
                            kind = "skip"
                        else:
                            kind = "diag"
                    elif not causal or kc < qc:
                        kind = "full"
                    elif kc == qc:
                        kind = "diag"
                    else:
                        kind = "skip"
                    out.append(Pair(r, t, qc, kc, kind))
    return out


def per_rank_pairs(P: int, layout: str, causal: bool, S: int | None = None) -> list[int]:
    """Unmasked chunk pairs per rank (a diagonal pair counts as one).

    Counting of "Lesson 8", section 4B (a diagonal pair counts once).
    """
    cnt = [0] * P
    for p in ring_pairs(P, layout, causal, S):
        if p.kind != "skip":
            cnt[p.rank] += 1
    return cnt


def chunk_len(S: int, P: int, layout: str) -> int:
    """Rows per chunk (per stripe for the striped split).

    Chunk length of "Lesson 8", sections 4A and 4B.
    """
    name, k = parse_layout(layout)
    n = P * k
    if S % n:
        raise ValueError("S must divide into the chunks")
    return S // n


def tile_classes(S: int, P: int, layout: str, causal: bool, tile_q: int, tile_k: int):
    """Tile classes for one (batch, head), enumerated tile by tile.

    Each chunk pair met by the ring is cut into tiles of tile_q query rows and
    tile_k key rows in the chunks' row order (the last tile of a chunk may be
    shorter).  From the global token positions of the tile's rows a tile is
    'full' if its last key precedes its first query (max key <= min query),
    'skip' if its first key follows its last query (min key > max query),
    else 'partial' (causal); all tiles are full otherwise.
    Returns (full, partial, skipped, per_rank_processed[P]) where processed
    counts full + partial tiles by the rank owning the queries.

    Causal rule of "Lesson 8", section 4, applied tile by tile.
    """
    pos = {c: np.asarray(v, dtype=np.int64) for c, v in chunk_positions(S, P, layout).items()}

    def spans(x, t):
        lo = np.array([x[a:a + t].min() for a in range(0, len(x), t)])
        hi = np.array([x[a:a + t].max() for a in range(0, len(x), t)])
        return lo, hi

    qspan = {c: spans(x, tile_q) for c, x in pos.items()}
    kspan = {c: spans(x, tile_k) for c, x in pos.items()}
    full = partial = skipped = 0
    per_rank = [0] * P
    for pr in ring_pairs(P, layout, causal, S):
        q0, q1 = qspan[pr.q_chunk]
        k0, k1 = kspan[pr.kv_chunk]
        if not causal:
            f, sk = q0.size * k0.size, 0
        else:
            f = int(np.sum(k1[None, :] <= q0[:, None]))
            sk = int(np.sum(k0[None, :] > q1[:, None]))
        pa = q0.size * k0.size - f - sk
        full += f
        partial += pa
        skipped += sk
        per_rank[pr.rank] += f + pa
    return full, partial, skipped, per_rank


def kv_visit_order(P: int, layout: str, rank: int) -> list[int]:
    """Global K/V chunk indices in the order rank ``rank`` meets them during
    one ring loop (for zig-zag, both chunks of the source rank at each step,
    in the order that rank owns them).

    Rotation of "Lesson 8", section 2.
    """
    own = layout_assignment(P, layout)
    return [c for src in ring_rotation(P, rank) for c in own[src]]
