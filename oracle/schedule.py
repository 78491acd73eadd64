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
    query chunk q attends K/V chunks 0..q; a rank's workload is counted here
    by walking its ring loop pair by pair (per_rank_pairs).
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


def _front_bands(k: int) -> int:
    """Zig-zag split: the sequence of P*k chunks is read as k bands of P
    consecutive chunks.  The first ceil(k/2) bands are dealt front to back in
    order of rank; the others are mirrored (rank 0 takes the band's last
    chunk), which is section 4B's pairing of an early chunk with a late one."""
    return (k + 1) // 2


def chunk_owner(c: int, P: int, layout: str) -> int:
    """Rank that owns global chunk c.

    Contiguous split (section 4A; k chunks per rank: the worked example's
    sequential assignment): chunks r*k .. r*k+k-1 belong to rank r.  Zig-zag
    split (section 4B; k per rank: the code exercise's rule, restated by
    bands): chunk c sits in band c // P at place c mod P; a front band gives
    it to rank (c mod P), a back band to rank P-1-(c mod P).  Striped split:
    the one "chunk" of rank r is its stripe, numbered r.
    """
    name, k = parse_layout(layout)
    if name == "contiguous":
        return c // k
    if name == "striped":
        return c
    band, place = divmod(c, P)
    return place if band < _front_bands(k) else P - 1 - place


def layout_assignment(P: int, layout: str) -> dict[int, list[int]]:
    """Chunks owned by each rank, in the rank's slot order.

    Contiguous: ascending.  Zig-zag: the rank's chunk of the first front band,
    then of the last back band, then of the second front band, of the
    next-to-last back band, and so on (slot 2i from the front, slot 2i+1 from
    the back: section 4B and the code exercise).  For 'striped' the one
    "chunk" of rank r is its stripe, numbered r.  Every chunk's owner comes
    from chunk_owner; this only fixes the order in which a rank lists them.
    """
    name, k = parse_layout(layout)
    if name == "striped":
        return {r: [r] for r in range(P)}
    if name == "contiguous":
        order = list(range(P * k))
    else:
        fronts = list(range(_front_bands(k)))
        backs = list(range(k - 1, _front_bands(k) - 1, -1))
        bands = [b for i in range(len(fronts)) for b in fronts[i:i + 1] + backs[i:i + 1]]
        order = [c for b in bands for c in range(b * P, (b + 1) * P)]
    held: dict[int, list[int]] = {r: [] for r in range(P)}
    for c in order:
        held[chunk_owner(c, P, layout)].append(c)
    return held


def striped_tokens(S: int, P: int) -> dict[int, list[int]]:
    """Striped split: rank r holds tokens r, r+P, r+2P, ... in that order.

    Reading of the striped variant named in "Sequence parallelism and ring
    attention", outlook.
    """
    return {r: list(range(r, S, P)) for r in range(P)}


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


def block_sources(P: int, rank: int, start: int | None = None) -> list[int]:
    """The rank whose K/V block rank ``rank`` holds at steps t = 0..P-1.

    Section 2: every step each block moves on to the next rank, so at step t
    a rank holds the block that began t hops behind it, i.e. on rank
    (start - t) mod P (start defaults to the rank itself).
    """
    first = rank if start is None else start
    return [(first - hop) % P for hop in range(P)]


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
        for t, src in enumerate(block_sources(P, r)):
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
    return [c for src in block_sources(P, rank) for c in own[src]]
