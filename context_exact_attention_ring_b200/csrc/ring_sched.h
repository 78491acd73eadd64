// Ring scheduler shared by every prefill kernel and by the host statistics.
//
// Ownership of chunks, the ring visiting order and the causal tile filter of
// "Lesson 8: Context Parallelism":
//   * section 4A -- contiguous split: rank r owns chunk r (with k chunks per
//                   rank, the sequential assignment of the worked example:
//                   chunks r*k .. r*k+k-1);
//   * section 4B -- zig-zag split: 2P chunks, rank r owns chunks r, 2P-1-r;
//                   the code exercise generalises it to k chunks per rank
//                   (even slots count up from the front of the sequence,
//                   odd slots down from the back);
//   * "Sequence parallelism and ring attention", outlook -- the striped
//                   split, read as: token t belongs to rank t mod P, so the
//                   shard of rank r is the stripe r, r+P, r+2P, ...;
//   * section 2  -- at ring step t rank r holds the K/V block that started on
//                   rank (r - t) mod P;
//   * section 4  -- causal rule: query position i sees key position j <= i,
//                   so K/V tiles that start after the last query of a tile
//                   are never issued, and only tiles straddling the diagonal
//                   (or a ragged chunk end) need the element mask.
// Everything is index arithmetic: no work list is stored, so the library
// needs no memory of its own.  Work items are handed out longest-first
// (queries at later positions meet more keys), which balances the
// persistent CTAs.
//
// Mask positions.  Chunked splits compare global token positions.  The
// striped split compares shard-local row indices instead: query row x of
// stripe r sits at x*P + r and key row y of stripe s at y*P + s, and
// y*P + s <= x*P + r  <=>  y + [s > r] <= x, so key rows are shifted by one
// when the key's stripe comes after the query's.  Both give the same
// "key position <= query position" test, tile filter and element mask.
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

enum { kLayoutContiguous = 0, kLayoutZigzag = 1, kLayoutStriped = 2 };
enum { kModeRing = 0, kModeStep = 1 };
enum { kMaxChunksPerRank = 8 };

struct Plan {
  int B, Hq, Hkv, D;
  int causal;
  int mode;      // kModeRing: buffers hold the whole sequence; kModeStep: one hop
  int layout;    // ring mode: split of the sequence
  int P;         // ring mode: virtual ranks
  int cpr;       // ring mode: chunks per rank
  int striped;   // striped split: chunk c is stripe c (step mode: ids are ranks)
  int strided;   // ring mode + striped: row x of stripe c is buffer row x*P + c
  int C;         // tokens per chunk (per stripe when striped)
  int nqc, nkc;  // chunks held in the Q buffer and in the K/V buffer
  int qid[kMaxChunksPerRank];     // step mode: global chunk index of each Q-buffer chunk
  int kid[kMaxChunksPerRank];     // step mode: global chunk index of each K/V-buffer chunk
  int qorder[kMaxChunksPerRank];  // step mode: Q slots by decreasing chunk index
  int Sq, Skv;   // rows of the Q buffer / K/V buffer (nqc*C, nkc*C)
};

RA_HD int imin(int a, int b) { return a < b ? a : b; }
RA_HD int imax(int a, int b) { return a > b ? a : b; }
RA_HD int cdiv(int a, int b) { return (a + b - 1) / b; }

RA_HD int chunks_per_rank(const Plan& p) { return p.cpr; }

// Owner rank of global chunk c (ring mode).
RA_HD int chunk_owner(const Plan& p, int c) {
  if (p.layout == kLayoutZigzag) {
    const int m = c / p.P;                                 // block of P chunks
    return m < (p.cpr + 1) / 2 ? c - m * p.P              // counted from the front
                               : (m + 1) * p.P - 1 - c;   // counted from the back
  }
  if (p.layout == kLayoutContiguous) return c / p.cpr;
  return c;                                                // striped
}

// j-th chunk (j < chunks_per_rank) owned by rank r.
RA_HD int rank_chunk(const Plan& p, int r, int j) {
  if (p.layout == kLayoutZigzag) {
    const int i = j >> 1;
    return (j & 1) ? p.cpr * p.P - 1 - i * p.P - r : i * p.P + r;
  }
  if (p.layout == kLayoutContiguous) return r * p.cpr + j;
  return r;
}

RA_HD int q_gid(const Plan& p, int slot) { return p.mode == kModeRing ? slot : p.qid[slot]; }
RA_HD int kv_gid(const Plan& p, int slot) { return p.mode == kModeRing ? slot : p.kid[slot]; }

// Mask position of row 0 of a Q chunk / of a K/V chunk met by Q chunk qg.
RA_HD int q_pos_base(const Plan& p, int qslot) { return p.striped ? 0 : q_gid(p, qslot) * p.C; }
RA_HD int kv_pos_base(const Plan& p, int qg, int kslot) {
  return p.striped ? (kv_gid(p, kslot) > qg ? 1 : 0) : kv_gid(p, kslot) * p.C;
}

// Buffer row of row x of chunk slot c.
RA_HD int buf_row(const Plan& p, int slot, int x) { return p.strided ? x * p.P + slot : slot * p.C + x; }

// One K/V tile: rows k0 .. k0 + nvalid - 1 of chunk slot `slot` (buffer row
// row0 for the first when rows are not strided), mask positions
// [pos0, pos0 + nvalid), and the chunk's global id.
struct KvTile {
  int row0, k0, pos0, nvalid, slot, gid, first_in_chunk;
};

// Walks the K/V chunks met by the queries of one Q chunk, in the owning
// rank's ring order (ring mode) or in buffer order (step mode), and the
// tiles inside each chunk.  Incremental: no division per step.
struct KvIter {
  int idx;  // visited chunk index, 0 .. nkc-1
  int kt;   // next tile inside the current chunk
  int src;  // ring mode: the rank whose K/V block is held at this step
  int j;    // ring mode: which of that rank's chunks
  int qg;   // global id of the Q chunk (mask positions of the striped split)
};

RA_HD void kv_begin(const Plan& p, int qslot, KvIter& it) {
  it.idx = 0;
  it.kt = 0;
  it.j = 0;
  it.qg = q_gid(p, qslot);
  it.src = p.mode == kModeRing ? chunk_owner(p, qslot) : 0;   // step 0: the rank's own block
}

RA_HD int kv_cur_slot(const Plan& p, const KvIter& it) {
  return p.mode == kModeStep ? it.idx : rank_chunk(p, it.src, it.j);
}

RA_HD void kv_next_chunk(const Plan& p, KvIter& it) {
  it.idx++;
  it.kt = 0;
  if (p.mode == kModeRing && ++it.j == chunks_per_rank(p)) {
    it.j = 0;
    it.src = it.src == 0 ? p.P - 1 : it.src - 1;   // next step: the block of rank (src - 1) mod P
  }
}

// Next K/V tile (of BN keys; tpc = tiles per chunk) for queries whose last
// valid global position is qhi.  Tiles entirely after qhi are skipped when
// causal.
RA_HD bool kv_next(const Plan& p, int qhi, int BN, int tpc, KvIter& it, KvTile& t) {
  while (it.idx < p.nkc) {
    const int slot = kv_cur_slot(p, it);
    const int gid = kv_gid(p, slot);
    const int k0 = it.kt * BN;
    const int pos0 = kv_pos_base(p, it.qg, slot) + k0;
    if (it.kt >= tpc || (p.causal && pos0 > qhi)) {
      kv_next_chunk(p, it);
      continue;
    }
    t.row0 = buf_row(p, slot, k0);
    t.k0 = k0;
    t.pos0 = pos0;
    t.nvalid = imin(BN, p.C - k0);
    t.slot = slot;
    t.gid = gid;
    t.first_in_chunk = (it.kt == 0);
    it.kt++;
    return true;
  }
  return false;
}

// Number of tiles kv_next yields for these queries (one step per chunk).
RA_HD int kv_count(const Plan& p, int qslot, int qhi, int BN, int tpc) {
  KvIter it;
  kv_begin(p, qslot, it);
  int n = 0;
  for (; it.idx < p.nkc; kv_next_chunk(p, it)) {
    const int cpos = kv_pos_base(p, it.qg, kv_cur_slot(p, it));
    if (!p.causal) {
      n += tpc;
    } else if (cpos <= qhi) {
      n += imin(tpc, (qhi - cpos) / BN + 1);
    }
  }
  return n;
}

// Q slots ordered by decreasing global chunk id (longest work first).
RA_HD int q_slot_by_rank(const Plan& p, int k) { return p.mode == kModeRing ? p.nqc - 1 - k : p.qorder[k]; }

// ---------------------------------------------------------------------------
// Work items of the tensor-core kernel: two 128-row query tiles that share
// every K/V tile.  When the GQA group G = Hq/Hkv is even the two tiles are two
// query heads of one K/V head at the same rows (identical masks); otherwise
// they are two consecutive row tiles of one head inside one chunk.
// ---------------------------------------------------------------------------
struct Item {
  int b, hkv, h[2];
  int qslot;
  int qoff[2];   // first row of tile i inside its chunk
  int qrow0[2];  // buffer row of that row (when rows are not strided)
  int qpos0[2];  // mask position of that row
  int nrows[2];  // valid rows of tile i (0..BM)
  int qlo, qhi;  // first / last valid global position over both tiles
  int tile_in_chunk[2];
};

struct ItemSpace {
  int head_pairs;  // 1: two heads per item; 0: two row tiles per item
  int tq;          // BM-row tiles per Q chunk
  int per_chunk;   // items per Q chunk and head group
  int nbh;         // head groups x batch
  int count;       // total items
};

RA_HD ItemSpace item_space(const Plan& p, int BM) {
  ItemSpace s;
  const int G = p.Hq / p.Hkv;
  s.head_pairs = (G % 2 == 0) ? 1 : 0;
  s.tq = cdiv(p.C, BM);
  s.per_chunk = s.head_pairs ? s.tq : cdiv(s.tq, 2);
  s.nbh = s.head_pairs ? p.B * p.Hkv * (G / 2) : p.B * p.Hq;
  s.count = s.nbh * p.nqc * s.per_chunk;
  return s;
}

// Items are ordered head group by head group, and inside one head group by
// decreasing query position.  A wave of concurrently running CTAs therefore
// streams the K/V of a single kv head (which stays resident in L2), and the
// persistent CTAs, which take the items in waves of the grid size (turn_item;
// the one-CTA kernel deals every other wave in reverse, the CTA-pair kernel
// in the same order every wave, each measured the faster for it), each get an
// even spread of long and short items; the shortest come last.
RA_HD Item item_at(const Plan& p, const ItemSpace& s, int BM, int L) {
  Item it;
  const int per_bh = p.nqc * s.per_chunk;
  const int bh = L / per_bh;
  const int pos_index = L - bh * per_bh;
  const int slot_rank = pos_index / s.per_chunk;
  const int within = s.per_chunk - 1 - (pos_index - slot_rank * s.per_chunk);
  it.qslot = q_slot_by_rank(p, slot_rank);
  const int G = p.Hq / p.Hkv;
  int t0, t1;
  if (s.head_pairs) {
    const int hp_per_b = p.Hkv * (G / 2);
    it.b = bh / hp_per_b;
    const int r = bh - it.b * hp_per_b;
    it.hkv = r / (G / 2);
    const int pair = r - it.hkv * (G / 2);
    it.h[0] = it.hkv * G + 2 * pair;
    it.h[1] = it.h[0] + 1;
    t0 = t1 = within;
  } else {
    it.b = bh / p.Hq;
    it.h[0] = it.h[1] = bh - it.b * p.Hq;
    it.hkv = it.h[0] / G;
    t0 = 2 * within;
    t1 = 2 * within + 1;
  }
  const int cbase_pos = q_pos_base(p, it.qslot);
  const int ts[2] = {t0, t1};
  it.qlo = 0x7fffffff;
  it.qhi = -1;
  for (int i = 0; i < 2; ++i) {
    const int off = ts[i] * BM;
    it.tile_in_chunk[i] = ts[i];
    it.qoff[i] = off;
    it.qrow0[i] = buf_row(p, it.qslot, off);
    it.qpos0[i] = cbase_pos + off;
    it.nrows[i] = ts[i] < s.tq ? imin(BM, p.C - off) : 0;
    if (it.nrows[i] > 0) {
      it.qlo = imin(it.qlo, it.qpos0[i]);
      it.qhi = imax(it.qhi, it.qpos0[i] + it.nrows[i] - 1);
    }
  }
  return it;
}

// ---------------------------------------------------------------------------
// Work items of the CTA-pair kernel: four 128-row query tiles that share every
// K/V tile, two in each CTA of the pair (tile x = 2*cta + i is tile i of CTA
// cta; the pair's M = 256 products for tile i span both CTAs' tile i).  The
// four tiles are four query heads of one kv head at the same rows when the
// GQA group G is a multiple of 4 (identical masks); two heads of one kv head
// at two consecutive row tiles (one row tile per CTA) when G is even; else
// four consecutive row tiles of one head.  qhi is the last valid position
// over all four tiles, so both CTAs walk the same K/V tiles; a tile whose rows
// all precede a K/V tile of that walk gets it fully masked.  Ordering as in
// item_at: head group by head group, longest first.
// ---------------------------------------------------------------------------
RA_HD ItemSpace item_space_pair(const Plan& p, int BM) {
  ItemSpace s;
  const int G = p.Hq / p.Hkv;
  s.tq = cdiv(p.C, BM);
  if (G % 4 == 0) {
    s.head_pairs = 2;
    s.per_chunk = s.tq;
    s.nbh = p.B * p.Hkv * (G / 4);
  } else if (G % 2 == 0) {
    s.head_pairs = 1;
    s.per_chunk = cdiv(s.tq, 2);
    s.nbh = p.B * p.Hkv * (G / 2);
  } else {
    s.head_pairs = 0;
    s.per_chunk = cdiv(s.tq, 4);
    s.nbh = p.B * p.Hq;
  }
  s.count = s.nbh * p.nqc * s.per_chunk;
  return s;
}

// The two tiles of item L that CTA `cta` (0 or 1) of the pair computes.
RA_HD Item item_pair_at(const Plan& p, const ItemSpace& s, int BM, int L, int cta) {
  Item it;
  const int per_bh = p.nqc * s.per_chunk;
  const int bh = L / per_bh;
  const int pos_index = L - bh * per_bh;
  const int slot_rank = pos_index / s.per_chunk;
  const int within = s.per_chunk - 1 - (pos_index - slot_rank * s.per_chunk);
  it.qslot = q_slot_by_rank(p, slot_rank);
  const int G = p.Hq / p.Hkv;
  int hs[4], ts[4];
  if (s.head_pairs == 2) {
    const int per_b = p.Hkv * (G / 4);
    it.b = bh / per_b;
    const int r = bh - it.b * per_b;
    it.hkv = r / (G / 4);
    const int quad = r - it.hkv * (G / 4);
    for (int x = 0; x < 4; ++x) {
      hs[x] = it.hkv * G + 4 * quad + x;
      ts[x] = within;
    }
  } else if (s.head_pairs == 1) {
    const int per_b = p.Hkv * (G / 2);
    it.b = bh / per_b;
    const int r = bh - it.b * per_b;
    it.hkv = r / (G / 2);
    const int pair = r - it.hkv * (G / 2);
    for (int x = 0; x < 4; ++x) {
      hs[x] = it.hkv * G + 2 * pair + (x & 1);
      ts[x] = 2 * within + (x >> 1);
    }
  } else {
    it.b = bh / p.Hq;
    const int h = bh - it.b * p.Hq;
    it.hkv = h / G;
    for (int x = 0; x < 4; ++x) {
      hs[x] = h;
      ts[x] = 4 * within + x;
    }
  }
  const int cbase_pos = q_pos_base(p, it.qslot);
  it.qlo = 0x7fffffff;
  it.qhi = -1;
  for (int x = 0; x < 4; ++x) {
    const int off = ts[x] * BM;
    const int nrows = ts[x] < s.tq ? imin(BM, p.C - off) : 0;
    if (nrows > 0) {
      it.qlo = imin(it.qlo, cbase_pos + off);
      it.qhi = imax(it.qhi, cbase_pos + off + nrows - 1);
    }
    if ((x >> 1) == cta) {
      const int i = x & 1;
      it.h[i] = hs[x];
      it.tile_in_chunk[i] = ts[x];
      it.qoff[i] = off;
      it.qrow0[i] = buf_row(p, it.qslot, off);
      it.qpos0[i] = cbase_pos + off;
      it.nrows[i] = nrows;
    }
  }
  return it;
}

// The item of a persistent CTA's w-th turn (cta < grid CTAs or CTA pairs), or
// -1 when it has none left.  Turns run through the items in waves of `grid`;
// with `snake`, every other wave is dealt in reverse order.  The kernels'
// items are ordered so that neighbouring items have nearly equal work, and
// that work falls along the order (longest first); dealt in the same order
// every wave, the CTAs given the later items of each wave would gain on the
// others with every wave, and the CTAs would drift apart over the launch.  In
// reverse every other wave, a CTA's items of two consecutive waves add up to
// about the same work as any other CTA's, so the CTAs stay in step and read
// the same K/V (or Q/dO) tiles within a short time of one another, while they
// are still in L2.
RA_HD int turn_item(int w, int cta, int grid, int items, bool snake) {
  const long long base = (long long)w * grid;
  if (base >= items) return -1;
  const long long L = base + ((snake && (w & 1)) ? grid - 1 - cta : cta);
  return L < items ? (int)L : -1;
}

// Causal class of a tile with valid query positions [q0,q1] and key positions
// [k0,k1]: 0 full (no mask), 1 partial (mask), 2 skipped.
RA_HD int tile_class(int causal, int q0, int q1, int k0, int k1) {
  if (!causal || k1 <= q0) return 0;
  if (k0 > q1) return 2;
  return 1;
}

}  // namespace ra
