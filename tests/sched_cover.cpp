// Host-side walk of the ring scheduler (context_exact_attention_ring_b200/
// csrc/ring_sched.h), the code every prefill kernel uses to pick its work.
// Built with g++ by tests/test_sched_cover.py; no GPU involved.
//
// For one problem it runs through every work item the way the tensor-core
// kernel does (item_at over all items; for both query tiles of an item, the
// K/V tiles of kv_next with the element mask "key position <= query
// position" and "column < valid keys") and records which (query token, key
// token) pairs of which (batch, head) get computed.  It then checks, against
// the true global token positions of the split:
//   * every pair the causal rule of "Lesson 8: Context Parallelism",
//     section 4, allows (all pairs when not causal) is computed exactly once,
//     and no other pair is;
//   * every output row (batch, head, query token) is owned by exactly one
//     item tile, so no two CTAs write the same row;
//   * every buffer row, head and batch index stays inside its tensor, and an
//     item's kv head is the GQA group of both of its query heads;
//   * kv_count, which tells the MMA warp how many tiles to expect, equals the
//     number of tiles kv_next hands the producer, so neither waits for a tile
//     the other never sends.
// Returns 0 if every check holds, else a code naming the first failure (and
// fills `msg`).
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <vector>

#include "../context_exact_attention_ring_b200/csrc/ring_sched.h"

using namespace ra;

namespace {

struct Walk {
  const Plan& p;
  int S, BM, BN;
  // global token of buffer row `row` of chunk slot `slot` (rows are global tokens in ring mode;
  // in step mode, the shard's chunks / stripes give them)
  std::vector<int> qtok, ktok;  // per buffer row
  std::vector<uint8_t> cover;   // [B][Hq][Sq][Skv] (buffer rows)
  std::vector<uint8_t> owner;   // [B][Hq][Sq]
  int64_t items = 0, tiles = 0, pairs = 0;
  char* msg;

  Walk(const Plan& pl, int S_, int BM_, int BN_, char* m) : p(pl), S(S_), BM(BM_), BN(BN_), msg(m) {}

  int fail(int code, const char* what, int a = 0, int b = 0, int c = 0) {
    snprintf(msg, 256, "%s (%d, %d, %d)", what, a, b, c);
    return code;
  }

  int run() {
    cover.assign((size_t)p.B * p.Hq * p.Sq * p.Skv, 0);
    owner.assign((size_t)p.B * p.Hq * p.Sq, 0);
    const ItemSpace sp = item_space(p, BM);
    const int tpc = cdiv(p.C, BN);
    const int G = p.Hq / p.Hkv;
    for (int L = 0; L < sp.count; ++L) {
      const Item it = item_at(p, sp, BM, L);
      ++items;
      if (it.b < 0 || it.b >= p.B || it.hkv < 0 || it.hkv >= p.Hkv) return fail(1, "item batch/kv head out of range", L);
      if (it.qslot < 0 || it.qslot >= p.nqc) return fail(2, "item query chunk out of range", L, it.qslot);
      for (int i = 0; i < 2; ++i) {
        if (it.h[i] < 0 || it.h[i] >= p.Hq || it.h[i] / G != it.hkv) return fail(3, "query head not in the kv group", L, i);
        if (it.nrows[i] < 0 || it.nrows[i] > BM || (it.nrows[i] > 0 && it.qoff[i] + it.nrows[i] > p.C))
          return fail(4, "query tile rows out of range", L, i, it.nrows[i]);
        for (int r = 0; r < it.nrows[i]; ++r) {
          const int row = buf_row(p, it.qslot, it.qoff[i] + r);
          if (row < 0 || row >= p.Sq) return fail(5, "query buffer row out of range", L, i, row);
          if (!p.strided && row != it.qrow0[i] + r) return fail(6, "qrow0 disagrees with buf_row", L, i, r);
          uint8_t& o = owner[((size_t)it.b * p.Hq + it.h[i]) * p.Sq + row];
          if (++o != 1) return fail(7, "output row owned by two item tiles", L, i, row);
        }
      }
      KvIter iter;
      kv_begin(p, it.qslot, iter);
      KvTile t;
      int n = 0;
      while (kv_next(p, it.qhi, BN, tpc, iter, t)) {
        ++n;
        ++tiles;
        if (t.slot < 0 || t.slot >= p.nkc || t.nvalid < 1 || t.nvalid > BN || t.k0 + t.nvalid > p.C)
          return fail(8, "kv tile out of range", L, t.slot, t.k0);
        for (int i = 0; i < 2; ++i) {
          for (int r = 0; r < it.nrows[i]; ++r) {
            const int qpos = it.qpos0[i] + r;
            const int qrow = buf_row(p, it.qslot, it.qoff[i] + r);
            for (int c = 0; c < t.nvalid; ++c) {
              if (p.causal && t.pos0 + c > qpos) continue;             // the kernel's element mask
              const int krow = buf_row(p, t.slot, t.k0 + c);
              if (krow < 0 || krow >= p.Skv) return fail(9, "key buffer row out of range", L, krow);
              if (!p.strided && krow != t.row0 + c) return fail(10, "row0 disagrees with buf_row", L, c);
              uint8_t& x = cover[(((size_t)it.b * p.Hq + it.h[i]) * p.Sq + qrow) * p.Skv + krow];
              if (++x > 1) return fail(11, "pair computed twice", L, qrow, krow);
              ++pairs;
            }
          }
        }
      }
      if (n != kv_count(p, it.qslot, it.qhi, BN, tpc)) return fail(12, "kv_count disagrees with kv_next", L, n);
    }
    // every allowed pair once, no other pair; every row owned once
    for (int b = 0; b < p.B; ++b)
      for (int h = 0; h < p.Hq; ++h)
        for (int qr = 0; qr < p.Sq; ++qr) {
          if (owner[((size_t)b * p.Hq + h) * p.Sq + qr] != 1) return fail(13, "output row owned by no item tile", b, h, qr);
          for (int kr = 0; kr < p.Skv; ++kr) {
            const bool allowed = !p.causal || ktok[kr] <= qtok[qr];
            const uint8_t x = cover[(((size_t)b * p.Hq + h) * p.Sq + qr) * p.Skv + kr];
            if (x != (allowed ? 1 : 0))
              return fail(allowed ? 14 : 15, allowed ? "allowed pair never computed" : "masked pair computed", h,
                          qtok[qr], ktok[kr]);
          }
        }
    return 0;
  }
};

}  // namespace

extern "C" {

// Ring mode: the whole sequence of S tokens split into P ranks with `cpr` chunks each
// (layout 0 contiguous, 1 zig-zag, 2 striped).  stats = {items, tiles, pairs}.
int sched_cover_ring(int B, int Hq, int Hkv, int S, int P, int layout, int cpr, int causal, int BM, int BN,
                     int64_t* stats, char* msg) {
  msg[0] = 0;
  Plan p{};
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.D = 128;
  p.causal = causal;
  p.mode = kModeRing;
  p.layout = layout;
  p.P = P;
  p.cpr = cpr;
  p.striped = layout == kLayoutStriped;
  p.strided = p.striped;
  p.nqc = p.nkc = P * cpr;
  p.C = S / (P * cpr);
  p.Sq = p.Skv = S;
  Walk w(p, S, BM, BN, msg);
  w.qtok.resize(S);
  w.ktok.resize(S);
  for (int r = 0; r < S; ++r) w.qtok[r] = w.ktok[r] = r;   // ring-mode buffers hold the sequence in order
  const int rc = w.run();
  stats[0] = w.items; stats[1] = w.tiles; stats[2] = w.pairs;
  return rc;
}

// Step mode: a query shard of nq chunks (global ids qid) against a held block of nk chunks
// (kid), C tokens each; with stripes = P > 0, one stripe qid[0] against one stripe kid[0].
int sched_cover_step(int B, int Hq, int Hkv, int C, int nq, const int* qid, int nk, const int* kid, int stripes,
                     int causal, int BM, int BN, int64_t* stats, char* msg) {
  msg[0] = 0;
  Plan p{};
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.D = 128;
  p.causal = causal;
  p.mode = kModeStep;
  p.layout = stripes > 0 ? kLayoutStriped : kLayoutContiguous;
  p.P = stripes > 0 ? stripes : 1;
  p.cpr = 1;
  p.striped = stripes > 0;
  p.strided = 0;
  p.C = C;
  p.nqc = nq;
  p.nkc = nk;
  for (int i = 0; i < nq; ++i) p.qid[i] = qid[i];
  for (int i = 0; i < nk; ++i) p.kid[i] = kid[i];
  // Q slots by decreasing chunk id, as the library orders them
  for (int i = 0; i < nq; ++i) p.qorder[i] = i;
  for (int i = 1; i < nq; ++i)
    for (int j = i; j > 0 && p.qid[p.qorder[j]] > p.qid[p.qorder[j - 1]]; --j) {
      const int t = p.qorder[j];
      p.qorder[j] = p.qorder[j - 1];
      p.qorder[j - 1] = t;
    }
  p.Sq = nq * C;
  p.Skv = nk * C;
  Walk w(p, 0, BM, BN, msg);
  w.qtok.resize(p.Sq);
  w.ktok.resize(p.Skv);
  for (int s = 0; s < nq; ++s)
    for (int x = 0; x < C; ++x) w.qtok[s * C + x] = stripes ? x * stripes + qid[0] : qid[s] * C + x;
  for (int s = 0; s < nk; ++s)
    for (int y = 0; y < C; ++y) w.ktok[s * C + y] = stripes ? y * stripes + kid[0] : kid[s] * C + y;
  const int rc = w.run();
  stats[0] = w.items; stats[1] = w.tiles; stats[2] = w.pairs;
  return rc;
}

}  // extern "C"
