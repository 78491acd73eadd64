// Host-side walk of the schedulers the attention kernels use to pick their
// work: the ring scheduler (context_exact_attention_ring_b200/csrc/
// ring_sched.h) and the backward's items and steps (csrc/bwd_sched.h).
// Built with g++ by tests/test_sched_cover.py; no GPU involved.
//
// For one problem it runs through every work item the way a kernel does and
// records which (query token, key token) pairs of which (batch, query head)
// get computed:
//   forward        item_at over all items; for both query tiles of an item,
//                  the K/V tiles of kv_next, with the element mask "key
//                  position <= query position" and "column < valid keys";
//   forward pair   item_pair_at over all items of the CTA-pair kernel, for
//                  both CTAs and both tiles of each, walking the K/V tiles of
//                  the item's shared qhi with the same element mask (both
//                  CTAs must agree on the item's chunk, batch, kv head and
//                  qhi, so they walk the same tiles);
//   backward K/V   kv_item over all items; the query steps of qstep_next,
//                  where key row r sees query column j iff k0 + r <= q0 + j
//                  and j is a valid query of the step;
//   backward Q     q_item over all items; the K/V tiles of kv_next with
//                  128-key steps and the forward's element mask.
// It then checks, against the true global token positions of the split:
//   * every pair the causal rule of "Lesson 8: Context Parallelism",
//     section 4, allows (all pairs when not causal) is computed exactly once,
//     and no other pair is;
//   * every output row (forward: out and lse of a query row; backward K/V:
//     dK, dV of a key row; backward Q: dQ of a query row) is owned by exactly
//     one item, so no two CTAs write the same row;
//   * every buffer row, head and batch index stays inside its tensor, and the
//     kv head of every computed pair is the GQA group of its query head;
//   * the step count the MMA warp expects (kv_count, qstep_count) equals the
//     number of steps the producer walks, so neither waits for a step the
//     other never issues.
// Returns 0 if every check holds, else a code naming the first failure (and
// fills `msg`).
#include <cstdint>
#include <cstdio>
#include <vector>

#include "../context_exact_attention_ring_b200/csrc/bwd_sched.h"
#include "../context_exact_attention_ring_b200/csrc/ring_sched.h"

using namespace ra;

namespace {

enum { kForward = 0, kBackwardKv = 1, kBackwardQ = 2, kForwardPair = 3 };

struct Problem {
  Plan p;
  std::vector<int> qtok, ktok;   // global token of each Q / K-V buffer row
};

struct Walk {
  const Plan& p;
  const Problem& pr;
  std::vector<uint8_t> cover;    // [B][Hq][Sq][Skv] (buffer rows)
  std::vector<uint8_t> owner;    // output rows: [B][Hq][Sq] or [B][Hkv][Skv]
  int64_t items = 0, steps = 0, pairs = 0;
  char* msg;

  Walk(const Problem& x, char* m) : p(x.p), pr(x), msg(m) {
    cover.assign((size_t)p.B * p.Hq * p.Sq * p.Skv, 0);
  }

  int fail(int code, const char* what, int a = 0, int b = 0, int c = 0) {
    snprintf(msg, 256, "%s (%d, %d, %d)", what, a, b, c);
    return code;
  }

  // one computed (query row, key row) pair of query head h
  int mark(int b, int h, int qrow, int krow, int L) {
    if (qrow < 0 || qrow >= p.Sq) return fail(5, "query buffer row out of range", L, qrow);
    if (krow < 0 || krow >= p.Skv) return fail(9, "key buffer row out of range", L, krow);
    uint8_t& x = cover[(((size_t)b * p.Hq + h) * p.Sq + qrow) * p.Skv + krow];
    if (++x > 1) return fail(11, "pair computed twice", L, qrow, krow);
    ++pairs;
    return 0;
  }

  int own(size_t idx, int L, int row) {
    if (idx >= owner.size()) return fail(16, "output row out of range", L, row);
    if (++owner[idx] != 1) return fail(7, "output row owned by two items", L, row);
    return 0;
  }

  int forward(int BM, int BN) {
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
          if (!p.strided && row != it.qrow0[i] + r) return fail(6, "qrow0 disagrees with buf_row", L, i, r);
          if (int e = own(((size_t)it.b * p.Hq + it.h[i]) * p.Sq + row, L, row)) return e;
        }
      }
      KvIter iter;
      kv_begin(p, it.qslot, iter);
      KvTile t;
      int n = 0;
      while (kv_next(p, it.qhi, BN, tpc, iter, t)) {
        ++n;
        ++steps;
        if (t.slot < 0 || t.slot >= p.nkc || t.nvalid < 1 || t.nvalid > BN || t.k0 + t.nvalid > p.C)
          return fail(8, "kv tile out of range", L, t.slot, t.k0);
        for (int i = 0; i < 2; ++i)
          for (int r = 0; r < it.nrows[i]; ++r) {
            const int qpos = it.qpos0[i] + r;
            for (int c = 0; c < t.nvalid; ++c) {
              if (p.causal && t.pos0 + c > qpos) continue;             // the kernel's element mask
              const int krow = buf_row(p, t.slot, t.k0 + c);
              if (!p.strided && krow != t.row0 + c) return fail(10, "row0 disagrees with buf_row", L, c);
              if (int e = mark(it.b, it.h[i], buf_row(p, it.qslot, it.qoff[i] + r), krow, L)) return e;
            }
          }
      }
      if (n != kv_count(p, it.qslot, it.qhi, BN, tpc)) return fail(12, "kv_count disagrees with kv_next", L, n);
    }
    return 0;
  }

  int forward_pair(int BM, int BN) {
    owner.assign((size_t)p.B * p.Hq * p.Sq, 0);
    const ItemSpace sp = item_space_pair(p, BM);
    const int tpc = cdiv(p.C, BN);
    const int G = p.Hq / p.Hkv;
    for (int L = 0; L < sp.count; ++L) {
      Item its[2] = {item_pair_at(p, sp, BM, L, 0), item_pair_at(p, sp, BM, L, 1)};
      ++items;
      if (its[0].b != its[1].b || its[0].hkv != its[1].hkv || its[0].qslot != its[1].qslot ||
          its[0].qhi != its[1].qhi)
        return fail(17, "the two CTAs of a pair disagree on the item", L);
      const Item& it0 = its[0];
      if (it0.b < 0 || it0.b >= p.B || it0.hkv < 0 || it0.hkv >= p.Hkv) return fail(1, "item batch/kv head out of range", L);
      if (it0.qslot < 0 || it0.qslot >= p.nqc) return fail(2, "item query chunk out of range", L, it0.qslot);
      if (it0.qhi < 0) return fail(4, "item without a valid query row", L);
      for (int c = 0; c < 2; ++c) {
        const Item& it = its[c];
        for (int i = 0; i < 2; ++i) {
          if (it.h[i] < 0 || it.h[i] >= p.Hq || it.h[i] / G != it.hkv)
            return fail(3, "query head not in the kv group", L, c, i);
          if (it.nrows[i] < 0 || it.nrows[i] > BM || (it.nrows[i] > 0 && it.qoff[i] + it.nrows[i] > p.C))
            return fail(4, "query tile rows out of range", L, i, it.nrows[i]);
          if (it.nrows[i] > 0 && it.qpos0[i] + it.nrows[i] - 1 > it.qhi) return fail(4, "tile beyond qhi", L, c, i);
          for (int r = 0; r < it.nrows[i]; ++r) {
            const int row = buf_row(p, it.qslot, it.qoff[i] + r);
            if (!p.strided && row != it.qrow0[i] + r) return fail(6, "qrow0 disagrees with buf_row", L, i, r);
            if (int e = own(((size_t)it.b * p.Hq + it.h[i]) * p.Sq + row, L, row)) return e;
          }
        }
      }
      KvIter iter;
      kv_begin(p, it0.qslot, iter);
      KvTile t;
      int n = 0;
      while (kv_next(p, it0.qhi, BN, tpc, iter, t)) {
        ++n;
        ++steps;
        if (t.slot < 0 || t.slot >= p.nkc || t.nvalid < 1 || t.nvalid > BN || t.k0 + t.nvalid > p.C)
          return fail(8, "kv tile out of range", L, t.slot, t.k0);
        for (int c = 0; c < 2; ++c)
          for (int i = 0; i < 2; ++i)
            for (int r = 0; r < its[c].nrows[i]; ++r) {
              const int qpos = its[c].qpos0[i] + r;
              for (int k = 0; k < t.nvalid; ++k) {
                if (p.causal && t.pos0 + k > qpos) continue;           // the kernel's element mask
                const int krow = buf_row(p, t.slot, t.k0 + k);
                if (!p.strided && krow != t.row0 + k) return fail(10, "row0 disagrees with buf_row", L, k);
                if (int e = mark(its[c].b, its[c].h[i], buf_row(p, its[c].qslot, its[c].qoff[i] + r), krow, L))
                  return e;
              }
            }
      }
      if (n != kv_count(p, it0.qslot, it0.qhi, BN, tpc)) return fail(12, "kv_count disagrees with kv_next", L, n);
    }
    return 0;
  }

  int backward_kv() {
    owner.assign((size_t)p.B * p.Hkv * p.Skv, 0);
    const int G = p.Hq / p.Hkv;
    const long long n_items = (long long)p.B * p.Hkv * p.nkc * cdiv(p.C, tb::BR);   // as the launcher counts
    for (int L = 0; L < n_items; ++L) {
      const KvItem it = kv_item(p, L);
      ++items;
      if (it.b < 0 || it.b >= p.B || it.g < 0 || it.g >= p.Hkv || it.ks < 0 || it.ks >= p.nkc)
        return fail(1, "item batch/kv head/chunk out of range", L);
      if (it.nk < 1 || it.nk > tb::BR || it.k_off + it.nk > p.C) return fail(4, "key tile rows out of range", L, it.nk);
      for (int r = 0; r < it.nk; ++r) {
        const int krow = buf_row(p, it.ks, it.k_off + r);
        if (int e = own(((size_t)it.b * p.Hkv + it.g) * p.Skv + krow, L, krow)) return e;
      }
      QStepIter si{0, 0, 0};
      QStep st;
      int n = 0;
      while (qstep_next(p, it, si, st)) {
        ++n;
        ++steps;
        if (st.h < it.g * G || st.h >= (it.g + 1) * G) return fail(3, "step head not in the kv group", L, st.h);
        if (st.qs < 0 || st.qs >= p.nqc || st.nq < 1 || st.nq > tb::BS || st.q_off + st.nq > p.C)
          return fail(8, "query step out of range", L, st.qs, st.q_off);
        if (st.q0 != q_pos_base(p, st.qs) + st.q_off) return fail(10, "step q0 disagrees with its rows", L, st.q0);
        if (st.k0 != kv_pos_base(p, q_gid(p, st.qs), it.ks) + it.k_off)
          return fail(10, "step k0 disagrees with its rows", L, st.k0);
        for (int r = 0; r < it.nk; ++r)
          for (int j = 0; j < st.nq; ++j) {
            if (p.causal && st.k0 + r > st.q0 + j) continue;           // the kernel's element mask
            if (int e = mark(it.b, st.h, buf_row(p, st.qs, st.q_off + j), buf_row(p, it.ks, it.k_off + r), L))
              return e;
          }
      }
      if (n != qstep_count(p, it)) return fail(12, "qstep_count disagrees with qstep_next", L, n);
    }
    return 0;
  }

  int backward_q() {
    owner.assign((size_t)p.B * p.Hq * p.Sq, 0);
    const int G = p.Hq / p.Hkv, SR = tb::BR, tpc = cdiv(p.C, SR);
    const long long n_items = (long long)p.B * p.Hq * p.nqc * cdiv(p.C, tb::BR);    // as the launcher counts
    for (int L = 0; L < n_items; ++L) {
      const QItem it = q_item(p, L);
      ++items;
      if (it.b < 0 || it.b >= p.B || it.h < 0 || it.h >= p.Hq || it.g != it.h / G || it.qs < 0 || it.qs >= p.nqc)
        return fail(1, "item batch/head/chunk out of range", L);
      if (it.nq < 1 || it.nq > tb::BR || it.q_off + it.nq > p.C) return fail(4, "query tile rows out of range", L, it.nq);
      if (it.q0 != q_pos_base(p, it.qs) + it.q_off) return fail(10, "item q0 disagrees with its rows", L, it.q0);
      for (int r = 0; r < it.nq; ++r) {
        const int qrow = buf_row(p, it.qs, it.q_off + r);
        if (int e = own(((size_t)it.b * p.Hq + it.h) * p.Sq + qrow, L, qrow)) return e;
      }
      KvIter ki;
      kv_begin(p, it.qs, ki);
      KvTile t;
      int n = 0;
      while (kv_next(p, it.q0 + it.nq - 1, SR, tpc, ki, t)) {
        ++n;
        ++steps;
        if (t.slot < 0 || t.slot >= p.nkc || t.nvalid < 1 || t.nvalid > SR || t.k0 + t.nvalid > p.C)
          return fail(8, "kv tile out of range", L, t.slot, t.k0);
        for (int r = 0; r < it.nq; ++r)
          for (int j = 0; j < t.nvalid; ++j) {
            if (p.causal && t.pos0 + j > it.q0 + r) continue;          // the kernel's element mask
            if (int e = mark(it.b, it.h, buf_row(p, it.qs, it.q_off + r), buf_row(p, t.slot, t.k0 + j), L)) return e;
          }
      }
      if (n != kv_count(p, it.qs, it.q0 + it.nq - 1, SR, tpc)) return fail(12, "kv_count disagrees with kv_next", L, n);
    }
    return 0;
  }

  // every allowed pair once, no other pair; every output row owned once
  int finish() {
    for (size_t i = 0; i < owner.size(); ++i)
      if (owner[i] != 1) return fail(13, "output row owned by no item", (int)i);
    for (int b = 0; b < p.B; ++b)
      for (int h = 0; h < p.Hq; ++h)
        for (int qr = 0; qr < p.Sq; ++qr)
          for (int kr = 0; kr < p.Skv; ++kr) {
            const bool allowed = !p.causal || pr.ktok[kr] <= pr.qtok[qr];
            const uint8_t x = cover[(((size_t)b * p.Hq + h) * p.Sq + qr) * p.Skv + kr];
            if (x != (allowed ? 1 : 0))
              return fail(allowed ? 14 : 15, allowed ? "allowed pair never computed" : "masked pair computed", h,
                          pr.qtok[qr], pr.ktok[kr]);
          }
    return 0;
  }
};

int run(const Problem& pr, int which, int BM, int BN, int64_t* stats, char* msg) {
  msg[0] = 0;
  Walk w(pr, msg);
  int rc = which == kForward       ? w.forward(BM, BN)
           : which == kForwardPair ? w.forward_pair(BM, BN)
           : which == kBackwardKv  ? w.backward_kv()
                                   : w.backward_q();
  if (rc == 0) rc = w.finish();
  stats[0] = w.items;
  stats[1] = w.steps;
  stats[2] = w.pairs;
  return rc;
}

}  // namespace

extern "C" {

// Ring mode: the whole sequence of S tokens split into P ranks with `cpr` chunks each
// (layout 0 contiguous, 1 zig-zag, 2 striped).  which: 0 forward (BM x BN tiles),
// 1 backward K/V-major, 2 backward Q-major, 3 forward of the CTA-pair kernel.
// stats = {items, steps, pairs}.
int sched_cover_ring(int B, int Hq, int Hkv, int S, int P, int layout, int cpr, int causal, int which, int BM,
                     int BN, int64_t* stats, char* msg) {
  Problem pr;
  Plan& p = pr.p;
  p = Plan{};
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
  pr.qtok.resize(S);
  pr.ktok.resize(S);
  for (int r = 0; r < S; ++r) pr.qtok[r] = pr.ktok[r] = r;   // ring-mode buffers hold the sequence in order
  return run(pr, which, BM, BN, stats, msg);
}

// The dealing of work items to persistent CTAs (turn_item, used by the forward and backward kernels): every item of
// [0, items) goes to exactly one turn of one CTA, each CTA's turns ascend through the waves,
// and a CTA that has no item in some turn has none in any later turn (the kernels stop at the
// first -1).  Returns 0, or a code naming the first failure.
int sched_cover_turns(int items, int grid, int snake, char* msg) {
  msg[0] = 0;
  std::vector<int> seen((size_t)items, 0);
  for (int cta = 0; cta < grid; ++cta) {
    int last = -1;
    bool ended = false;
    for (int w = 0; w <= items / grid + 1; ++w) {
      const int L = turn_item(w, cta, grid, items, snake != 0);
      if (L < 0) {
        ended = true;
        continue;
      }
      if (ended) return snprintf(msg, 256, "cta %d gets item %d after a turn with none", cta, L), 1;
      if (L >= items) return snprintf(msg, 256, "cta %d gets item %d of %d", cta, L, items), 2;
      if (L <= last) return snprintf(msg, 256, "cta %d: item %d after %d", cta, L, last), 3;
      if (L / grid != w) return snprintf(msg, 256, "cta %d: item %d outside wave %d", cta, L, w), 4;
      last = L;
      ++seen[(size_t)L];
    }
  }
  for (int L = 0; L < items; ++L)
    if (seen[(size_t)L] != 1) return snprintf(msg, 256, "item %d dealt %d times", L, seen[(size_t)L]), 5;
  return 0;
}

// The item a CTA takes at its w-th turn (-1 when it has none), as the kernels deal them.
int sched_turn_item(int w, int cta, int grid, int items, int snake) { return turn_item(w, cta, grid, items, snake != 0); }

// Step mode: a query shard of nq chunks (global ids qid) against a held block of nk chunks
// (kid), C tokens each; with stripes = P > 0, one stripe qid[0] against one stripe kid[0].
int sched_cover_step(int B, int Hq, int Hkv, int C, int nq, const int* qid, int nk, const int* kid, int stripes,
                     int causal, int which, int BM, int BN, int64_t* stats, char* msg) {
  Problem pr;
  Plan& p = pr.p;
  p = Plan{};
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
  pr.qtok.resize(p.Sq);
  pr.ktok.resize(p.Skv);
  for (int s = 0; s < nq; ++s)
    for (int x = 0; x < C; ++x) pr.qtok[s * C + x] = stripes ? x * stripes + qid[0] : qid[s] * C + x;
  for (int s = 0; s < nk; ++s)
    for (int y = 0; y < C; ++y) pr.ktok[s * C + y] = stripes ? y * stripes + kid[0] : kid[s] * C + y;
  return run(pr, which, BM, BN, stats, msg);
}

}  // extern "C"
