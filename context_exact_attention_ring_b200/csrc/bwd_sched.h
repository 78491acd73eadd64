// Work items and steps of the tensor-core backward (attn_bwd_tc.cu), kept in a
// header of their own so that the host can walk them as the kernel does.
//
// K/V-major launch: an item is a 128-key tile of one kv head; its steps are
// the 64-row query tiles (of every query head of the group) the block meets
// as it travels round the ring ("Lesson 8: Context Parallelism", section 2:
// the block of rank s meets every rank once), skipping under the causal rule
// ("Lesson 8", section 4) the tiles whose every query precedes every key.
// Inside one GPU the tiles are walked in buffer order, not hop by hop (see
// qstep_next).  Q-major launch: an item is a 128-row query tile of one head,
// longest work first; its steps are the K/V tiles of the ring scheduler
// (ring_sched.h).
#pragma once
#include "ring_sched.h"

namespace ra {

namespace tb {
constexpr int BR = 128;                 // rows of an item tile (and of T1/T2)
constexpr int BS = 64;                  // rows of a K/V-major step (query rows)
}  // namespace tb

// ---------------------------------------------------------------- work items
// K/V-major item: one 128-key tile of chunk slot ks, kv head g, batch b.
// Items run (batch, kv head) by (batch, kv head); inside one, the key tiles
// run in buffer order, and in the reverse order for every other one, counted
// from the last (which thus runs forward).  In ring mode a tile's walk gets
// shorter with its position, so the items dealt out at one time have nearly
// equal walks also where one (batch, kv head) ends and the next begins: the
// short walks at the end of one meet the short walks at the start of the
// next, and the launch ends with short walks.
struct KvItem {
  int b, g, ks, k_off, nk;
};
RA_HD KvItem kv_item(const Plan& p, int L) {
  const int tpk = cdiv(p.C, tb::BR);
  const int per_bg = p.nkc * tpk;
  KvItem it;
  const int bg = L / per_bg;
  int r = L - bg * per_bg;
  if ((p.B * p.Hkv - 1 - bg) & 1) r = per_bg - 1 - r;
  it.b = bg / p.Hkv;
  it.g = bg - it.b * p.Hkv;
  it.ks = r / tpk;
  it.k_off = (r - it.ks * tpk) * tb::BR;
  it.nk = imin(tb::BR, p.C - it.k_off);
  return it;
}

// One step of a K/V-major item: a 64-row query tile of head h in chunk qs.
struct QStep {
  int h, qs, q_off, nq, q0, k0;
};
struct QStepIter {
  int h, n, qt;
};
// The steps of every item follow one path: the Q buffer's chunks in buffer
// order (ring mode: the sequence in order), their 64-row tiles in order, and
// the group's query heads innermost; the causal rule skips the tiles whose
// every query precedes every key.  Items dealt out together hold neighbouring
// key tiles, so at any time their CTAs are at nearby points of the same path
// and read the same Q/dO tiles a short time apart.  (Walking each block in its
// ring order, from its own rank, puts the CTAs of different ranks' blocks on
// different parts of Q at once; the sums are the same either way.)
RA_HD bool qstep_next(const Plan& p, const KvItem& it, QStepIter& s, QStep& out) {
  const int G = p.Hq / p.Hkv, tpq = cdiv(p.C, tb::BS);
  while (s.n < p.nqc) {
    if (s.qt >= tpq) {
      s.qt = 0;
      s.h = 0;
      ++s.n;
      continue;
    }
    const int qs = s.n;
    const int qb = q_pos_base(p, qs);
    const int k0 = kv_pos_base(p, q_gid(p, qs), it.ks) + it.k_off;
    if (s.qt == 0 && s.h == 0 && p.causal) {
      // tiles whose last query precedes the first key are never met: start at the first one that is
      if (qb + p.C - 1 < k0) {
        s.qt = tpq;
        continue;
      }
      s.qt = imax(0, (k0 - qb + 1 + tb::BS - 1) / tb::BS - 1);
    }
    const int q_off = s.qt * tb::BS;
    const int nq = imin(tb::BS, p.C - q_off);
    const int q0 = qb + q_off;
    if (p.causal && k0 > q0 + nq - 1) {   // every key after every query of the tile
      ++s.qt;
      s.h = 0;
      continue;
    }
    out.h = it.g * G + s.h;
    out.qs = qs;
    out.q_off = q_off;
    out.nq = nq;
    out.q0 = q0;
    out.k0 = k0;
    if (++s.h == G) {
      s.h = 0;
      ++s.qt;
    }
    return true;
  }
  return false;
}

RA_HD int qstep_count(const Plan& p, const KvItem& it) {
  const int G = p.Hq / p.Hkv, tpq = cdiv(p.C, tb::BS);
  int n = 0;
  for (int qs = 0; qs < p.nqc; ++qs) {
    const int qb = q_pos_base(p, qs);
    const int k0 = kv_pos_base(p, q_gid(p, qs), it.ks) + it.k_off;
    if (!p.causal) {
      n += tpq;
    } else if (qb + p.C - 1 >= k0) {
      int t = imax(0, (k0 - qb + 1 + tb::BS - 1) / tb::BS - 1);
      if (qb + imin((t + 1) * tb::BS, p.C) - 1 < k0) ++t;   // (defensive: the formula already lands here)
      n += tpq - t;
    }
  }
  return n * G;
}

// Q-major item: one 128-row query tile of head h (longest work first).
struct QItem {
  int b, h, g, qs, q_off, nq, q0;
};
RA_HD QItem q_item(const Plan& p, int L) {
  const int tpq = cdiv(p.C, tb::BR);
  const int per_bh = p.nqc * tpq;
  QItem it;
  const int bh = L / per_bh, r = L - bh * per_bh;
  it.b = bh / p.Hq;
  it.h = bh - it.b * p.Hq;
  it.g = it.h / (p.Hq / p.Hkv);
  const int k = r / tpq;
  it.qs = q_slot_by_rank(p, k);
  it.q_off = (tpq - 1 - (r - k * tpq)) * tb::BR;
  it.nq = imin(tb::BR, p.C - it.q_off);
  it.q0 = q_pos_base(p, it.qs) + it.q_off;
  return it;
}

}  // namespace ra
