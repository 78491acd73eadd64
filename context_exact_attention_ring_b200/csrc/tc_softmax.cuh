// The softmax warpgroups of the tensor-core ring kernels (attn_tc.cu: one CTA
// per SM; attn_tc_pair.cu: a CTA pair per TPC), and the epilogue they run at
// the end of every work item.
//
// Each of the two warpgroups owns one 128-row query tile of the item; thread
// t owns row t.  For every K/V tile of the walk it reads the 128 scores of
// its row from tensor memory, masks them on partial tiles, and folds them
// into the running (m, l, O) of "Lesson 8: Context Parallelism", section 3,
// in log2 units x = s * scale * log2(e):
//   m_new = max(m, max_j x_j); the base m is only moved when m_new exceeds it
//   by more than 8 (a factor 256), in which case l and the O row are rescaled
//   by 2^(m - m_new) in place; p_j = 2^(x_j - m) is written as bf16 over the
//   first 64 columns of the scores for the PV product and l += sum p_j in
//   fp32.  lt is l corrected by the bf16 rounding of each tile's largest
//   weight (the error that does not average out when one key dominates).
//   Using a stale base is exact: l, lt and O share it.
// At the end of an item: out = O / lt, lse = (m + log2 l) * ln 2 (ring mode),
// or the block result folded into the caller's state (step mode).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ptx.cuh"
#include "ring_sched.h"

namespace ra {

namespace tc {
constexpr int BM = 128, BN = 128;
constexpr int THREADS = 384;
constexpr int SLAB = 128 * 64 * 2;   // one 128-row x 64-column bf16 box (16 KB, 128-byte swizzle)
constexpr float LAZY = 8.f;
constexpr uint32_t TMEM_COLS = 512;
constexpr int REG_LOW = 96, REG_HIGH = 184;
constexpr int REG_NEED = (128 * REG_LOW + 256 * REG_HIGH + THREADS - 1) / THREADS;   // per thread at launch
constexpr int kEpiFloats = 32 * 16;   // a softmax warp's staging tile: 32 rows x 16 columns
}  // namespace tc

struct TcParams {
  Plan p;
  ItemSpace space;
  TcArgs a;
  float scale_log2;
};

__device__ __forceinline__ float mergew_exp(float x) { return expf(x); }

// Barriers the role uses (shared::cta addresses, each an array of two, one per
// query tile): s_full (the MMA issuer: the scores of tile j are in tensor
// memory), o_final (the last PV product of the item is complete) and the
// p_full arrival (this group's weights are in tensor memory and the O row is
// rescaled).  kPair: the p_full barriers live in the leader CTA and count one
// arrival per warp of both CTAs (p_full_arrive is their shared::cluster
// address); otherwise every thread arrives on the local barrier.  Items are
// dealt to CTA (or pair) item0 of `stride` by turn_item, in alternating wave
// order for one CTA per SM only; `cta` picks the pair item's tiles.  `epi` is this warp's staging tile for the step-mode epilogue
// (kEpiFloats floats).
template <int D, bool kPair>
__device__ __forceinline__ void tc_softmax_role(const TcParams& prm, uint32_t tmem, int warp, int lane,
                                                uint32_t s_full, uint32_t p_full_arrive, uint32_t o_final,
                                                volatile int* abort_flag, int item0, int stride, int cta,
                                                float* epi) {
  using namespace tc;
  const Plan& p = prm.p;
  const ItemSpace& space = prm.space;
  unsigned int* err = prm.a.err;
  const int i = (warp - 4) >> 2;                 // query tile of this group
  const int wi = warp & 3;                       // tensor-memory lane quarter
  const int row = wi * 32 + lane;                // row of the tile owned by this thread
  const uint32_t lane_off = (uint32_t)(wi * 32) << 16;
  const uint32_t tS = tmem + lane_off + i * 128;
  const uint32_t tO = tmem + lane_off + 256 + i * D;
  const float sl2 = prm.scale_log2;
  const int tpc = cdiv(p.C, BN);
  uint32_t tiles_done = 0, items_with_tiles = 0;
  unsigned long long cnt_full = 0, cnt_part = 0;
  bool ok = true;

  // items dealt as in the role's kernel: in alternating wave order on one CTA per SM, in
  // the same order every wave on CTA pairs (measured faster for each)
  for (int w = 0, L = turn_item(0, item0, stride, space.count, !kPair); L >= 0 && ok;
       L = turn_item(++w, item0, stride, space.count, !kPair)) {
    const Item it = kPair ? item_pair_at(p, space, BM, L, cta) : item_at(p, space, BM, L);
    const int nrows = it.nrows[i];
    const int q0 = it.qpos0[i], q1 = it.qpos0[i] + nrows - 1;
    const int qpos = it.qpos0[i] + row;
    const int rank = p.mode == kModeRing ? chunk_owner(p, it.qslot) : 0;
    // l: fp32 sum of p (gives lse); lt: l corrected by the bf16 rounding of
    // each tile's largest weight (normalises O; see exp_pass)
    float m_run = -CUDART_INF_F, m_max = -CUDART_INF_F, l = 0.f, lt = 0.f;
    KvIter iter;
    kv_begin(p, it.qslot, iter);
    KvTile t;
    uint32_t j = 0;
    while (kv_next(p, it.qhi, BN, tpc, iter, t)) {
      if (prm.a.counters && row == 0 && nrows > 0) {
        const int cls = tile_class(p.causal, q0, q1, t.pos0, t.pos0 + t.nvalid - 1);
        if (cls == 0) ++cnt_full;
        if (cls == 1) ++cnt_part;
        if (cls != 2 && t.first_in_chunk && it.tile_in_chunk[i] == 0 && p.mode == kModeRing)
          atomicAdd(prm.a.counters + 2 + rank, 1ull);
      }
      __syncwarp();
      const bool got = mbar_wait(s_full + 8 * i, (tiles_done + j) & 1u, abort_flag, kWaitSFull, err);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BN];
      {
        // the row's 128 scores in one load (measured 0.7% faster than four 32-column loads)
        uint32_t r[BN];
        tmem_ld128(tS, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < BN; ++e) s[e] = __uint_as_float(r[e]);
      }
      const bool need_mask = (p.causal && t.pos0 + BN - 1 > q0) || t.nvalid < BN;
      if (need_mask) {
        const int lim_causal = p.causal ? qpos - t.pos0 : BN;   // keys with index <= lim are allowed
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= t.nvalid || c > lim_causal) s[c] = -CUDART_INF_F;
      }
      // Row max first, then the exponentials against the (lazily moved) base.
      const uint64_t sl2x2 = pack2(sl2, sl2);
      float alpha = 1.f, rs = 0.f, rt = 0.f, mxs, mx_raw;
      auto exp_pass = [&](float base) {
        const uint64_t nbase2 = pack2(-base, -base);
        uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a0 = s[c * 32 + 2 * e], a1 = s[c * 32 + 2 * e + 1];
            float x0, x1;
            unpack2(ffma2(pack2(a0, a1), sl2x2, nbase2), x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            rs2[e & 3] = fadd2(rs2[e & 3], pack2(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);
        }
        rs = hsum2(fadd2(fadd2(rs2[0], rs2[1]), fadd2(rs2[2], rs2[3])));
        // The PV product uses bf16(p).  When one key dominates a row, the rounding of
        // its weight is the one error that does not average out; folding it into
        // the normaliser makes the weights applied to V sum to one in that case.
        const float pm = ex2(fmaf(mx_raw, sl2, -base));
        rt = rs + (__uint_as_float(pack_bf16x2(pm, pm) & 0xffff0000u) - pm);
      };
      auto row_max = [&]() -> float {
        float mq[4];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const float* sc = s + ch * 32;
          float x = fmax3(sc[0], sc[1], sc[2]);
#pragma unroll
          for (int e = 3; e < 31; e += 2) x = fmax3(x, sc[e], sc[e + 1]);
          mq[ch] = fmaxf(x, sc[31]);
        }
        return fmax3(fmaxf(mq[0], mq[1]), mq[2], mq[3]);
      };
      // (exp_pass stores to tensor memory with warp-collective instructions; it
      // runs unconditionally, by the whole warp)
      mx_raw = row_max();
      mxs = mx_raw * sl2;
      if (mxs > m_run + LAZY) {   // always for a row without a base yet (m_run = -inf)
        alpha = (m_run == -CUDART_INF_F) ? 0.f : ex2(m_run - mxs);
        m_run = mxs;
      }
      exp_pass(m_run == -CUDART_INF_F ? 0.f : m_run);
      m_max = fmaxf(m_max, mxs);
      l = l * alpha + rs;
      lt = lt * alpha + rt;
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(tO + c * 32, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      if constexpr (kPair) {
        // one arrival per warp, on the leader's barrier: every lane's tensor-memory stores are
        // complete (tcgen05.wait::st above), so no cluster-scope fence is needed
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(p_full_arrive + 8 * i);
      } else {
        mbar_arrive(p_full_arrive + 8 * i);
      }
      ++j;
    }
    if (!ok) break;
    tiles_done += j;
    if (j == 0) continue;   // step mode: nothing of this block is visible to these rows

    const bool fin = mbar_wait(o_final + 8 * i, items_with_tiles & 1u, abort_flag, kWaitOFinal, err);
    if (!__all_sync(0xffffffffu, fin)) {
      ok = false;
      break;
    }
    ++items_with_tiles;
    tc_fence_after();
    const bool active = row < nrows;
    const int qr = p.strided ? (it.qoff[i] + row) * p.P + it.qslot : it.qrow0[i] + row;
    const int h = it.h[i];
    const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
    if (p.mode == kModeRing) {
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(prm.a.out) + (((size_t)it.b * p.Sq + qr) * p.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_wait_ld();
        if (active) {
          uint4 w[4];
          uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            wp[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = w[e];
        }
        __syncwarp();
      }
      if (active)
        prm.a.lse[((size_t)it.b * p.Hq + h) * p.Sq + qr] =
            l > 0.f ? (m_run + log2f(l)) * 0.6931471805599453f : -CUDART_INF_F;
    } else {
      // fold this block into the caller's state (natural-log units, exact max).  The call
      // before this one on the stream may still be writing the same state rows (step calls
      // are launched to overlap their predecessor's tail): wait for it to complete first.
      grid_dependency_wait();
      const size_t si = ((size_t)it.b * p.Hq + h) * p.Sq + (active ? qr : it.qrow0[i]);
      float m_old = -CUDART_INF_F, l_old = 0.f;
      if (active) {
        m_old = prm.a.m[si];
        l_old = prm.a.l[si];
      }
      const bool live = l > 0.f;
      const float m_b = live ? m_max * 0.6931471805599453f : -CUDART_INF_F;
      const float l_b = live ? l * ex2(m_run - m_max) : 0.f;
      float w_old = 1.f, w_blk = 0.f, m_new = m_old, l_new = l_old;
      if (live) {
        const float mn = fmaxf(m_old, m_b);
        const float a = (m_old == -CUDART_INF_F) ? 0.f : mergew_exp(m_old - mn) * l_old;
        const float cb = mergew_exp(m_b - mn) * l_b;
        m_new = mn;
        l_new = a + cb;
        w_old = a / l_new;
        w_blk = cb / l_new;
      }
      // The stored O rows are read and written through this warp's 32 x 16 staging tile in shared
      // memory, 16 columns at a time: four lanes move a row's 64 bytes, so a warp instruction
      // touches 8 rows instead of one row per lane (32 lines), and the loads of four chunks are
      // in flight while a chunk is combined.  Tile layout: row r, float4 q at float4
      // index r*4 + (q ^ ((r >> 1) & 3)), conflict-free for both access patterns.
      const float wb = w_blk * inv_l;
      const int rbase = wi * 32;                     // first tile row of this warp
      const int crow = lane >> 2, cq = lane & 3;     // cooperative pattern: rows crow + 8k, float4 cq
      float4* const tile = reinterpret_cast<float4*>(epi);
      auto tidx = [](int r, int q) { return r * 4 + (q ^ ((r >> 1) & 3)); };
      auto orow = [&](int r) {   // global O row of tile row rbase + r (step mode: rows not strided)
        return prm.a.O + (((size_t)it.b * p.Sq + it.qrow0[i] + rbase + r) * p.Hq + h) * D;
      };
      // four chunks of loads in flight: chunk c + 4 is requested as soon as chunk c is staged
      constexpr int NCH = D / 16, DEPTH = 4;
      float4 ld[DEPTH][4];
      auto load_chunk = [&](int c, float4 (&dst)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = crow + 8 * k;
          dst[k] = rbase + r < nrows ? reinterpret_cast<const float4*>(orow(r) + c * 16)[cq]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      };
#pragma unroll
      for (int c = 0; c < DEPTH; ++c) load_chunk(c, ld[c]);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
#pragma unroll
        for (int k = 0; k < 4; ++k) tile[tidx(crow + 8 * k, cq)] = ld[c % DEPTH][k];
        if (c + DEPTH < NCH) load_chunk(c + DEPTH, ld[c % DEPTH]);
        uint32_t r16[16];
        tmem_ld16(tO + c * 16, r16);
        tmem_wait_ld();
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // this lane's own row
          float4 o = tile[tidx(lane, q)];
          o.x = w_old * o.x + wb * __uint_as_float(r16[4 * q + 0]);
          o.y = w_old * o.y + wb * __uint_as_float(r16[4 * q + 1]);
          o.z = w_old * o.z + wb * __uint_as_float(r16[4 * q + 2]);
          o.w = w_old * o.w + wb * __uint_as_float(r16[4 * q + 3]);
          tile[tidx(lane, q)] = o;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = crow + 8 * k;
          if (rbase + r < nrows) reinterpret_cast<float4*>(orow(r) + c * 16)[cq] = tile[tidx(r, cq)];
        }
        __syncwarp();
      }
      if (active) {
        prm.a.m[si] = m_new;
        prm.a.l[si] = l_new;
      }
    }
    tc_fence_before();
  }
  if (prm.a.counters && row == 0) {
    atomicAdd(prm.a.counters + 0, cnt_full);
    atomicAdd(prm.a.counters + 1, cnt_part);
  }
}

}  // namespace ra
