// Backward of ring attention on the tensor cores (tcgen05, bf16 operands,
// fp32 accumulation in tensor memory).  The gradients are the calculus of the
// forward (the pages give no backward):
//   P = exp(scale * Q K^T - lse),  dP = dO V^T,  dS = P o (dP - delta),
//   dV = P^T dO,  dK = scale * dS^T Q,  dQ = scale * dS K,
// with P recomputed tile by tile from the forward's lse.  Two launches of one
// kernel template, neither with atomics:
//   kKvMajor = true   a work item is a 128-key K/V tile of one kv head; its
//                     steps are the 64-row query tiles (of every query head
//                     of the group) that the block meets as it travels round
//                     the ring ("Lesson 8: Context Parallelism", section 2),
//                     walked in buffer order with the heads innermost
//                     (bwd_sched.h):
//                       T1 = K Q^T, T2 = V dO^T      (SS: K, V, Q, dO in smem)
//                       P^T, dS^T from T1, T2          (two elementwise groups)
//                       dV += P^T dO, dK += dS^T Q    (TS: P^T, dS^T in tmem)
//   kKvMajor = false  a work item is a 128-row query tile of one head; its
//                     steps are the 128-key K/V tiles in the rank's ring order:
//                       T1 = Q K^T, T2 = dO V^T,  dS from T1, T2,
//                       dQ += dS K                    (TS)
// Every product has M = 128: the K/V-major launch's T1, T2 are 128 x 64 (64
// query rows per step), every other product 128 x 128 or 128 x D.  The
// shared-memory tiles are the forward's 128-byte-swizzled boxes, read K-major
// by the SS products and MN-major by the TS products.
//
// K/V-major: each step covers 64 query rows, so tensor memory holds two T1/T2
// pairs beside dK and dV, and the two elementwise groups ping-pong: while one
// turns its pair into P / dS, the tensor cores accumulate the other's and
// compute the next pair (issue order T(0) T(1) | TS(0) T(2) | TS(1) T(3) | ...),
// as the forward kernel does with its two query tiles.
// Q-major: each step covers 128 keys and both groups work on it (group g on the
// columns [64g, 64g + 64)).  Three 128-column regions rotate between S and dP
// beside dQ, so S(i+1), dP(i+1) and S(i+2) are computed around the
// elementwise pass of step i.
//
// Warp roles (12 warps): warp 0 TMA producer (the whole warp also stages the
// step's lse and delta in the K/V-major kernel), warp 1 MMA issuer and
// tensor-memory owner, warps 4-7 and 8-11 the two elementwise groups (K/V-major:
// group g takes the steps i with i % 2 == g of every item; thread t owns row t
// of its tiles).  Tensor memory (512 columns): K/V-major: T1 pair [0,64)
// [64,128), T2 pair [128,192) [192,256), dK, dV [256, 256 + 2D); Q-major:
// regions [0,128) [128,256) [384,512) and dQ [256, 256 + D).  The bf16 P / dS of
// a step overwrite the first 32 columns of the group's part of T1 / T2 once
// read.  Every wait is bounded (as in the forward kernel).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ptx.cuh"
#include "bwd_sched.h"
#include "ring_sched.h"

namespace ra {

namespace tb {
constexpr int THREADS = 384;
constexpr int SLAB = 128 * 64 * 2;      // one 128-row x 64-column bf16 box
constexpr uint32_t TMEM_COLS = 512;
// Register split: 120 for the producer / MMA warpgroup (96 made the K/V-major
// launch spill there), 184 for the elementwise warpgroups.  128*120 + 256*184 =
// 62,464 must not exceed 384 threads x the registers a thread is launched with
// (the launcher checks REG_NEED against the built kernel before every launch).
constexpr int REG_LOW = 120, REG_HIGH = 184;
constexpr int REG_NEED = (128 * REG_LOW + 256 * REG_HIGH + THREADS - 1) / THREADS;
}  // namespace tb

template <int D, int SR>
struct BwdSmem {
  static constexpr int NST = SR == 64 ? 4 : 2;          // step stages
  alignas(1024) uint8_t x[2][tb::BR * D * 2];           // item tiles (K, V) or (Q, dO)
  alignas(1024) uint8_t y[NST][2][SR * D * 2];          // step tiles (Q, dO) or (K, V)
  alignas(16) float ylse[NST][SR];                      // K/V-major: -lse * log2(e) of the step's queries
  alignas(16) float ydl[NST][SR];                       //            and -delta
  alignas(8) uint64_t x_full, x_empty, teardown;
  alignas(8) uint64_t y_full[NST];
  alignas(8) uint64_t y_empty[NST];
  alignas(8) uint64_t s_full[2];
  alignas(8) uint64_t p_full[2];
  alignas(8) uint64_t acc_full, acc_empty;
  uint32_t tmem_base;
  int abort_flag;
};

struct BwdTcParams {
  Plan p;
  BwdArgs a;
  float sl2;     // scale * log2(e)
  int items;
  unsigned int* err;
};

// TMA load of one ROWS-row tile (D/64 boxes of ROWS x 64, slab after slab) at
// row x of chunk slot `slot`
template <int D, int ROWS>
__device__ __forceinline__ void load_tile(const Plan& p, uint32_t dst, const CUtensorMap* tm, uint32_t bar, int head,
                                          int slot, int x, int b, uint64_t pol) {
#pragma unroll
  for (int sl = 0; sl < D / 64; ++sl) {
    if (p.strided)
      tma_load_5d(dst + sl * ROWS * 128, tm, bar, sl * 64, head, slot, x, b, pol);
    else
      tma_load_4d(dst + sl * ROWS * 128, tm, bar, sl * 64, head, buf_row(p, slot, x), b, pol);
  }
}

template <int D, bool kKvMajor>
__global__ void __launch_bounds__(tb::THREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmX1, const __grid_constant__ CUtensorMap tmX2,
                       const __grid_constant__ CUtensorMap tmY1, const __grid_constant__ CUtensorMap tmY2,
                       const BwdTcParams prm) {
  using namespace tb;
  // K/V-major: 64-row steps, the two groups ping-pong between two T1/T2 pairs; Q-major:
  // 128-key steps (tensor memory holds one pair beside dQ), both groups on every step,
  // group g on the columns [64g, 64g + 64)
  constexpr int SR = kKvMajor ? BS : BR;
  constexpr bool PP = kKvMajor;
  using Smem = BwdSmem<D, SR>;
  constexpr int NST = Smem::NST;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Plan& p = prm.p;
  unsigned int* err = prm.err;
  volatile int* abort_flag = &sm.abort_flag;
  constexpr uint32_t XTILE = BR * D * 2, YTILE = SR * D * 2;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.x_full), 1);
    mbar_init(smem_u32(&sm.x_empty), 1);
    mbar_init(smem_u32(&sm.teardown), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&sm.y_full[s]), 1);
      mbar_init(smem_u32(&sm.y_empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full[0]), 1);
    mbar_init(smem_u32(&sm.s_full[1]), 1);
    mbar_init(smem_u32(&sm.p_full[0]), 128);
    mbar_init(smem_u32(&sm.p_full[1]), 128);
    mbar_init(smem_u32(&sm.acc_full), 1);
    mbar_init(smem_u32(&sm.acc_empty), 256);
    sm.abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
    setmaxnreg_dec<REG_LOW>();
    if (warp == 0) {
      // ============================================================ producer (whole warp)
      const uint64_t pol_x = l2_policy_evict_first();
      const uint64_t pol_y = l2_policy_evict_last();
      const CUtensorMap* x1 = &tmX1;
      const CUtensorMap* x2 = &tmX2;
      const CUtensorMap* y1 = &tmY1;
      const CUtensorMap* y2 = &tmY2;
      if (lane == 0) {
        tma_prefetch_desc(x1);
        tma_prefetch_desc(x2);
        tma_prefetch_desc(y1);
        tma_prefetch_desc(y2);
      }
      uint32_t ycnt = 0, n_items = 0;
      bool ok = true;
      auto stage_wait = [&](uint32_t c) -> bool {
        const bool w = mbar_wait(smem_u32(&sm.y_empty[c % NST]), ((c / NST) & 1u) ^ 1u, abort_flag, kWaitKvEmpty, err);
        return __all_sync(0xffffffffu, w);
      };
      for (int w = 0, L = turn_item(0, blockIdx.x, gridDim.x, prm.items, kKvMajor); L >= 0 && ok;
           L = turn_item(++w, blockIdx.x, gridDim.x, prm.items, kKvMajor), ++n_items) {
        if (n_items > 0) {
          const bool w = mbar_wait(smem_u32(&sm.x_empty), (n_items - 1) & 1u, abort_flag, kWaitQEmpty, err);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        }
        if constexpr (kKvMajor) {
          const KvItem it = kv_item(p, L);
          if (lane == 0) {
            const uint32_t xb = smem_u32(&sm.x_full);
            mbar_arrive_expect_tx(xb, 2 * XTILE);
            load_tile<D, BR>(p, smem_u32(sm.x[0]), x1, xb, it.g, it.ks, it.k_off, it.b, pol_x);
            load_tile<D, BR>(p, smem_u32(sm.x[1]), x2, xb, it.g, it.ks, it.k_off, it.b, pol_x);
          }
          __syncwarp();
          // The step's lse (log2 units) and delta feed its elementwise pass.  They are loaded one
          // step ahead: step i+1's loads are in flight while step i waits for a free stage and
          // issues its copies.  Columns past the tile get +inf / 0 (P = 0).
          auto load_ld = [&](const QStep& q, float (&l2)[BS / 32], float (&dl)[BS / 32]) {
            const size_t base = ((size_t)it.b * p.Hq + q.h) * p.Sq;
#pragma unroll
            for (int i = 0; i < BS / 32; ++i) {
              const int c = lane + 32 * i;
              l2[i] = CUDART_INF_F;
              dl[i] = 0.f;
              if (c < q.nq) {
                const size_t li = base + buf_row(p, q.qs, q.q_off + c);
                l2[i] = __ldg(prm.a.lse + li);
                dl[i] = __ldg(prm.a.delta + li);
              }
            }
          };
          QStepIter si{0, 0, 0};
          QStep st, st_next;
          float l2[BS / 32], dl[BS / 32];
          bool have = qstep_next(p, it, si, st);
          if (have) load_ld(st, l2, dl);
          while (have) {
            float l2n[BS / 32], dln[BS / 32];
            const bool have_next = qstep_next(p, it, si, st_next);
            if (have_next) load_ld(st_next, l2n, dln);
            if (!stage_wait(ycnt)) { ok = false; break; }
            const int s = ycnt % NST;
#pragma unroll
            for (int i = 0; i < BS / 32; ++i) {   // stored negated: the elementwise pass adds them
              sm.ylse[s][lane + 32 * i] = -(l2[i] * 1.4426950408889634f);
              sm.ydl[s][lane + 32 * i] = -dl[i];
            }
            __syncwarp();
            if (lane == 0) {
              const uint32_t fb = smem_u32(&sm.y_full[s]);
              mbar_arrive_expect_tx(fb, 2 * YTILE);   // the arrive also publishes ylse / ydl
              load_tile<D, BS>(p, smem_u32(sm.y[s][0]), y1, fb, st.h, st.qs, st.q_off, it.b, pol_y);
              load_tile<D, BS>(p, smem_u32(sm.y[s][1]), y2, fb, st.h, st.qs, st.q_off, it.b, pol_y);
            }
            __syncwarp();
            ++ycnt;
            have = have_next;
            if (have) {
              st = st_next;
#pragma unroll
              for (int i = 0; i < BS / 32; ++i) {
                l2[i] = l2n[i];
                dl[i] = dln[i];
              }
            }
          }
        } else {
          const QItem it = q_item(p, L);
          if (lane == 0) {
            const uint32_t xb = smem_u32(&sm.x_full);
            mbar_arrive_expect_tx(xb, 2 * XTILE);
            load_tile<D, BR>(p, smem_u32(sm.x[0]), x1, xb, it.h, it.qs, it.q_off, it.b, pol_x);
            load_tile<D, BR>(p, smem_u32(sm.x[1]), x2, xb, it.h, it.qs, it.q_off, it.b, pol_x);
          }
          __syncwarp();
          KvIter ki;
          kv_begin(p, it.qs, ki);
          KvTile t;
          while (kv_next(p, it.q0 + it.nq - 1, SR, cdiv(p.C, SR), ki, t)) {
            if (!stage_wait(ycnt)) { ok = false; break; }
            const int s = ycnt % NST;
            if (lane == 0) {
              const uint32_t fb = smem_u32(&sm.y_full[s]);
              mbar_arrive_expect_tx(fb, 2 * YTILE);
              load_tile<D, SR>(p, smem_u32(sm.y[s][0]), y1, fb, it.g, t.slot, t.k0, it.b, pol_y);
              load_tile<D, SR>(p, smem_u32(sm.y[s][1]), y2, fb, it.g, t.slot, t.k0, it.b, pol_y);
            }
            __syncwarp();
            ++ycnt;
          }
        }
      }
      // let every copy already issued land before the CTA can exit
      if (lane == 0) {
        if (n_items > 0) mbar_wait(smem_u32(&sm.x_full), (n_items - 1) & 1u, nullptr, kWaitTeardown, err);
        for (uint32_t c = (ycnt > (uint32_t)NST ? ycnt - NST : 0); c < ycnt; ++c)
          mbar_wait(smem_u32(&sm.y_full[c % NST]), (c / NST) & 1u, nullptr, kWaitTeardown, err);
      }
    } else if (warp == 1) {
      // ============================================================ MMA issuer
      if (lane == 0) {
        const uint32_t idesc_ss = idesc_bf16_f32(BR, SR, false);   // T = X (128 rows) x Y^T (SR rows)
        const uint32_t idesc_ts = idesc_bf16_f32(BR, D, true);     // acc += T (bf16) x Y (MN-major)
        const uint32_t hi = (uint32_t)(sw128_desc(0, 16, 1024) >> 32);
        const uint32_t T1[2] = {tmem, tmem + 64}, T2[2] = {tmem + 128, tmem + 192};
        const uint32_t A0 = tmem + 256, A1 = tmem + 256 + D;
        constexpr uint32_t YSLAB = SR * 128;                         // one SR-row x 64-column box
        constexpr uint32_t YSTAGE16 = (2 * YTILE) >> 4, YTILE16 = YTILE >> 4;
        const uint32_t lx0 = (uint32_t)sw128_desc(smem_u32(sm.x[0]), 16, 1024);
        const uint32_t lx1 = (uint32_t)sw128_desc(smem_u32(sm.x[1]), 16, 1024);
        const uint32_t ly_k = (uint32_t)sw128_desc(smem_u32(sm.y[0][0]), 16, 1024);     // K-major (SS)
        const uint32_t ly_mn = (uint32_t)sw128_desc(smem_u32(sm.y[0][0]), YSLAB, 1024); // MN-major (TS)
        uint32_t ycnt = 0, n_items = 0, pb[2] = {0u, 0u};
        bool ok = true;
        auto wait_y = [&](uint32_t c) -> bool {
          if (!mbar_wait(smem_u32(&sm.y_full[c % NST]), (c / NST) & 1u, abort_flag, kWaitKvFull, err)) return false;
          tc_fence_after();
          return true;
        };
        // dst = X Y^T for tile j (0: X1 Y1^T, 1: X2 Y2^T) of the step in stage c (no commit)
        auto issue_prod = [&](uint32_t dst, int j, uint32_t c) {
          const uint32_t xa = j ? lx1 : lx0;
          const uint32_t yb = ly_k + (c % NST) * YSTAGE16 + (j ? YTILE16 : 0u);
          mma_ss_lo_first(dst, xa, yb, hi, idesc_ss);
#pragma unroll
          for (int k = 1; k < D / 16; ++k)
            mma_ss_lo(dst, xa + (((k / 4) * SLAB + (k % 4) * 32) >> 4), yb + (((k / 4) * YSLAB + (k % 4) * 32) >> 4),
                      hi, idesc_ss);
        };
        // T1[b] = X1 Y1^T, T2[b] = X2 Y2^T for the step in stage c
        auto issue_T = [&](int b, uint32_t c) {
          const uint32_t y1 = ly_k + (c % NST) * YSTAGE16, y2 = y1 + YTILE16;
          mma_ss_lo_first(T1[b], lx0, y1, hi, idesc_ss);
#pragma unroll
          for (int k = 1; k < D / 16; ++k)
            mma_ss_lo(T1[b], lx0 + (((k / 4) * SLAB + (k % 4) * 32) >> 4), y1 + (((k / 4) * YSLAB + (k % 4) * 32) >> 4),
                      hi, idesc_ss);
          mma_ss_lo_first(T2[b], lx1, y2, hi, idesc_ss);
#pragma unroll
          for (int k = 1; k < D / 16; ++k)
            mma_ss_lo(T2[b], lx1 + (((k / 4) * SLAB + (k % 4) * 32) >> 4), y2 + (((k / 4) * YSLAB + (k % 4) * 32) >> 4),
                      hi, idesc_ss);
          mma_commit(smem_u32(&sm.s_full[b]));
        };
        // acc += T (bf16 pairs) x Y (MN-major) over the 64 rows k0 .. k0 + 63 of the step tile: the
        // pairs of those rows start at column tsrc; `first` clears acc
        auto issue_ts = [&](uint32_t acc, uint32_t tsrc, uint32_t ymn, int k0, bool first) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t bk = ymn + (k0 / 16 + k) * ((16 * 128) >> 4);
            if (first && k == 0)
              mma_ts_lo_pred(acc, tsrc, bk, hi, idesc_ts, 0u);
            else
              mma_ts_lo(acc, tsrc + k * 8, bk, hi, idesc_ts);
          }
        };
        for (int w = 0, L = turn_item(0, blockIdx.x, gridDim.x, prm.items, kKvMajor); L >= 0 && ok;
             L = turn_item(++w, blockIdx.x, gridDim.x, prm.items, kKvMajor), ++n_items) {
          if (!mbar_wait(smem_u32(&sm.x_full), n_items & 1u, abort_flag, kWaitQFull, err)) { ok = false; break; }
          tc_fence_after();
          int n;
          if constexpr (kKvMajor) {
            n = qstep_count(p, kv_item(p, L));
          } else {
            const QItem it = q_item(p, L);
            n = kv_count(p, it.qs, it.q0 + it.nq - 1, SR, cdiv(p.C, SR));
          }
          if constexpr (!PP) {
            // Three 128-column regions rotate between S and dP: step i puts S in region
            // (2i) % 3 and dP in (2i + 1) % 3.  S(i) is free once the groups have read it, so
            // dP(i+1) reuses it and S(i+2) takes the third region: while the groups work on
            // step i the tensor cores compute S(i+1); after them, dQ += dS(i) K(i), dP(i+1), S(i+2).
            auto region = [&](int r) -> uint32_t { return tmem + (r == 2 ? 384u : 128u * r); };
            if (n > 0 && ok) {
              if ((ok = wait_y(ycnt))) {
                issue_prod(region(0), 0, ycnt);
                issue_prod(region(1), 1, ycnt);
                mma_commit(smem_u32(&sm.s_full[0]));
                if (n > 1 && (ok = wait_y(ycnt + 1))) issue_prod(region(2), 0, ycnt + 1);
              }
            }
            if (ok && n > 0 && n_items > 0) {
              ok = mbar_wait(smem_u32(&sm.acc_empty), (n_items - 1) & 1u, abort_flag, kWaitOFinal, err);
              tc_fence_after();
            }
            for (int i = 0; i < n && ok; ++i) {
              const uint32_t c = ycnt + i;
              const uint32_t rd = region((2 * i + 1) % 3);
              const uint32_t ymn = ly_mn + (c % NST) * YSTAGE16;
              for (int w = 0; w < 2 && ok; ++w) {
                if (!(ok = mbar_wait(smem_u32(&sm.p_full[w]), pb[0] & 1u, abort_flag, kWaitPFull, err))) break;
                tc_fence_after();
                issue_ts(A0, rd + 64 * w, ymn, 64 * w, i == 0 && w == 0);   // dQ += dS(i) K(i)
              }
              if (!ok) break;
              ++pb[0];
              mma_commit(smem_u32(&sm.y_empty[c % NST]));
              if (i + 1 < n) {
                issue_prod(region((2 * (i + 1) + 1) % 3), 1, c + 1);        // dP(i+1) over S(i)
                mma_commit(smem_u32(&sm.s_full[0]));                        // S(i+1) and dP(i+1)
              }
              if (i + 2 < n) {
                if (!(ok = wait_y(c + 2))) break;
                issue_prod(region((2 * (i + 2)) % 3), 0, c + 2);             // S(i+2) over dS(i)
              }
            }
          }
          // T(0), T(1) | TS(0) T(2) | TS(1) T(3) | ...
          for (int i = 0; PP && i < 2 && i < n && ok; ++i) {
            if (!(ok = wait_y(ycnt + i))) break;
            issue_T(i, ycnt + i);
          }
          if (PP && n > 0 && ok && n_items > 0) {
            // the accumulators are read by the previous item's epilogue until acc_empty
            ok = mbar_wait(smem_u32(&sm.acc_empty), (n_items - 1) & 1u, abort_flag, kWaitOFinal, err);
            tc_fence_after();
          }
          for (int i = 0; PP && i < n && ok; ++i) {
            const int b = i & 1;
            const uint32_t c = ycnt + i;
            if (!(ok = mbar_wait(smem_u32(&sm.p_full[b]), pb[b] & 1u, abort_flag, kWaitPFull, err))) break;
            ++pb[b];
            tc_fence_after();
            const uint32_t ymn = ly_mn + (c % NST) * YSTAGE16;
            issue_ts(A0, T2[b], ymn, 0, i == 0);                                  // dK += dS^T x Q
            issue_ts(A1, T1[b], ymn + YTILE16, 0, i == 0);                          // dV += P^T x dO
            mma_commit(smem_u32(&sm.y_empty[c % NST]));
            if (i + 2 < n) {
              if (!(ok = wait_y(c + 2))) break;
              issue_T(b, c + 2);
            }
          }
          if (!ok) break;
          ycnt += n;
          if (n == 0 && n_items > 0) {
            // an item without steps still hands the accumulators over in order
            if (!mbar_wait(smem_u32(&sm.acc_empty), (n_items - 1) & 1u, abort_flag, kWaitOFinal, err)) {
              ok = false;
              break;
            }
          }
          mma_commit(smem_u32(&sm.x_empty));
          mma_commit(smem_u32(&sm.acc_full));
        }
        // every MMA issued so far must be complete before tensor memory is freed
        mma_commit(smem_u32(&sm.teardown));
        mbar_wait(smem_u32(&sm.teardown), 0, nullptr, kWaitTeardown, err);
      }
    }
  } else {
    setmaxnreg_inc<REG_HIGH>();
    // ============================================================ elementwise groups
    const int g = (warp - 4) >> 2;            // group: steps i with i % 2 == g of every item
    const int wi = warp & 3;                  // tensor-memory lane quarter
    const int row = wi * 32 + lane;           // row of T1/T2 owned by this thread
    const uint32_t lane_off = (uint32_t)(wi * 32) << 16;
    // ping-pong: this group's own pair, all its 64 columns; otherwise the step's pair of rotating
    // regions (see the MMA issuer), columns [64g, 64g + 64)
    uint32_t T1 = tmem + lane_off + (PP ? 64 * g : 0), T2 = tmem + lane_off + 128 + (PP ? 64 * g : 0);
    const int cb = PP ? 0 : 64 * g;             // first column of this group in its pair
    auto region = [&](int r) -> uint32_t { return tmem + lane_off + (r == 2 ? 384u : 128u * r); };
    const uint32_t A0 = tmem + lane_off + 256, A1 = tmem + lane_off + 256 + D;
    const float sl2 = prm.sl2;
    uint32_t ycnt = 0, ns = 0, n_items = 0;
    bool ok = true;

    // One step of this group: read the pair, write bf16 P (K/V-major only) and dS over its
    // first 32 columns, hand it to the MMA issuer.  nl_of(j) / nd_of(j) give -lse*log2(e) and
    // -delta of columns j, j+1 as a packed pair; masked(j) tells whether column j is cut.
    const uint64_t sl2x2 = pack2(sl2, sl2);
    auto step = [&](auto nl_of, auto nd_of, auto masked, bool need) -> bool {
      const bool got = mbar_wait(smem_u32(&sm.s_full[PP ? g : 0]), ns & 1u, abort_flag, kWaitSFull, err);
      if (!__all_sync(0xffffffffu, got)) return false;
      ++ns;
      if constexpr (kKvMajor) {
        // the producer's ylse / ydl stores are published by this stage's full barrier
        const bool f = mbar_wait(smem_u32(&sm.y_full[ycnt % NST]), (ycnt / NST) & 1u, abort_flag, kWaitKvFull, err);
        if (!__all_sync(0xffffffffu, f)) return false;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r1[32], r2[32];
        tmem_ld32(T1 + cb + 32 * c, r1);
        tmem_ld32(T2 + cb + 32 * c, r2);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j = cb + 32 * c + 2 * e;   // column of the step tile (pair j, j+1)
          float x0, x1;
          unpack2(ffma2(pack2(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1])), sl2x2, nl_of(j)), x0, x1);
          float p0 = ex2(x0), p1 = ex2(x1);
          if (need) {
            if (masked(j)) p0 = 0.f;
            if (masked(j + 1)) p1 = 0.f;
          }
          const uint64_t pp = pack2(p0, p1);
          float d0, d1;
          unpack2(fmul2(pp, fadd2(pack2(__uint_as_float(r2[2 * e]), __uint_as_float(r2[2 * e + 1])), nd_of(j))), d0,
                  d1);
          pk[e] = pack_bf16x2(p0, p1);
          dk[e] = pack_bf16x2(d0, d1);
        }
        if constexpr (kKvMajor) tmem_st16(T1 + cb + 16 * c, pk);
        tmem_st16(T2 + cb + 16 * c, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.p_full[g]));
      return true;
    };

    for (int w = 0, L = turn_item(0, blockIdx.x, gridDim.x, prm.items, kKvMajor); L >= 0 && ok;
         L = turn_item(++w, blockIdx.x, gridDim.x, prm.items, kKvMajor), ++n_items) {
      int nsteps = 0;
      if constexpr (kKvMajor) {
        const KvItem it = kv_item(p, L);
        QStepIter si{0, 0, 0};
        QStep st;
        const bool row_live = row < it.nk;
        while (qstep_next(p, it, si, st)) {
          if ((nsteps & 1) == g) {
            // key row (position k0 + row) sees query column j iff k0 + row <= q0 + j; columns
            // past the tile carry lse = +inf (P = 0); rows past the tile see nothing
            const int lim = p.causal ? (st.k0 + row) - st.q0 : -BS;
            const bool need = (p.causal && st.k0 + BR - 1 > st.q0) || !row_live;
            const int sidx = ycnt % NST;
            const float2* nl = reinterpret_cast<const float2*>(sm.ylse[sidx]);
            const float2* nd = reinterpret_cast<const float2*>(sm.ydl[sidx]);
            if (!(ok = step([&](int j) { const float2 v = nl[j >> 1]; return pack2(v.x, v.y); },
                            [&](int j) { const float2 v = nd[j >> 1]; return pack2(v.x, v.y); },
                            [&](int j) { return !row_live || j < lim; }, need)))
              break;
          }
          ++ycnt;
          ++nsteps;
        }
        if (!ok) break;
        // ---- epilogue: dK (scaled) and dV rows of this item; group g writes columns [D/2 g, D/2 (g+1))
        const bool fin = mbar_wait(smem_u32(&sm.acc_full), n_items & 1u, abort_flag, kWaitOFinal, err);
        if (!__all_sync(0xffffffffu, fin)) { ok = false; break; }
        tc_fence_after();
        const bool live = row < it.nk;
        const size_t orow = ((size_t)it.b * p.Skv + buf_row(p, it.ks, it.k_off + (live ? row : 0))) * p.Hkv + it.g;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const int col = (D / 2) * g + 32 * c;
          uint32_t rk[32], rv[32];
          tmem_ld32(A0 + col, rk);
          tmem_ld32(A1 + col, rv);
          tmem_wait_ld();
          if (live) {
            if (prm.a.dk_acc) {
              float* dkp = prm.a.dk_acc + orow * D + col;
              float* dvp = prm.a.dv_acc + orow * D + col;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                dkp[e] += nsteps ? prm.a.scale * __uint_as_float(rk[e]) : 0.f;
                dvp[e] += nsteps ? __uint_as_float(rv[e]) : 0.f;
              }
            } else {
              uint4 wk[4], wv[4];
              uint32_t* pk = reinterpret_cast<uint32_t*>(wk);
              uint32_t* pv = reinterpret_cast<uint32_t*>(wv);
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float k0v = nsteps ? prm.a.scale * __uint_as_float(rk[2 * e]) : 0.f;
                const float k1v = nsteps ? prm.a.scale * __uint_as_float(rk[2 * e + 1]) : 0.f;
                pk[e] = pack_bf16x2(k0v, k1v);
                pv[e] = nsteps ? pack_bf16x2(__uint_as_float(rv[2 * e]), __uint_as_float(rv[2 * e + 1])) : 0u;
              }
              uint4* dk4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.a.dk) + orow * D + col);
              uint4* dv4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.a.dv) + orow * D + col);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                dk4[e] = wk[e];
                dv4[e] = wv[e];
              }
            }
          }
          __syncwarp();
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.acc_empty));
      } else {
        const QItem it = q_item(p, L);
        const bool live = row < it.nq;
        const size_t li = ((size_t)it.b * p.Hq + it.h) * p.Sq + buf_row(p, it.qs, it.q_off + (live ? row : 0));
        const float l2_row = live ? prm.a.lse[li] * 1.4426950408889634f : CUDART_INF_F;   // +inf: P = 0
        const float dl_row = live ? prm.a.delta[li] : 0.f;
        const int qpos = it.q0 + row;
        KvIter ki;
        kv_begin(p, it.qs, ki);
        KvTile t;
        while (kv_next(p, it.q0 + it.nq - 1, SR, cdiv(p.C, SR), ki, t)) {
          {
            // query row (position q0 + row) sees key column j iff pos0 + j <= q0 + row
            const int lim = p.causal ? qpos - t.pos0 : SR;
            const int nv = t.nvalid;
            const bool need = (p.causal && t.pos0 + SR - 1 > it.q0) || nv < SR;
            const uint64_t nl2 = pack2(-l2_row, -l2_row), nd2 = pack2(-dl_row, -dl_row);
            T1 = region((2 * nsteps) % 3);
            T2 = region((2 * nsteps + 1) % 3);
            if (!(ok = step([&](int) { return nl2; }, [&](int) { return nd2; },
                            [&](int j) { return j > lim || j >= nv; }, need)))
              break;
          }
          ++ycnt;
          ++nsteps;
        }
        if (!ok) break;
        const bool fin = mbar_wait(smem_u32(&sm.acc_full), n_items & 1u, abort_flag, kWaitOFinal, err);
        if (!__all_sync(0xffffffffu, fin)) { ok = false; break; }
        tc_fence_after();
        const size_t orow = ((size_t)it.b * p.Sq + buf_row(p, it.qs, it.q_off + (live ? row : 0))) * p.Hq + it.h;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const int col = (D / 2) * g + 32 * c;
          uint32_t rq[32];
          tmem_ld32(A0 + col, rq);
          tmem_wait_ld();
          if (live) {
            if (prm.a.dq_acc) {
              float* dqp = prm.a.dq_acc + orow * D + col;
#pragma unroll
              for (int e = 0; e < 32; ++e) dqp[e] += nsteps ? prm.a.scale * __uint_as_float(rq[e]) : 0.f;
            } else {
              uint4 wq[4];
              uint32_t* pq = reinterpret_cast<uint32_t*>(wq);
#pragma unroll
              for (int e = 0; e < 16; ++e)
                pq[e] = nsteps ? pack_bf16x2(prm.a.scale * __uint_as_float(rq[2 * e]),
                                             prm.a.scale * __uint_as_float(rq[2 * e + 1]))
                               : 0u;
              uint4* dq4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.a.dq) + orow * D + col);
#pragma unroll
              for (int e = 0; e < 4; ++e) dq4[e] = wq[e];
            }
          }
          __syncwarp();
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.acc_empty));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D, bool kKvMajor>
static cudaError_t launch_bwd_tc_d(const Plan& p, const BwdArgs& a, unsigned int* err, cudaStream_t st) {
  // item tiles: 128-row boxes; step tiles: 64-row boxes
  auto map = [&](CUtensorMap* m, const void* base, int rows, int heads, int box_rows) {
    return p.strided ? make_tmap_striped(m, base, p.B, rows, p.P, heads, D, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B)
                     : make_tmap_bhsd(m, base, p.B, rows, heads, D, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  };
  CUtensorMap x1, x2, y1, y2;
  bool ok;
  if (kKvMajor)
    ok = map(&x1, a.k, p.Skv, p.Hkv, tb::BR) && map(&x2, a.v, p.Skv, p.Hkv, tb::BR) &&
         map(&y1, a.q, p.Sq, p.Hq, tb::BS) && map(&y2, a.dout, p.Sq, p.Hq, tb::BS);
  else
    ok = map(&x1, a.q, p.Sq, p.Hq, tb::BR) && map(&x2, a.dout, p.Sq, p.Hq, tb::BR) &&
         map(&y1, a.k, p.Skv, p.Hkv, tb::BR) && map(&y2, a.v, p.Skv, p.Hkv, tb::BR);
  if (!ok) return cudaErrorInvalidValue;
  BwdTcParams prm;
  prm.p = p;
  prm.a = a;
  prm.sl2 = a.scale * 1.4426950408889634f;
  prm.err = err;
  const long long items = kKvMajor ? (long long)p.B * p.Hkv * p.nkc * cdiv(p.C, tb::BR)
                                   : (long long)p.B * p.Hq * p.nqc * cdiv(p.C, tb::BR);
  if (items <= 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  prm.items = (int)items;
  const size_t smem = sizeof(BwdSmem<D, kKvMajor ? tb::BS : tb::BR>) + 1024;
  auto kern = attn_bwd_tc_kernel<D, kKvMajor>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < tb::REG_NEED) return cudaErrorNotSupported;
  const int grid = prm.items < num_sms() ? prm.items : num_sms();
  kern<<<grid, tb::THREADS, smem, st>>>(x1, x2, y1, y2, prm);
  return cudaGetLastError();
}

cudaError_t launch_bwd_tc(const Plan& p, const BwdArgs& a, unsigned int* err, cudaStream_t st) {
  cudaError_t e;
  if (p.D == 128) {
    e = launch_bwd_tc_d<128, true>(p, a, err, st);
    if (e != cudaSuccess) return e;
    return launch_bwd_tc_d<128, false>(p, a, err, st);
  }
  if (p.D == 64) {
    e = launch_bwd_tc_d<64, true>(p, a, err, st);
    if (e != cudaSuccess) return e;
    return launch_bwd_tc_d<64, false>(p, a, err, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace ra
