// Backward of ring attention on the tensor cores (tcgen05, bf16 operands,
// fp32 accumulation in tensor memory).  The gradients are the calculus of the
// forward (the pages give no backward):
//   P = exp(scale * Q K^T - lse),  dP = dO V^T,  dS = P o (dP - delta),
//   dV = P^T dO,  dK = scale * dS^T Q,  dQ = scale * dS K,
// with P recomputed tile by tile from the forward's lse.  Two launches of one
// kernel template, neither with atomics:
//   kKvMajor = true   a work item is a 128-key K/V tile of one kv head; its
//                     steps are the 128-row query tiles (of every query head
//                     of the group) that the block meets as it travels round
//                     the ring ("Lesson 8: Context Parallelism", section 2):
//                       T1 = K Q^T, T2 = V dO^T      (SS: K, V, Q, dO in smem)
//                       P^T, dS^T from T1, T2          (two elementwise groups)
//                       dV += P^T dO, dK += dS^T Q    (TS: P^T, dS^T in tmem)
//   kKvMajor = false  a work item is a 128-row query tile of one head; its
//                     steps are the K/V tiles in the rank's ring order:
//                       T1 = Q K^T, T2 = dO V^T,  dS from T1, T2,
//                       dQ += dS K                    (TS)
// Every MMA is 128 x 128 (x 16), the shapes of the forward kernel; the
// shared-memory tiles are the forward's 128-row, 128-byte-swizzled boxes,
// read K-major by the SS products and MN-major by the TS products.
//
// Warp roles (12 warps): warp 0 TMA producer (the whole warp also stages the
// step's lse and delta in the K/V-major kernel), warp 1 MMA issuer and
// tensor-memory owner, warps 4-7 and 8-11 the two elementwise groups: thread
// t owns row t of T1/T2, group w the columns [64w, 64w + 64).  Tensor memory
// (512 columns): T1 [0,128), T2 [128,256), accumulators [256, 256 + 2D);
// the bf16 P / dS of group w overwrite columns [64w, 64w + 32) of T1 / T2
// once read.  Every wait is bounded (as in the forward kernel).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ptx.cuh"
#include "ring_sched.h"

namespace ra {

namespace tb {
constexpr int BR = 128;                 // rows of every tile
constexpr int NST = 2;                  // step stages
constexpr int THREADS = 384;
constexpr int SLAB = 128 * 64 * 2;      // one 128-row x 64-column bf16 box
constexpr uint32_t TMEM_COLS = 512;
constexpr int REG_LOW = 96, REG_HIGH = 184;
constexpr int REG_NEED = (128 * REG_LOW + 256 * REG_HIGH + THREADS - 1) / THREADS;
}  // namespace tb

template <int D>
struct BwdSmem {
  alignas(1024) uint8_t x[2][tb::BR * D * 2];           // item tiles (K, V) or (Q, dO)
  alignas(1024) uint8_t y[tb::NST][2][tb::BR * D * 2];  // step tiles (Q, dO) or (K, V)
  float ylse[tb::NST][tb::BR];                          // K/V-major: lse * log2(e) of the step's queries
  float ydl[tb::NST][tb::BR];                           //            and their delta
  alignas(8) uint64_t x_full, x_empty, teardown;
  alignas(8) uint64_t y_full[tb::NST];
  alignas(8) uint64_t y_empty[tb::NST];
  alignas(8) uint64_t s_full;
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

// ---------------------------------------------------------------- work items
// K/V-major item: one 128-key tile of chunk slot ks, kv head g, batch b.
struct KvItem {
  int b, g, ks, k_off, nk, srank;
};
__device__ __forceinline__ KvItem kv_item(const Plan& p, int L) {
  const int tpk = cdiv(p.C, tb::BR);
  const int per_bg = p.nkc * tpk;
  KvItem it;
  const int bg = L / per_bg, r = L - bg * per_bg;
  it.b = bg / p.Hkv;
  it.g = bg - it.b * p.Hkv;
  it.ks = r / tpk;
  it.k_off = (r - it.ks * tpk) * tb::BR;
  it.nk = imin(tb::BR, p.C - it.k_off);
  it.srank = p.mode == kModeRing ? chunk_owner(p, it.ks) : 0;
  return it;
}

// One step of a K/V-major item: a 128-row query tile of head h in chunk qs.
struct QStep {
  int h, qs, q_off, nq, q0, k0;
};
struct QStepIter {
  int h, n, qt;
};
__device__ __forceinline__ bool qstep_next(const Plan& p, const KvItem& it, QStepIter& s, QStep& out) {
  const int G = p.Hq / p.Hkv, tpq = cdiv(p.C, tb::BR);
  while (s.h < G) {
    if (s.n >= p.nqc) {
      s.n = 0;
      ++s.h;
      continue;
    }
    if (s.qt >= tpq) {
      s.qt = 0;
      ++s.n;
      continue;
    }
    // the block of rank srank meets ranks srank, srank+1, ... (ring mode); buffer order (step mode)
    const int qs = p.mode == kModeRing ? rank_chunk(p, (it.srank + s.n / p.cpr) % p.P, s.n % p.cpr) : s.n;
    const int q_off = s.qt * tb::BR;
    const int nq = imin(tb::BR, p.C - q_off);
    const int q0 = q_pos_base(p, qs) + q_off;
    const int k0 = kv_pos_base(p, q_gid(p, qs), it.ks) + it.k_off;
    ++s.qt;
    if (p.causal && k0 > q0 + nq - 1) continue;   // every key after every query of the tile
    out.h = it.g * G + s.h;
    out.qs = qs;
    out.q_off = q_off;
    out.nq = nq;
    out.q0 = q0;
    out.k0 = k0;
    return true;
  }
  return false;
}

// Q-major item: one 128-row query tile of head h (longest work first).
struct QItem {
  int b, h, g, qs, q_off, nq, q0;
};
__device__ __forceinline__ QItem q_item(const Plan& p, int L) {
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

// TMA load of one 128-row tile (D/64 boxes) at row x of chunk slot `slot`
template <int D>
__device__ __forceinline__ void load_tile(const Plan& p, uint32_t dst, const CUtensorMap* tm, uint32_t bar, int head,
                                          int slot, int x, int b, uint64_t pol) {
#pragma unroll
  for (int sl = 0; sl < D / 64; ++sl) {
    if (p.strided)
      tma_load_5d(dst + sl * tb::SLAB, tm, bar, sl * 64, head, slot, x, b, pol);
    else
      tma_load_4d(dst + sl * tb::SLAB, tm, bar, sl * 64, head, buf_row(p, slot, x), b, pol);
  }
}

template <int D, bool kKvMajor>
__global__ void __launch_bounds__(tb::THREADS, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const BwdTcParams prm) {
  using namespace tb;
  extern __shared__ uint8_t smem_raw[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Plan& p = prm.p;
  unsigned int* err = prm.err;
  volatile int* abort_flag = &sm.abort_flag;
  constexpr uint32_t TILE = BR * D * 2;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.x_full), 1);
    mbar_init(smem_u32(&sm.x_empty), 1);
    mbar_init(smem_u32(&sm.teardown), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&sm.y_full[s]), 1);
      mbar_init(smem_u32(&sm.y_empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
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
      const CUtensorMap* x1 = kKvMajor ? &tmK : &tmQ;
      const CUtensorMap* x2 = kKvMajor ? &tmV : &tmO;
      const CUtensorMap* y1 = kKvMajor ? &tmQ : &tmK;
      const CUtensorMap* y2 = kKvMajor ? &tmO : &tmV;
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
      for (int L = blockIdx.x; L < prm.items && ok; L += gridDim.x, ++n_items) {
        if (n_items > 0) {
          const bool w = mbar_wait(smem_u32(&sm.x_empty), (n_items - 1) & 1u, abort_flag, kWaitQEmpty, err);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        }
        if constexpr (kKvMajor) {
          const KvItem it = kv_item(p, L);
          if (lane == 0) {
            const uint32_t xb = smem_u32(&sm.x_full);
            mbar_arrive_expect_tx(xb, 2 * TILE);
            load_tile<D>(p, smem_u32(sm.x[0]), x1, xb, it.g, it.ks, it.k_off, it.b, pol_x);
            load_tile<D>(p, smem_u32(sm.x[1]), x2, xb, it.g, it.ks, it.k_off, it.b, pol_x);
          }
          __syncwarp();
          QStepIter si{0, 0, 0};
          QStep st;
          while (qstep_next(p, it, si, st)) {
            if (!stage_wait(ycnt)) { ok = false; break; }
            const int s = ycnt % NST;
            // the step's lse (log2 units) and delta; columns past the tile get +inf / 0, i.e. P = 0
            const size_t base = ((size_t)it.b * p.Hq + st.h) * p.Sq;
#pragma unroll
            for (int i = 0; i < BR / 32; ++i) {
              const int c = lane + 32 * i;
              float l2 = CUDART_INF_F, dl = 0.f;
              if (c < st.nq) {
                const size_t li = base + buf_row(p, st.qs, st.q_off + c);
                l2 = prm.a.lse[li] * 1.4426950408889634f;
                dl = prm.a.delta[li];
              }
              sm.ylse[s][c] = l2;
              sm.ydl[s][c] = dl;
            }
            __syncwarp();
            if (lane == 0) {
              const uint32_t fb = smem_u32(&sm.y_full[s]);
              mbar_arrive_expect_tx(fb, 2 * TILE);   // the arrive also publishes ylse / ydl
              load_tile<D>(p, smem_u32(sm.y[s][0]), y1, fb, st.h, st.qs, st.q_off, it.b, pol_y);
              load_tile<D>(p, smem_u32(sm.y[s][1]), y2, fb, st.h, st.qs, st.q_off, it.b, pol_y);
            }
            __syncwarp();
            ++ycnt;
          }
        } else {
          const QItem it = q_item(p, L);
          if (lane == 0) {
            const uint32_t xb = smem_u32(&sm.x_full);
            mbar_arrive_expect_tx(xb, 2 * TILE);
            load_tile<D>(p, smem_u32(sm.x[0]), x1, xb, it.h, it.qs, it.q_off, it.b, pol_x);
            load_tile<D>(p, smem_u32(sm.x[1]), x2, xb, it.h, it.qs, it.q_off, it.b, pol_x);
          }
          __syncwarp();
          KvIter ki;
          kv_begin(p, it.qs, ki);
          KvTile t;
          while (kv_next(p, it.q0 + it.nq - 1, BR, cdiv(p.C, BR), ki, t)) {
            if (!stage_wait(ycnt)) { ok = false; break; }
            const int s = ycnt % NST;
            if (lane == 0) {
              const uint32_t fb = smem_u32(&sm.y_full[s]);
              mbar_arrive_expect_tx(fb, 2 * TILE);
              load_tile<D>(p, smem_u32(sm.y[s][0]), y1, fb, it.g, t.slot, t.k0, it.b, pol_y);
              load_tile<D>(p, smem_u32(sm.y[s][1]), y2, fb, it.g, t.slot, t.k0, it.b, pol_y);
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
        const uint32_t idesc_ss = idesc_bf16_f32(BR, BR, false);
        const uint32_t idesc_ts = idesc_bf16_f32(BR, D, true);
        const uint32_t hi = (uint32_t)(sw128_desc(0, 16, 1024) >> 32);
        const uint32_t T1 = tmem, T2 = tmem + 128, A0 = tmem + 256, A1 = tmem + 256 + D;
        const uint32_t lx[2] = {(uint32_t)sw128_desc(smem_u32(sm.x[0]), 16, 1024),
                                (uint32_t)sw128_desc(smem_u32(sm.x[1]), 16, 1024)};
        uint32_t ly_k[NST][2], ly_mn[NST][2];   // step tiles read K-major (SS) and MN-major (TS)
#pragma unroll
        for (int s = 0; s < NST; ++s)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            ly_k[s][j] = (uint32_t)sw128_desc(smem_u32(sm.y[s][j]), 16, 1024);
            ly_mn[s][j] = (uint32_t)sw128_desc(smem_u32(sm.y[s][j]), SLAB, 1024);
          }
        uint32_t ycnt = 0, steps = 0, n_items = 0;
        bool ok = true;
        auto issue_ss = [&](uint32_t d, uint32_t a, uint32_t b) {
          mma_ss_lo_first(d, a, b, hi, idesc_ss);
#pragma unroll
          for (int k = 1; k < D / 16; ++k) {
            const uint32_t off = ((k / 4) * SLAB + (k % 4) * 32) >> 4;
            mma_ss_lo(d, a + off, b + off, hi, idesc_ss);
          }
        };
        // acc += T[:, half w] (bf16, tmem) x Y[rows of half w] (MN-major); `first` clears acc
        auto issue_ts_half = [&](uint32_t acc, uint32_t tsrc, uint32_t b, int w, bool first) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int k = 4 * w + kk;
            const uint32_t a = tsrc + 64 * w + kk * 8;
            const uint32_t bk = b + k * ((16 * 128) >> 4);
            if (first && kk == 0)
              mma_ts_lo_pred(acc, a, bk, hi, idesc_ts, 0u);
            else
              mma_ts_lo(acc, a, bk, hi, idesc_ts);
          }
        };
        for (int L = blockIdx.x; L < prm.items && ok; L += gridDim.x, ++n_items) {
          if (!mbar_wait(smem_u32(&sm.x_full), n_items & 1u, abort_flag, kWaitQFull, err)) { ok = false; break; }
          tc_fence_after();
          bool first = true;
          auto run_step = [&]() -> bool {
            const int s = ycnt % NST;
            if (!mbar_wait(smem_u32(&sm.y_full[s]), (ycnt / NST) & 1u, abort_flag, kWaitKvFull, err)) return false;
            tc_fence_after();
            issue_ss(T1, lx[0], ly_k[s][0]);
            issue_ss(T2, lx[1], ly_k[s][1]);
            mma_commit(smem_u32(&sm.s_full));
            if (first && n_items > 0) {
              // the accumulators are read by the previous item's epilogue until acc_empty
              if (!mbar_wait(smem_u32(&sm.acc_empty), (n_items - 1) & 1u, abort_flag, kWaitOFinal, err))
                return false;
              tc_fence_after();
            }
            for (int w = 0; w < 2; ++w) {
              if (!mbar_wait(smem_u32(&sm.p_full[w]), steps & 1u, abort_flag, kWaitPFull, err)) return false;
              tc_fence_after();
              issue_ts_half(A0, T2, ly_mn[s][0], w, first && w == 0);        // dK or dQ += dS x Y1
              if constexpr (kKvMajor) issue_ts_half(A1, T1, ly_mn[s][1], w, first && w == 0);   // dV += P x Y2
            }
            mma_commit(smem_u32(&sm.y_empty[s]));
            first = false;
            ++ycnt;
            ++steps;
            return true;
          };
          if constexpr (kKvMajor) {
            const KvItem it = kv_item(p, L);
            QStepIter si{0, 0, 0};
            QStep st;
            while (qstep_next(p, it, si, st))
              if (!(ok = run_step())) break;
          } else {
            const QItem it = q_item(p, L);
            KvIter ki;
            kv_begin(p, it.qs, ki);
            KvTile t;
            while (kv_next(p, it.q0 + it.nq - 1, BR, cdiv(p.C, BR), ki, t))
              if (!(ok = run_step())) break;
          }
          if (!ok) break;
          if (first && n_items > 0) {
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
    const int w = (warp - 4) >> 2;            // column half of this group
    const int wi = warp & 3;                  // tensor-memory lane quarter
    const int row = wi * 32 + lane;           // row of T1/T2 owned by this thread
    const uint32_t lane_off = (uint32_t)(wi * 32) << 16;
    const uint32_t T1 = tmem + lane_off, T2 = tmem + lane_off + 128;
    const uint32_t A0 = tmem + lane_off + 256, A1 = tmem + lane_off + 256 + D;
    const float sl2 = prm.sl2;
    uint32_t ycnt = 0, steps = 0, n_items = 0;
    bool ok = true;

    // Q-major step: dS of this thread's query row over the group's 64 key columns.  Column j
    // is masked when j > lim (causal) or j >= ncols (past the tile); rows past the tile carry
    // lse = +inf, i.e. P = 0.
    auto elementwise_q = [&](float l2_row, float dl_row, int lim, int ncols, bool need_mask) -> bool {
      const bool got = mbar_wait(smem_u32(&sm.s_full), steps & 1u, abort_flag, kWaitSFull, err);
      if (!__all_sync(0xffffffffu, got)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int col = 64 * w + 32 * c;
        uint32_t r1[32], r2[32];
        tmem_ld32(T1 + col, r1);
        tmem_ld32(T2 + col, r2);
        tmem_wait_ld();
        uint32_t dk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float ds[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int j = col + 2 * e + u;
            float x = ex2(fmaf(__uint_as_float(r1[2 * e + u]), sl2, -l2_row));
            if (need_mask && (j > lim || j >= ncols)) x = 0.f;
            ds[u] = x * (__uint_as_float(r2[2 * e + u]) - dl_row);
          }
          dk[e] = pack_bf16x2(ds[0], ds[1]);
        }
        tmem_st16(T2 + 64 * w + 16 * c, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.p_full[w]));
      ++ycnt;
      ++steps;
      return true;
    };

    for (int L = blockIdx.x; L < prm.items && ok; L += gridDim.x, ++n_items) {
      int nsteps = 0;
      if constexpr (kKvMajor) {
        const KvItem it = kv_item(p, L);
        QStepIter si{0, 0, 0};
        QStep st;
        while (qstep_next(p, it, si, st)) {
          // key row `row` (position k0 + row) sees query column j iff k0 + row <= q0 + j, so
          // columns j < lim_causal are masked; rows past the tile see nothing; columns past
          // the tile carry lse = +inf (P = 0)
          const int lim_causal = p.causal ? (st.k0 + row) - st.q0 : -BR;
          const bool full = !p.causal || st.k0 + BR - 1 <= st.q0;
          const bool need = !full || it.nk < BR;
          const int s = ycnt % NST;
          const bool got = mbar_wait(smem_u32(&sm.s_full), steps & 1u, abort_flag, kWaitSFull, err);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          const bool f = mbar_wait(smem_u32(&sm.y_full[s]), (ycnt / NST) & 1u, abort_flag, kWaitKvFull, err);
          if (!__all_sync(0xffffffffu, f)) { ok = false; break; }
          tc_fence_after();
          const bool row_live = row < it.nk;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int col = 64 * w + 32 * c;
            uint32_t r1[32], r2[32];
            tmem_ld32(T1 + col, r1);
            tmem_ld32(T2 + col, r2);
            tmem_wait_ld();
            uint32_t pk[16], dk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float pe[2], ds[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int j = col + 2 * e + u;
                float x = ex2(fmaf(__uint_as_float(r1[2 * e + u]), sl2, -sm.ylse[s][j]));
                if (need && (!row_live || j < lim_causal)) x = 0.f;   // columns >= nq carry lse = +inf
                pe[u] = x;
                ds[u] = x * (__uint_as_float(r2[2 * e + u]) - sm.ydl[s][j]);
              }
              pk[e] = pack_bf16x2(pe[0], pe[1]);
              dk[e] = pack_bf16x2(ds[0], ds[1]);
            }
            tmem_st16(T1 + 64 * w + 16 * c, pk);
            tmem_st16(T2 + 64 * w + 16 * c, dk);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(smem_u32(&sm.p_full[w]));
          ++ycnt;
          ++steps;
          ++nsteps;
        }
        if (!ok) break;
        // ---- epilogue: dK (scaled) and dV rows of this item; group w writes columns [D/2 w, D/2 (w+1))
        const bool fin = mbar_wait(smem_u32(&sm.acc_full), n_items & 1u, abort_flag, kWaitOFinal, err);
        if (!__all_sync(0xffffffffu, fin)) { ok = false; break; }
        tc_fence_after();
        const bool live = row < it.nk;
        const size_t orow = ((size_t)it.b * p.Skv + buf_row(p, it.ks, it.k_off + (live ? row : 0))) * p.Hkv + it.g;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const int col = (D / 2) * w + 32 * c;
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
        while (kv_next(p, it.q0 + it.nq - 1, BR, cdiv(p.C, BR), ki, t)) {
          // query row (position q0 + row) sees key column j iff pos0 + j <= q0 + row
          const int lim = p.causal ? qpos - t.pos0 : BR;
          const bool need = (p.causal && t.pos0 + BR - 1 > it.q0) || t.nvalid < BR;
          if (!(ok = elementwise_q(l2_row, dl_row, lim, t.nvalid, need))) break;
          ++nsteps;
        }
        if (!ok) break;
        const bool fin = mbar_wait(smem_u32(&sm.acc_full), n_items & 1u, abort_flag, kWaitOFinal, err);
        if (!__all_sync(0xffffffffu, fin)) { ok = false; break; }
        tc_fence_after();
        const size_t orow = ((size_t)it.b * p.Sq + buf_row(p, it.qs, it.q_off + (live ? row : 0))) * p.Hq + it.h;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const int col = (D / 2) * w + 32 * c;
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
  CUtensorMap tq, tk, tv, to;
  const void* qp = a.q;
  if (p.strided) {
    if (!make_tmap_striped(&tq, qp, p.B, p.Sq, p.P, p.Hq, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_striped(&to, a.dout, p.B, p.Sq, p.P, p.Hq, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_striped(&tk, a.k, p.B, p.Skv, p.P, p.Hkv, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_striped(&tv, a.v, p.B, p.Skv, p.P, p.Hkv, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else if (!make_tmap_bhsd(&tq, qp, p.B, p.Sq, p.Hq, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_bhsd(&to, a.dout, p.B, p.Sq, p.Hq, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_bhsd(&tk, a.k, p.B, p.Skv, p.Hkv, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_bhsd(&tv, a.v, p.B, p.Skv, p.Hkv, D, 64, tb::BR, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return cudaErrorInvalidValue;
  }
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
  const size_t smem = sizeof(BwdSmem<D>) + 1024;
  auto kern = attn_bwd_tc_kernel<D, kKvMajor>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < tb::REG_NEED) return cudaErrorNotSupported;
  const int grid = prm.items < num_sms() ? prm.items : num_sms();
  kern<<<grid, tb::THREADS, smem, st>>>(tq, tk, tv, to, prm);
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
