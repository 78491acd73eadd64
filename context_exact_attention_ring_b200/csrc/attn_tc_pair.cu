// Tensor-core ring attention on CTA pairs (sm_100a, D = 128): the ring of
// attn_tc.cu with every product spread over the two SMs of a TPC.
//
// A cluster of two CTAs takes work items of four 128-row query tiles that
// share every K/V tile (ring_sched.h, item_pair_at): two tiles per CTA.  The
// leader (CTA 0) issues tcgen05.mma.cta_group::2 products with M = 256, rows
// 0-127 from CTA 0's tile and rows 128-255 from CTA 1's tile i:
//     S_i  = Q_i K_j^T   N = 128 keys: each CTA holds 64 of the keys of K_j
//     O_i += P_i V_j     N = 128 dims: each CTA holds 64 of the dims of V_j
// so a CTA stages half of every K/V tile (16 KB of K, 16 KB of V) where the
// one-CTA kernel stages all of it, and its tensor cores read half of B from
// its own shared memory and half from its peer's.  Per K/V tile and SM this
// halves the TMA traffic into shared memory and cuts the shared-memory reads
// of the score products by a quarter ("Lesson 8: Context Parallelism",
// section 1: the ring step's compute per K/V element moved grows with the
// query rows that share it).  The walk of the K/V tiles in each virtual
// rank's ring order, the causal skipping, the online softmax and the
// epilogue are those of attn_tc.cu (tc_softmax_role).
//
// Warp roles per CTA (12 warps):
//   warp 0       TMA producer (one thread): this CTA's two Q tiles, then its
//                half of K_j and of V_j into an 8-stage ring of 16 KB stages;
//                each copy completes on the leader's barrier, which only the
//                leader arms with the bytes of both CTAs.  No multicast.
//   warp 1       tensor-memory owner; in the leader also the MMA issuer;
//   warps 4-11   the two softmax groups (one query tile each).
// Commits from the leader arrive on the barrier of both CTAs (multicast
// commit); the softmax warps of both CTAs arrive on the leader's p_full.
// Tensor memory per CTA as in attn_tc.cu: S0, S1, O0, O1 (512 columns).
// Every wait is bounded; at the end both CTAs meet at a bounded exit barrier
// (the leader's products read the peer's shared memory and write its tensor
// memory) before tensor memory is freed.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ptx.cuh"
#include "ring_sched.h"
#include "tc_softmax.cuh"

namespace ra {

namespace tcp {
constexpr int D = 128;
constexpr int NST = 8;                       // stages of half a K tile or half a V tile
constexpr int STAGE = 16384;                 // bytes per stage
constexpr int SLAB_K = 64 * 64 * 2;          // 64 key rows x 64 dims (8 KB, 128-byte swizzle)
constexpr int Q_BYTES = tc::BM * D * 2;      // one query tile (32 KB)
// Register split: 120 for the producer / MMA warpgroup (the four-tile items need
// more than the one-CTA kernel's 96), 184 for the softmax warpgroups; 128*120 +
// 256*184 = 62,464 must fit the 384 threads x registers the kernel is launched
// with (checked by the launcher).
constexpr int REG_LOW = 120;
constexpr int REG_NEED = (128 * REG_LOW + 256 * tc::REG_HIGH + tc::THREADS - 1) / tc::THREADS;
}  // namespace tcp

struct TcPairSmem {
  alignas(1024) uint8_t q[2][tcp::Q_BYTES];
  alignas(1024) uint8_t kv[tcp::NST][tcp::STAGE];
  alignas(16) float epi[8][tc::kEpiFloats];   // step-mode epilogue staging, one tile per softmax warp
  alignas(8) uint64_t q_full, q_empty, teardown, exit_bar;
  alignas(8) uint64_t kv_full[tcp::NST];
  alignas(8) uint64_t kv_empty[tcp::NST];
  alignas(8) uint64_t s_full[2];
  alignas(8) uint64_t p_full[2];
  alignas(8) uint64_t o_final[2];
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(tc::THREADS, 1)
    attn_tc_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const TcParams prm) {
  using namespace tc;
  using tcp::D;
  using tcp::NST;
  extern __shared__ uint8_t smem_raw[];
  TcPairSmem& sm = *reinterpret_cast<TcPairSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Plan& p = prm.p;
  const ItemSpace& space = prm.space;
  unsigned int* err = prm.a.err;
  volatile int* abort_flag = &sm.abort_flag;
  // A cluster of two along x holds blocks 2c and 2c + 1: cluster c, ranks 0 (leader) and 1.
  // Derived from blockIdx / gridDim where used (the compiler can re-read them
  // instead of holding them in registers across the roles).
#define PAIR_CTA ((uint32_t)blockIdx.x & 1u)
#define PAIR_ITEM0 ((int)(blockIdx.x >> 1))
#define PAIR_STRIDE ((int)(gridDim.x >> 1))

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    mbar_init(smem_u32(&sm.teardown), 1);
    mbar_init(smem_u32(&sm.exit_bar), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&sm.kv_full[s]), 1);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.p_full[i]), 8);   // one arrival per softmax warp of both CTAs
      mbar_init(smem_u32(&sm.o_final[i]), 1);
    }
    sm.abort_flag = 0;
    // the pair layout assumed throughout (ranks 0 and 1 are blocks 2c and 2c + 1); if the
    // hardware numbered them otherwise, every role unwinds at its first wait
    if (cluster_ctarank() != PAIR_CTA) {
      atomicCAS(err, 0u, (unsigned int)kPairRank);
      sm.abort_flag = 1;
    }
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&sm.tmem_base), TMEM_COLS);
    tmem_relinquish_pair();
  }
  // step mode: let the next call on the stream start on SMs as this call's CTAs exit; it
  // waits for this call's completion before it touches the caller's state
  if (prm.p.mode == kModeStep) grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers are initialised before any copy or arrival reaches them
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
    setmaxnreg_dec<tcp::REG_LOW>();
    if (warp == 0) {
      // ================================================================ producer (both CTAs)
      if (lane == 0) {
        const uint32_t cta = PAIR_CTA;
        const bool leader = cta == 0;
        // the leader's barriers, as shared::cluster addresses
        const uint32_t q_full_L = mapa_shared(smem_u32(&sm.q_full), 0);
        const uint32_t kv_full_L = mapa_shared(smem_u32(&sm.kv_full[0]), 0);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        const uint64_t pol_q = l2_policy_evict_first();
        const uint64_t pol_kv = l2_policy_evict_last();
        const int tpc = cdiv(p.C, BN);
        uint32_t kv_cnt = 0, n_items = 0;
        bool ok = true;
        for (int w = 0, L = turn_item(0, PAIR_ITEM0, PAIR_STRIDE, space.count, false); L >= 0 && ok;
             L = turn_item(++w, PAIR_ITEM0, PAIR_STRIDE, space.count, false), ++n_items) {
          const Item it = item_pair_at(p, space, BM, L, (int)cta);
          if (n_items > 0 && !mbar_wait(smem_u32(&sm.q_empty), (n_items - 1) & 1u, abort_flag, kWaitQEmpty, err)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(smem_u32(&sm.q_full), 2 * 2 * tcp::Q_BYTES);   // both CTAs' tiles
          for (int i = 0; i < 2; ++i)
            for (int sl = 0; sl < D / 64; ++sl)
              if (p.strided)
                tma_load_5d_pair(smem_u32(sm.q[i]) + sl * SLAB, &tmQ, q_full_L, sl * 64, it.h[i], it.qslot,
                                 it.qoff[i], it.b, pol_q);
              else
                tma_load_4d_pair(smem_u32(sm.q[i]) + sl * SLAB, &tmQ, q_full_L, sl * 64, it.h[i], it.qrow0[i],
                                 it.b, pol_q);
          KvIter iter;
          kv_begin(p, it.qslot, iter);
          KvTile t;
          while (ok && kv_next(p, it.qhi, BN, tpc, iter, t)) {
            for (int kind = 0; kind < 2; ++kind) {
              const int s = kv_cnt % NST;
              if (!mbar_wait(smem_u32(&sm.kv_empty[s]), ((kv_cnt / NST) & 1u) ^ 1u, abort_flag, kWaitKvEmpty,
                             err)) {
                ok = false;
                break;
              }
              if (leader) mbar_arrive_expect_tx(smem_u32(&sm.kv_full[s]), 2 * tcp::STAGE);
              const uint32_t fb = kv_full_L + 8u * s;
              const uint32_t dst = smem_u32(sm.kv[s]);
              if (kind == 0) {
                // K: this CTA's 64 keys of the tile, both 64-dim slabs
                for (int sl = 0; sl < D / 64; ++sl) {
                  if (p.strided)
                    tma_load_5d_pair(dst + sl * tcp::SLAB_K, &tmK, fb, sl * 64, it.hkv, t.slot, t.k0 + 64 * (int)cta,
                                     it.b, pol_kv);
                  else
                    tma_load_4d_pair(dst + sl * tcp::SLAB_K, &tmK, fb, sl * 64, it.hkv, t.row0 + 64 * (int)cta, it.b,
                                     pol_kv);
                }
              } else {
                // V: this CTA's 64 dims of all 128 keys of the tile
                if (p.strided)
                  tma_load_5d_pair(dst, &tmV, fb, 64 * (int)cta, it.hkv, t.slot, t.k0, it.b, pol_kv);
                else
                  tma_load_4d_pair(dst, &tmV, fb, 64 * (int)cta, it.hkv, t.row0, it.b, pol_kv);
              }
              ++kv_cnt;
            }
          }
        }
        // let every copy already issued land before the CTA can exit (the leader's barriers
        // count the bytes of both CTAs)
        if (leader) {
          if (n_items > 0) mbar_wait(smem_u32(&sm.q_full), (n_items - 1) & 1u, nullptr, kWaitTeardown, err);
          for (uint32_t c = (kv_cnt > (uint32_t)NST ? kv_cnt - NST : 0); c < kv_cnt; ++c)
            mbar_wait(smem_u32(&sm.kv_full[c % NST]), (c / NST) & 1u, nullptr, kWaitTeardown, err);
        }
      }
    } else if (warp == 1 && PAIR_CTA == 0) {
      // ================================================================ MMA issuer (leader)
      if (lane == 0) {
        const uint32_t idesc_qk = idesc_bf16_f32(2 * BM, BN, false);
        const uint32_t idesc_pv = idesc_bf16_f32(2 * BM, D, true);
        const uint32_t tS[2] = {tmem, tmem + 128};
        const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
        const uint32_t hi = (uint32_t)(sw128_desc(0, 16, 1024) >> 32);
        const uint32_t lq[2] = {(uint32_t)sw128_desc(smem_u32(sm.q[0]), 16, 1024),
                                (uint32_t)sw128_desc(smem_u32(sm.q[1]), 16, 1024)};
        const uint32_t lk0 = (uint32_t)sw128_desc(smem_u32(sm.kv[0]), 16, 1024);     // K half, K-major
        const uint32_t lv0 = (uint32_t)sw128_desc(smem_u32(sm.kv[0]), SLAB, 1024);   // V half, MN-major
        constexpr uint32_t STAGE16 = tcp::STAGE >> 4;
        const int tpc = cdiv(p.C, BN);
        uint32_t kv_cnt = 0, n_items = 0, tiles_done = 0;
        bool ok = true;

        auto issue_S = [&](int i, uint32_t s) {
          const uint32_t a = lq[i], b = lk0 + s * STAGE16;
          mma_ss_lo_first_pair(tS[i], a, b, hi, idesc_qk);
#pragma unroll
          for (int k = 1; k < D / 16; ++k) {
            const uint32_t off_a = ((k / 4) * SLAB + (k % 4) * 32) >> 4;
            const uint32_t off_b = ((k / 4) * tcp::SLAB_K + (k % 4) * 32) >> 4;
            mma_ss_lo_pair(tS[i], a + off_a, b + off_b, hi, idesc_qk);
          }
        };
        auto issue_PV = [&](int i, uint32_t s, bool acc) {
          const uint32_t b = lv0 + s * STAGE16;
          mma_ts_lo_pred_pair(tO[i], tS[i], b, hi, idesc_pv, acc ? 1u : 0u);
#pragma unroll
          for (int k = 1; k < BN / 16; ++k)
            mma_ts_lo_pair(tO[i], tS[i] + k * 8, b + k * ((16 * 128) >> 4), hi, idesc_pv);
        };
        auto wait_stage = [&](uint32_t c) -> bool {
          return mbar_wait(smem_u32(&sm.kv_full[c % NST]), (c / NST) & 1u, abort_flag, kWaitKvFull, err);
        };
        auto wait_p = [&](int i, uint32_t parity) -> bool {
          return mbar_wait(smem_u32(&sm.p_full[i]), parity, abort_flag, kWaitPFull, err);
        };
        // the producer fills the stages in the order K_0, V_0, K_1, V_1, ... (one count kv_cnt)
        for (int w = 0, L = turn_item(0, PAIR_ITEM0, PAIR_STRIDE, space.count, false); L >= 0 && ok;
             L = turn_item(++w, PAIR_ITEM0, PAIR_STRIDE, space.count, false), ++n_items) {
          const Item it = item_pair_at(p, space, BM, L, 0);
          const int n = kv_count(p, it.qslot, it.qhi, BN, tpc);
          if (!mbar_wait(smem_u32(&sm.q_full), n_items & 1u, abort_flag, kWaitQFull, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (n == 0) {
            mma_commit_pair_both(smem_u32(&sm.q_empty));
            continue;
          }
          const uint32_t sK = kv_cnt;
          if (!wait_stage(sK)) {
            ok = false;
            break;
          }
          issue_S(0, sK % NST);
          mma_commit_pair_both(smem_u32(&sm.s_full[0]));
          issue_S(1, sK % NST);
          mma_commit_pair_both(smem_u32(&sm.s_full[1]));
          mma_commit_pair_both(smem_u32(&sm.kv_empty[sK % NST]));
          ++kv_cnt;
          for (int j = 0; j < n; ++j) {
            const bool has_next = j + 1 < n;
            const uint32_t sV = kv_cnt++;
            if (!wait_stage(sV)) {
              ok = false;
              break;
            }
            if (!wait_p(0, (tiles_done + j) & 1u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_PV(0, sV % NST, j > 0);
            if (!has_next) mma_commit_pair_both(smem_u32(&sm.o_final[0]));
            uint32_t sKn = 0;
            if (has_next) {
              sKn = kv_cnt;
              if (!wait_stage(sKn)) {
                ok = false;
                break;
              }
              issue_S(0, sKn % NST);
              mma_commit_pair_both(smem_u32(&sm.s_full[0]));
            }
            if (!wait_p(1, (tiles_done + j) & 1u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_PV(1, sV % NST, j > 0);
            if (!has_next) mma_commit_pair_both(smem_u32(&sm.o_final[1]));
            mma_commit_pair_both(smem_u32(&sm.kv_empty[sV % NST]));
            if (has_next) {
              issue_S(1, sKn % NST);
              mma_commit_pair_both(smem_u32(&sm.s_full[1]));
              mma_commit_pair_both(smem_u32(&sm.kv_empty[sKn % NST]));
              ++kv_cnt;
            }
          }
          if (!ok) break;
          tiles_done += n;
          mma_commit_pair_both(smem_u32(&sm.q_empty));
        }
        // every product issued so far must be complete before either CTA frees tensor memory
        mma_commit_pair_local(smem_u32(&sm.teardown));
        mbar_wait(smem_u32(&sm.teardown), 0, nullptr, kWaitTeardown, err);
      }
    }
  } else {
    setmaxnreg_inc<REG_HIGH>();
    // ================================================================ softmax groups (both CTAs)
    tc_softmax_role<D, true>(prm, tmem, warp, lane, smem_u32(&sm.s_full[0]), mapa_shared(smem_u32(&sm.p_full[0]), 0),
                             smem_u32(&sm.o_final[0]), abort_flag, PAIR_ITEM0, PAIR_STRIDE, (int)PAIR_CTA,
                             sm.epi[warp - 4]);
  }

  tc_fence_before();
  __syncthreads();
  // Both CTAs are done: the leader's products (which read the peer's shared memory and write
  // its tensor memory) have completed, and every copy has landed.  A bounded exit barrier
  // keeps either CTA from leaving while its peer may still touch its memory.
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(mapa_shared(smem_u32(&sm.exit_bar), PAIR_CTA ^ 1u));
    mbar_wait_cluster(smem_u32(&sm.exit_bar), 0, nullptr, kWaitTeardown, err, kWaitLimitNs);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
#undef PAIR_CTA
#undef PAIR_ITEM0
#undef PAIR_STRIDE
}

// Launch of the pair kernel (D = 128).  The grid is a whole number of
// clusters of two, no more than can be resident at once.
cudaError_t launch_attn_tc_pair(const Plan& p, const TcArgs& a, cudaStream_t st) {
  if (p.D != tcp::D) return cudaErrorNotSupported;
  CUtensorMap tq, tk, tv;
  constexpr int D = tcp::D;
  if (p.strided) {
    if (!make_tmap_striped(&tq, a.q, p.B, p.Sq, p.P, p.Hq, D, 64, tc::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_striped(&tk, a.k, p.B, p.Skv, p.P, p.Hkv, D, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_striped(&tv, a.v, p.B, p.Skv, p.P, p.Hkv, D, 64, tc::BN, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else if (!make_tmap_bhsd(&tq, a.q, p.B, p.Sq, p.Hq, D, 64, tc::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_bhsd(&tk, a.k, p.B, p.Skv, p.Hkv, D, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_bhsd(&tv, a.v, p.B, p.Skv, p.Hkv, D, 64, tc::BN, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return cudaErrorInvalidValue;
  }
  TcParams prm;
  prm.p = p;
  prm.space = item_space_pair(p, tc::BM);
  prm.a = a;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  if (prm.space.count <= 0) return cudaSuccess;
  const size_t smem = sizeof(TcPairSmem) + 1024;
  auto kern = attn_tc_pair_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < tcp::REG_NEED) return cudaErrorNotSupported;   // setmaxnreg.inc could not be met
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // step mode: may overlap the previous kernel of the stream (see grid_dependency_wait)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(tc::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2 * 74);
  int max_clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (max_clusters < 1) return cudaErrorNotSupported;
  const int clusters = prm.space.count < max_clusters ? prm.space.count : max_clusters;
  cfg.gridDim = dim3(2 * clusters);
  if (p.mode == kModeStep) cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace ra
