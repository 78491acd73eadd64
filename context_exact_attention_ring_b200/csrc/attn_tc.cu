// Tensor-core ring attention for sm_100a: bf16 operands, fp32 accumulation in
// tensor memory (tcgen05), K/V tiles streamed by TMA.
//
// One persistent CTA per SM takes work items (two 128-row query tiles that
// share every K/V tile; see ring_sched.h) and, for each, walks the K/V tiles
// in the owning virtual rank's ring order ("Lesson 8: Context Parallelism",
// section 2), skipping tiles the causal mask removes (section 4).  The
// pages' double-buffered send/receive of K/V blocks becomes, inside one GPU, a
// 4-stage TMA ring of shared memory: the next tiles are in flight while the
// tensor cores work on the current one.  The running (m, l, O) of section 3
// lives on chip: m and l in registers of the softmax threads (one row each),
// O in tensor memory, so state never leaves the SM between ring steps.
//
// Warp roles (12 warps):
//   warp 0       TMA producer (one thread): Q tile pair, then K_j, V_j into
//                the stage ring;
//   warp 1       MMA issuer (one thread) and tensor-memory owner:
//                  S_i = Q_i K_j^T   (SS: both operands in shared memory)
//                  O_i += P_i V_j    (TS: P_i read from tensor memory)
//                issued as S0(j) S1(j) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//                so each softmax group works while the tensor cores serve the
//                other one;
//   warps 4-7    softmax group 0 (query tile 0), thread t owns row t;
//   warps 8-11   softmax group 1 (query tile 1).
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D); P_i (bf16 pairs) overwrites the first 64 columns of S_i
// once the row has been read.
//
// The online softmax of the two groups and the epilogue are tc_softmax_role
// (tc_softmax.cuh), shared with the CTA-pair kernel (attn_tc_pair.cu).
// Every wait is bounded; a wait that expires flags the device error word and
// all roles unwind, let in-flight copies and MMAs finish, and free tensor
// memory before the CTA exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <cstdlib>
#include <cstring>

#include "kernels.h"
#include "ptx.cuh"
#include "ring_sched.h"
#include "tc_softmax.cuh"

namespace ra {

namespace tc {
constexpr int NST = 4;        // K/V stages
}  // namespace tc

template <int D>
struct TcSmem {
  alignas(1024) uint8_t q[2][tc::BM * D * 2];
  alignas(1024) uint8_t kv[tc::NST][tc::BN * D * 2];
  alignas(16) float epi[8][tc::kEpiFloats];   // step-mode epilogue staging, one tile per softmax warp
  alignas(8) uint64_t q_full, q_empty, teardown;
  alignas(8) uint64_t kv_full[tc::NST];
  alignas(8) uint64_t kv_empty[tc::NST];
  alignas(8) uint64_t s_full[2];
  alignas(8) uint64_t p_full[2];
  alignas(8) uint64_t o_final[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(tc::THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const TcParams prm) {
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  TcSmem<D>& sm = *reinterpret_cast<TcSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Plan& p = prm.p;
  const ItemSpace& space = prm.space;
  unsigned int* err = prm.a.err;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    mbar_init(smem_u32(&sm.teardown), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&sm.kv_full[s]), 1);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.p_full[i]), 128);
      mbar_init(smem_u32(&sm.o_final[i]), 1);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  // step mode: let the next call on the stream start on SMs as this call's CTAs exit; it
  // waits for this call's completion before it touches the caller's state
  if (prm.p.mode == kModeStep) grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // Registers: the producer / MMA warpgroup needs few, the softmax warpgroups
  // hold a 128-column score row each.  128*REG_LOW + 256*REG_HIGH must not
  // exceed the 384 threads x registers the kernel was launched with (checked
  // by the launcher before every launch).

  if (warp < 4) {
  setmaxnreg_dec<REG_LOW>();
  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      const int tpc = cdiv(p.C, BN);
      uint32_t kv_cnt = 0, n_items = 0;
      bool ok = true;
      for (int w = 0, L = turn_item(0, blockIdx.x, gridDim.x, space.count, true); L >= 0 && ok;
             L = turn_item(++w, blockIdx.x, gridDim.x, space.count, true), ++n_items) {
        const Item it = item_at(p, space, BM, L);
        if (n_items > 0 && !mbar_wait(smem_u32(&sm.q_empty), (n_items - 1) & 1u, abort_flag, kWaitQEmpty, err)) {
          ok = false;
          break;
        }
        const uint32_t qb = smem_u32(&sm.q_full);
        mbar_arrive_expect_tx(qb, 2 * BM * D * 2);
        for (int i = 0; i < 2; ++i)
          for (int sl = 0; sl < D / 64; ++sl)
            if (p.strided)
              tma_load_5d(smem_u32(sm.q[i]) + sl * SLAB, &tmQ, qb, sl * 64, it.h[i], it.qslot, it.qoff[i], it.b,
                          pol_q);
            else
              tma_load_4d(smem_u32(sm.q[i]) + sl * SLAB, &tmQ, qb, sl * 64, it.h[i], it.qrow0[i], it.b, pol_q);
        KvIter iter;
        kv_begin(p, it.qslot, iter);
        KvTile t;
        while (ok && kv_next(p, it.qhi, BN, tpc, iter, t)) {
          for (int kind = 0; kind < 2; ++kind) {
            const int s = kv_cnt % NST;
            if (!mbar_wait(smem_u32(&sm.kv_empty[s]), ((kv_cnt / NST) & 1u) ^ 1u, abort_flag, kWaitKvEmpty, err)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&sm.kv_full[s]);
            mbar_arrive_expect_tx(fb, BN * D * 2);
            const void* tm = kind == 0 ? (const void*)&tmK : (const void*)&tmV;
            for (int sl = 0; sl < D / 64; ++sl) {
              if (p.strided)
                tma_load_5d(smem_u32(sm.kv[s]) + sl * SLAB, tm, fb, sl * 64, it.hkv, t.slot, t.k0, it.b, pol_kv);
              else
                tma_load_4d(smem_u32(sm.kv[s]) + sl * SLAB, tm, fb, sl * 64, it.hkv, t.row0, it.b, pol_kv);
            }
            ++kv_cnt;
          }
        }
      }
      // let every copy already issued land before the CTA can exit
      if (n_items > 0) mbar_wait(smem_u32(&sm.q_full), (n_items - 1) & 1u, nullptr, kWaitTeardown, err);
      for (uint32_t c = (kv_cnt > (uint32_t)NST ? kv_cnt - NST : 0); c < kv_cnt; ++c)
        mbar_wait(smem_u32(&sm.kv_full[c % NST]), (c / NST) & 1u, nullptr, kWaitTeardown, err);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
      const uint32_t idesc_pv = idesc_bf16_f32(BM, D, true);
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
      // descriptors built once: per MMA only a constant is added to a 32-bit low word
      const uint32_t hi = (uint32_t)(sw128_desc(0, 16, 1024) >> 32);   // same for K- and MN-major here
      const uint32_t lq[2] = {(uint32_t)sw128_desc(smem_u32(sm.q[0]), 16, 1024),
                              (uint32_t)sw128_desc(smem_u32(sm.q[1]), 16, 1024)};
      const uint32_t lk0 = (uint32_t)sw128_desc(smem_u32(sm.kv[0]), 16, 1024);     // K tile, K-major
      const uint32_t lv0 = (uint32_t)sw128_desc(smem_u32(sm.kv[0]), SLAB, 1024);   // V tile, MN-major
      constexpr uint32_t STAGE16 = (BN * D * 2) >> 4;                             // stage stride, 16-byte units
      const int tpc = cdiv(p.C, BN);
      uint32_t kv_cnt = 0, n_items = 0, tiles_done = 0;
      bool ok = true;

      auto issue_S = [&](int i, uint32_t s) {
        const uint32_t a = lq[i], b = lk0 + s * STAGE16;
        mma_ss_lo_first(tS[i], a, b, hi, idesc_qk);
#pragma unroll
        for (int k = 1; k < D / 16; ++k) {
          const uint32_t off = ((k / 4) * SLAB + (k % 4) * 32) >> 4;
          mma_ss_lo(tS[i], a + off, b + off, hi, idesc_qk);
        }
      };
      auto issue_PV = [&](int i, uint32_t s, bool acc) {
        const uint32_t b = lv0 + s * STAGE16;
        mma_ts_lo_pred(tO[i], tS[i], b, hi, idesc_pv, acc ? 1u : 0u);
#pragma unroll
        for (int k = 1; k < BN / 16; ++k) mma_ts_lo(tO[i], tS[i] + k * 8, b + k * ((16 * 128) >> 4), hi, idesc_pv);
      };
      // K/V tiles are written by TMA (async proxy) and published by the mbarrier's
      // transaction count; no tcgen05 fence is needed to read them.
      auto wait_stage = [&](uint32_t c) -> bool {
        return mbar_wait(smem_u32(&sm.kv_full[c % NST]), (c / NST) & 1u, abort_flag, kWaitKvFull, err);
      };

      for (int w = 0, L = turn_item(0, blockIdx.x, gridDim.x, space.count, true); L >= 0 && ok;
             L = turn_item(++w, blockIdx.x, gridDim.x, space.count, true), ++n_items) {
        const Item it = item_at(p, space, BM, L);
        const int n = kv_count(p, it.qslot, it.qhi, BN, tpc);
        if (!mbar_wait(smem_u32(&sm.q_full), n_items & 1u, abort_flag, kWaitQFull, err)) { ok = false; break; }
        tc_fence_after();
        if (n == 0) {
          mma_commit(smem_u32(&sm.q_empty));
          continue;
        }
        // S0(0), S1(0)
        const uint32_t sK = kv_cnt;
        if (!wait_stage(sK)) { ok = false; break; }
        issue_S(0, sK % NST);
        mma_commit(smem_u32(&sm.s_full[0]));
        issue_S(1, sK % NST);
        mma_commit(smem_u32(&sm.s_full[1]));
        mma_commit(smem_u32(&sm.kv_empty[sK % NST]));
        ++kv_cnt;
        for (int j = 0; j < n; ++j) {
          const bool has_next = j + 1 < n;
          const uint32_t sV = kv_cnt++;
          if (!wait_stage(sV)) { ok = false; break; }
          if (!mbar_wait(smem_u32(&sm.p_full[0]), (tiles_done + j) & 1u, abort_flag, kWaitPFull, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_PV(0, sV % NST, j > 0);
          if (!has_next) mma_commit(smem_u32(&sm.o_final[0]));
          uint32_t sKn = 0;
          if (has_next) {
            sKn = kv_cnt;
            if (!wait_stage(sKn)) { ok = false; break; }
            issue_S(0, sKn % NST);
            mma_commit(smem_u32(&sm.s_full[0]));
          }
          if (!mbar_wait(smem_u32(&sm.p_full[1]), (tiles_done + j) & 1u, abort_flag, kWaitPFull, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_PV(1, sV % NST, j > 0);
          if (!has_next) mma_commit(smem_u32(&sm.o_final[1]));
          mma_commit(smem_u32(&sm.kv_empty[sV % NST]));
          if (has_next) {
            issue_S(1, sKn % NST);
            mma_commit(smem_u32(&sm.s_full[1]));
            mma_commit(smem_u32(&sm.kv_empty[sKn % NST]));
            ++kv_cnt;
          }
        }
        if (!ok) break;
        tiles_done += n;
        mma_commit(smem_u32(&sm.q_empty));
      }
      // every MMA issued so far must be complete before tensor memory is freed
      mma_commit(smem_u32(&sm.teardown));
      mbar_wait(smem_u32(&sm.teardown), 0, nullptr, kWaitTeardown, err);
    }
  }
  } else {
    setmaxnreg_inc<REG_HIGH>();
    // ================================================================ softmax groups
    tc_softmax_role<D, false>(prm, tmem, warp, lane, smem_u32(&sm.s_full[0]), smem_u32(&sm.p_full[0]),
                              smem_u32(&sm.o_final[0]), abort_flag, blockIdx.x, gridDim.x, 0, sm.epi[warp - 4]);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D>
static cudaError_t launch_tc_d(const Plan& p, const TcArgs& a, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (p.strided) {
    if (!make_tmap_striped(&tq, a.q, p.B, p.Sq, p.P, p.Hq, D, 64, tc::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_striped(&tk, a.k, p.B, p.Skv, p.P, p.Hkv, D, 64, tc::BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_striped(&tv, a.v, p.B, p.Skv, p.P, p.Hkv, D, 64, tc::BN, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else if (!make_tmap_bhsd(&tq, a.q, p.B, p.Sq, p.Hq, D, 64, tc::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_bhsd(&tk, a.k, p.B, p.Skv, p.Hkv, D, 64, tc::BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_tmap_bhsd(&tv, a.v, p.B, p.Skv, p.Hkv, D, 64, tc::BN, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return cudaErrorInvalidValue;
  }
  TcParams prm;
  prm.p = p;
  prm.space = item_space(p, tc::BM);
  prm.a = a;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  if (prm.space.count <= 0) return cudaSuccess;
  const size_t smem = sizeof(TcSmem<D>) + 1024;
  auto kern = attn_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // the in-kernel register split needs this many registers per thread at launch;
  // with fewer, setmaxnreg.inc would wait forever, so refuse instead
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < tc::REG_NEED) return cudaErrorNotSupported;
  const int grid = prm.space.count < num_sms() ? prm.space.count : num_sms();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  // step mode: may overlap the previous kernel of the stream (see grid_dependency_wait)
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(tc::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = p.mode == kModeStep ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// D = 128 with a GQA group that is a multiple of 4 runs on CTA pairs
// (attn_tc_pair.cu): four query heads of one kv head share every K/V tile
// exactly.  Other groups would pair consecutive row tiles, whose shared walk
// computes a few fully masked tiles, and run on this one-CTA kernel.  The
// environment variable RING_ATTN_TC_KERNEL (single | pair) overrides the choice
// for D = 128; both compute the same result.  D = 64 always runs here.
cudaError_t launch_attn_tc(const Plan& p, const TcArgs& a, cudaStream_t st) {
  if (p.D == 128) {
    const char* k = getenv("RING_ATTN_TC_KERNEL");
    const bool pair = k && strcmp(k, "pair") == 0     ? true
                      : k && strcmp(k, "single") == 0 ? false
                                                        : (p.Hq / p.Hkv) % 4 == 0;
    return pair ? launch_attn_tc_pair(p, a, st) : launch_tc_d<128>(p, a, st);
  }
  if (p.D == 64) return launch_tc_d<64>(p, a, st);
  return cudaErrorNotSupported;
}

}  // namespace ra
