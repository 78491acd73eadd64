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
// Online softmax per row, in log2 units x = s * scale * log2(e):
//   m_new = max(m, max_j x_j); the base m is only moved when m_new exceeds it
//   by more than 8 (a factor 256), in which case l and the O row are rescaled
//   by 2^(m - m_new) in place; p_j = 2^(x_j - m) is written as bf16 for the PV
//   product and l += sum p_j in fp32.  lt is l corrected by the bf16 rounding
//   of each tile's largest weight (the error that does not average out when
//   one key dominates).  Using a stale base is exact: l, lt and O share it.
//   out = O / lt, lse = (m + log2 l) * ln 2.
// Every wait is bounded; a wait that expires flags the device error word and
// all roles unwind, let in-flight copies and MMAs finish, and free tensor
// memory before the CTA exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ptx.cuh"
#include "ring_sched.h"

namespace ra {

namespace tc {
constexpr int BM = 128, BN = 128;
constexpr int NST = 4;        // K/V stages
constexpr int THREADS = 384;
constexpr int SLAB = 128 * 64 * 2;   // one 128-row x 64-column bf16 box (16 KB, 128-byte swizzle)
constexpr float LAZY = 8.f;
constexpr uint32_t TMEM_COLS = 512;
constexpr int REG_LOW = 96, REG_HIGH = 184;
constexpr int REG_NEED = (128 * REG_LOW + 256 * REG_HIGH + THREADS - 1) / THREADS;   // per thread at launch
}  // namespace tc

template <int D>
struct TcSmem {
  alignas(1024) uint8_t q[2][tc::BM * D * 2];
  alignas(1024) uint8_t kv[tc::NST][tc::BN * D * 2];
  alignas(8) uint64_t q_full, q_empty, teardown;
  alignas(8) uint64_t kv_full[tc::NST];
  alignas(8) uint64_t kv_empty[tc::NST];
  alignas(8) uint64_t s_full[2];
  alignas(8) uint64_t p_full[2];
  alignas(8) uint64_t o_final[2];
  uint32_t tmem_base;
  int abort_flag;
};

struct TcParams {
  Plan p;
  ItemSpace space;
  TcArgs a;
  float scale_log2;
};

__device__ __forceinline__ float mergew_exp(float x) { return expf(x); }

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
      for (int L = blockIdx.x; L < space.count && ok; L += gridDim.x, ++n_items) {
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

      for (int L = blockIdx.x; L < space.count && ok; L += gridDim.x, ++n_items) {
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

    for (int L = blockIdx.x; L < space.count && ok; L += gridDim.x) {
      const Item it = item_at(p, space, BM, L);
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
        const bool got = mbar_wait(smem_u32(&sm.s_full[i]), (tiles_done + j) & 1u, abort_flag, kWaitSFull, err);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tS + c * 32, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
        }
        tmem_wait_ld();
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
        mbar_arrive(smem_u32(&sm.p_full[i]));
        ++j;
      }
      if (!ok) break;
      tiles_done += j;
      if (j == 0) continue;   // step mode: nothing of this block is visible to these rows

      const bool fin = mbar_wait(smem_u32(&sm.o_final[i]), items_with_tiles & 1u, abort_flag, kWaitOFinal, err);
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
        // fold this block into the caller's state (natural-log units, exact max)
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
        float* Orow = prm.a.O + (((size_t)it.b * p.Sq + qr) * p.Hq + h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
          if (active) {
            float4* dst = reinterpret_cast<float4*>(Orow + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4 o = dst[e];
              o.x = w_old * o.x + w_blk * (__uint_as_float(r[4 * e + 0]) * inv_l);
              o.y = w_old * o.y + w_blk * (__uint_as_float(r[4 * e + 1]) * inv_l);
              o.z = w_old * o.z + w_blk * (__uint_as_float(r[4 * e + 2]) * inv_l);
              o.w = w_old * o.w + w_blk * (__uint_as_float(r[4 * e + 3]) * inv_l);
              dst[e] = o;
            }
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
  kern<<<grid, tc::THREADS, smem, st>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const Plan& p, const TcArgs& a, cudaStream_t st) {
  if (p.D == 128) return launch_tc_d<128>(p, a, st);
  if (p.D == 64) return launch_tc_d<64>(p, a, st);
  return cudaErrorNotSupported;
}

}  // namespace ra
