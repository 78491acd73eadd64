// Backward of ring attention on CUDA cores (float32 FMA for float32 and bf16
// inputs).  The pages describe the ring for training but give no backward;
// the gradients are the calculus of the forward, as in a blockwise
// attention backward that recomputes P from the saved lse:
//   P    = exp(scale * Q K^T - lse)      (lse of the forward, natural log)
//   dP   = dO V^T
//   dS   = P o (dP - delta),  delta_i = dO_i . O_i
//   dV   = P^T dO,  dK = scale * dS^T Q,  dQ = scale * dS K
// Two kernels, both deterministic (no atomics):
//   attn_bwd_kv_kernel  one CTA per 64-key K/V tile of one kv head; it visits
//                       the query chunks in the order the block travels round
//                       the ring ("Lesson 8: Context Parallelism", section 2:
//                       the block of rank s meets rank s+t at step t) and sums
//                       dK, dV over them and over the query heads of the group;
//   attn_bwd_q_kernel   one CTA per 64-row query tile of one head; it visits
//                       the K/V tiles in the rank's ring order (the forward's
//                       order) and sums dQ.
// Both use the ring scheduler (ring_sched.h): every split, ring or step mode,
// the causal tile filter and the element mask of the forward.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ring_sched.h"

namespace ra {

namespace bwd {
constexpr int BQ = 64, BK = 64;
}

__device__ __forceinline__ float bld(const float* p) { return *p; }
__device__ __forceinline__ float bld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void bst(float* p, float x) { *p = x; }
__device__ __forceinline__ void bst(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// delta[b,h,i] = sum_d dO[b,i,h,d] * O[b,i,h,d]  (one warp per row)
template <typename T>
__global__ void bwd_delta_kernel(const T* __restrict__ out, const T* __restrict__ dout, float* __restrict__ delta,
                                 int B, int Hq, int S, int D) {
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (long long)B * S * Hq) return;
  const int h = (int)(row % Hq);
  const long long bi = row / Hq;
  const int i = (int)(bi % S), b = (int)(bi / S);
  const T* o = out + row * D;
  const T* g = dout + row * D;
  float acc = 0.f;
  for (int d = lane; d < D; d += 32) acc = fmaf(bld(o + d), bld(g + d), acc);
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[((size_t)b * Hq + h) * S + i] = acc;
}

// The same rowsum, HBM-bound, for D*sizeof(T) a multiple of 16 bytes: a warp
// takes 32 consecutive rows of delta's own [B, Hq, S] order (so its result
// leaves as one coalesced 128-byte store); LPR lanes share a row, each loading
// 16 bytes of out and of dout, and the warp covers 32 / LPR rows per
// iteration.  The iterations are unrolled so every lane has several
// independent loads in flight.
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_delta_vec_kernel(const T* __restrict__ out, const T* __restrict__ dout,
                                                            float* __restrict__ delta, int B, int Hq, int S) {
  constexpr int EPV = 16 / (int)sizeof(T);   // elements per 16-byte load
  constexpr int LPR = D / EPV;               // lanes per row
  constexpr int RPI = 32 / LPR;              // rows per warp iteration
  static_assert(D % EPV == 0 && LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "unsupported row size");
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)B * Hq * S;
  const long long r0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32;
  if (r0 >= nrows) return;
  const int sub = lane / LPR, part = lane % LPR;
  // position of row r0 in (b*Hq + h, i) form; later rows advance i and wrap
  const long long bh0 = r0 / S;
  const int i0 = (int)(r0 - bh0 * S);
  float mine = 0.f;
#pragma unroll
  for (int it = 0; it < LPR; ++it) {
    const int k = it * RPI + sub;   // row r0 + k
    float acc = 0.f;
    if (r0 + k < nrows) {
      long long bh = bh0;
      int i = i0 + k;
      while (i >= S) {
        i -= S;
        ++bh;
      }
      const long long b = bh / Hq;
      const int h = (int)(bh - b * Hq);
      const size_t off = (((size_t)b * S + i) * Hq + h) * D + (size_t)part * EPV;
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(out + off));
      const uint4 g = __ldg(reinterpret_cast<const uint4*>(dout + off));
      const T* av = reinterpret_cast<const T*>(&a);
      const T* gv = reinterpret_cast<const T*>(&g);
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc = fmaf(bld(av + e), bld(gv + e), acc);
    }
#pragma unroll
    for (int o = LPR / 2; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    // every lane of group `sub` now holds row k's sum; lane L collects row L
    const float v = __shfl_sync(0xffffffffu, acc, (lane % RPI) * LPR);
    if (lane / RPI == it) mine = v;
  }
  if (r0 + lane < nrows) delta[r0 + lane] = mine;
}

// S = Q K^T and dP = dO V^T for a 64 x 64 tile: thread (ty, tx) owns rows
// ty + 16*ii and keys tx + 16*jj; writes P and dS to shared memory.
template <int D>
__device__ __forceinline__ void tile_p_ds(const float* Qs, const float* Os, const float* Ks, const float* Vs,
                                          const float* Ls, const float* Dl, float* Ps, float* dSs, int nq, int nk,
                                          bool causal, int q0, int k0, float scale, int tid) {
  constexpr int DP = D + 1, PP = bwd::BK + 1;
  const int ty = tid >> 4, tx = tid & 15;
  float s[4][4], dp[4][4];
#pragma unroll
  for (int ii = 0; ii < 4; ++ii)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) s[ii][jj] = dp[ii][jj] = 0.f;
#pragma unroll 4
  for (int d = 0; d < D; ++d) {
    float qv[4], ov[4], kv[4], vv[4];
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      qv[ii] = Qs[(ty + 16 * ii) * DP + d];
      ov[ii] = Os[(ty + 16 * ii) * DP + d];
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      kv[jj] = Ks[(tx + 16 * jj) * DP + d];
      vv[jj] = Vs[(tx + 16 * jj) * DP + d];
    }
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        s[ii][jj] = fmaf(qv[ii], kv[jj], s[ii][jj]);
        dp[ii][jj] = fmaf(ov[ii], vv[jj], dp[ii][jj]);
      }
  }
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const int i = ty + 16 * ii;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = tx + 16 * jj;
      const bool ok = i < nq && j < nk && (!causal || k0 + j <= q0 + i);
      const float pe = ok ? expf(fmaf(s[ii][jj], scale, -Ls[i])) : 0.f;
      Ps[i * PP + j] = pe;
      dSs[i * PP + j] = pe * (dp[ii][jj] - Dl[i]);
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void load_rows(float* dst, const T* src, const Plan& p, int b, int slot, int off, int n,
                                          int S, int H, int h, int tid) {
  constexpr int DP = D + 1;
  for (int e = tid; e < 64 * D; e += 256) {
    const int r = e / D, d = e - r * D;
    float x = 0.f;
    if (r < n) x = bld(src + (((size_t)b * S + buf_row(p, slot, off + r)) * H + h) * D + d);
    dst[r * DP + d] = x;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_bwd_kv_kernel(Plan p, BwdArgs a) {
  using namespace bwd;
  constexpr int DP = D + 1, PP = BK + 1;
  extern __shared__ float smem[];
  float* Ks = smem;
  float* Vs = Ks + BK * DP;
  float* Qs = Vs + BK * DP;
  float* Os = Qs + BQ * DP;
  float* Ps = Os + BQ * DP;
  float* dSs = Ps + BQ * PP;
  float* Ls = dSs + BQ * PP;
  float* Dl = Ls + BQ;

  const T* q = static_cast<const T*>(a.q);
  const T* dout = static_cast<const T*>(a.dout);
  const int tpk = cdiv(p.C, BK), tpq = cdiv(p.C, BQ);
  const int ks = blockIdx.x / tpk, kt = blockIdx.x - ks * tpk;
  const int g = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int k_off = kt * BK, nk = imin(BK, p.C - k_off);
  const int tid = threadIdx.x;
  load_rows<T, D>(Ks, static_cast<const T*>(a.k), p, b, ks, k_off, nk, p.Skv, p.Hkv, g, tid);
  load_rows<T, D>(Vs, static_cast<const T*>(a.v), p, b, ks, k_off, nk, p.Skv, p.Hkv, g, tid);

  // this thread's part of dK, dV: key kk, dims dd + 4t
  const int kk = tid >> 2, dd = tid & 3;
  float dk[D / 4], dv[D / 4];
#pragma unroll
  for (int t = 0; t < D / 4; ++t) dk[t] = dv[t] = 0.f;

  // query chunks in the order the block travels: ranks s, s+1, ... (ring mode); buffer order (step mode)
  const int s_rank = p.mode == kModeRing ? chunk_owner(p, ks) : 0;
  for (int h = g * G; h < (g + 1) * G; ++h) {
    for (int n = 0; n < p.nqc; ++n) {
      int qs;
      if (p.mode == kModeRing) {
        const int r = (s_rank + n / p.cpr) % p.P;
        qs = rank_chunk(p, r, n % p.cpr);
      } else {
        qs = n;
      }
      const int qg = q_gid(p, qs);
      const int qpos0 = q_pos_base(p, qs);
      const int k0 = kv_pos_base(p, qg, ks) + k_off;
      for (int qt = 0; qt < tpq; ++qt) {
        const int q_off = qt * BQ, nq = imin(BQ, p.C - q_off);
        const int q0 = qpos0 + q_off;
        if (p.causal && k0 > q0 + nq - 1) continue;   // every key after every query of the tile
        __syncthreads();
        load_rows<T, D>(Qs, q, p, b, qs, q_off, nq, p.Sq, p.Hq, h, tid);
        load_rows<T, D>(Os, dout, p, b, qs, q_off, nq, p.Sq, p.Hq, h, tid);
        for (int r = tid; r < BQ; r += 256) {
          const bool live = r < nq;
          const size_t li = ((size_t)b * p.Hq + h) * p.Sq + buf_row(p, qs, q_off + (live ? r : 0));
          Ls[r] = live ? a.lse[li] : 0.f;
          Dl[r] = live ? a.delta[li] : 0.f;
        }
        __syncthreads();
        tile_p_ds<D>(Qs, Os, Ks, Vs, Ls, Dl, Ps, dSs, nq, nk, p.causal, q0, k0, a.scale, tid);
        __syncthreads();
        for (int i = 0; i < nq; ++i) {
          const float pv = Ps[i * PP + kk], sv = dSs[i * PP + kk];
#pragma unroll
          for (int t = 0; t < D / 4; ++t) {
            dv[t] = fmaf(pv, Os[i * DP + dd + 4 * t], dv[t]);
            dk[t] = fmaf(sv, Qs[i * DP + dd + 4 * t], dk[t]);
          }
        }
      }
    }
  }
  if (kk < nk) {
    const size_t row = ((size_t)b * p.Skv + buf_row(p, ks, k_off + kk)) * p.Hkv + g;
    if (a.dk_acc) {   // step mode: add to the caller's float32 sums
#pragma unroll
      for (int t = 0; t < D / 4; ++t) {
        a.dk_acc[row * D + dd + 4 * t] += a.scale * dk[t];
        a.dv_acc[row * D + dd + 4 * t] += dv[t];
      }
    } else {
      T* dkp = static_cast<T*>(a.dk) + row * D;
      T* dvp = static_cast<T*>(a.dv) + row * D;
#pragma unroll
      for (int t = 0; t < D / 4; ++t) {
        bst(dkp + dd + 4 * t, a.scale * dk[t]);
        bst(dvp + dd + 4 * t, dv[t]);
      }
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_bwd_q_kernel(Plan p, BwdArgs a) {
  using namespace bwd;
  constexpr int DP = D + 1, PP = BK + 1;
  extern __shared__ float smem[];
  float* Ks = smem;
  float* Vs = Ks + BK * DP;
  float* Qs = Vs + BK * DP;
  float* Os = Qs + BQ * DP;
  float* Ps = Os + BQ * DP;
  float* dSs = Ps + BQ * PP;
  float* Ls = dSs + BQ * PP;
  float* Dl = Ls + BQ;

  const int tpq = cdiv(p.C, BQ), tpk = cdiv(p.C, BK);
  const int qs = blockIdx.x / tpq, qt = blockIdx.x - qs * tpq;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.Hq / p.Hkv);
  const int q_off = qt * BQ, nq = imin(BQ, p.C - q_off);
  const int tid = threadIdx.x;
  const int q0 = q_pos_base(p, qs) + q_off;
  load_rows<T, D>(Qs, static_cast<const T*>(a.q), p, b, qs, q_off, nq, p.Sq, p.Hq, h, tid);
  load_rows<T, D>(Os, static_cast<const T*>(a.dout), p, b, qs, q_off, nq, p.Sq, p.Hq, h, tid);
  for (int r = tid; r < BQ; r += 256) {
    const bool live = r < nq;
    const size_t li = ((size_t)b * p.Hq + h) * p.Sq + buf_row(p, qs, q_off + (live ? r : 0));
    Ls[r] = live ? a.lse[li] : 0.f;
    Dl[r] = live ? a.delta[li] : 0.f;
  }
  // this thread's part of dQ: row qi, dims dd + 4t
  const int qi = tid >> 2, dd = tid & 3;
  float dq[D / 4];
#pragma unroll
  for (int t = 0; t < D / 4; ++t) dq[t] = 0.f;

  KvIter it;
  kv_begin(p, qs, it);
  KvTile t;
  while (kv_next(p, q0 + nq - 1, BK, tpk, it, t)) {
    __syncthreads();
    load_rows<T, D>(Ks, static_cast<const T*>(a.k), p, b, t.slot, t.k0, t.nvalid, p.Skv, p.Hkv, g, tid);
    load_rows<T, D>(Vs, static_cast<const T*>(a.v), p, b, t.slot, t.k0, t.nvalid, p.Skv, p.Hkv, g, tid);
    __syncthreads();
    tile_p_ds<D>(Qs, Os, Ks, Vs, Ls, Dl, Ps, dSs, nq, t.nvalid, p.causal, q0, t.pos0, a.scale, tid);
    __syncthreads();
    for (int j = 0; j < t.nvalid; ++j) {
      const float sv = dSs[qi * PP + j];
#pragma unroll
      for (int u = 0; u < D / 4; ++u) dq[u] = fmaf(sv, Ks[j * DP + dd + 4 * u], dq[u]);
    }
  }
  if (qi < nq) {
    const size_t row = ((size_t)b * p.Sq + buf_row(p, qs, q_off + qi)) * p.Hq + h;
    if (a.dq_acc) {
#pragma unroll
      for (int u = 0; u < D / 4; ++u) a.dq_acc[row * D + dd + 4 * u] += a.scale * dq[u];
    } else {
      T* dqp = static_cast<T*>(a.dq) + row * D;
#pragma unroll
      for (int u = 0; u < D / 4; ++u) bst(dqp + dd + 4 * u, a.scale * dq[u]);
    }
  }
}

static size_t bwd_smem(int D) {
  using namespace bwd;
  return sizeof(float) * ((size_t)2 * BK * (D + 1) + (size_t)2 * BQ * (D + 1) + (size_t)2 * BQ * (BK + 1) + 2 * BQ);
}

template <typename T, int D>
static cudaError_t launch_bwd_t(const Plan& p, const BwdArgs& a, cudaStream_t st) {
  using namespace bwd;
  const size_t smem = bwd_smem(D);
  auto kk = attn_bwd_kv_kernel<T, D>;
  auto kq = attn_bwd_q_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kk<<<dim3(p.nkc * cdiv(p.C, BK), p.Hkv, p.B), 256, smem, st>>>(p, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kq<<<dim3(p.nqc * cdiv(p.C, BQ), p.Hq, p.B), 256, smem, st>>>(p, a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_delta(const void* out, const void* dout, float* delta, int B, int Hq, int S, int D, bool bf16,
                             cudaStream_t st) {
  const long long rows = (long long)B * S * Hq;
  const int per = 8;   // warps per block
  if (D == 64 || D == 128) {
    const long long blocks = (rows + 32LL * per - 1) / (32LL * per);   // 32 rows per warp
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    const unsigned nb = (unsigned)blocks;
    if (bf16) {
      auto o = static_cast<const __nv_bfloat16*>(out);
      auto g = static_cast<const __nv_bfloat16*>(dout);
      if (D == 128) bwd_delta_vec_kernel<__nv_bfloat16, 128><<<nb, 32 * per, 0, st>>>(o, g, delta, B, Hq, S);
      else bwd_delta_vec_kernel<__nv_bfloat16, 64><<<nb, 32 * per, 0, st>>>(o, g, delta, B, Hq, S);
    } else {
      auto o = static_cast<const float*>(out);
      auto g = static_cast<const float*>(dout);
      if (D == 128) bwd_delta_vec_kernel<float, 128><<<nb, 32 * per, 0, st>>>(o, g, delta, B, Hq, S);
      else bwd_delta_vec_kernel<float, 64><<<nb, 32 * per, 0, st>>>(o, g, delta, B, Hq, S);
    }
    return cudaGetLastError();
  }
  const long long blocks = (rows + per - 1) / per;   // one warp per row
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (bf16)
    bwd_delta_kernel<__nv_bfloat16><<<(unsigned)blocks, 32 * per, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), delta, B, Hq, S, D);
  else
    bwd_delta_kernel<float><<<(unsigned)blocks, 32 * per, 0, st>>>(static_cast<const float*>(out),
                                                                   static_cast<const float*>(dout), delta, B, Hq,
                                                                   S, D);
  return cudaGetLastError();
}

cudaError_t launch_bwd_simt(const Plan& p, const BwdArgs& a, bool bf16, cudaStream_t st) {
  if (p.D != 64 && p.D != 128) return cudaErrorNotSupported;
  if (bf16) return p.D == 64 ? launch_bwd_t<__nv_bfloat16, 64>(p, a, st) : launch_bwd_t<__nv_bfloat16, 128>(p, a, st);
  return p.D == 64 ? launch_bwd_t<float, 64>(p, a, st) : launch_bwd_t<float, 128>(p, a, st);
}

}  // namespace ra
