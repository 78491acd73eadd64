// CUDA-core (float32 FMA) ring attention, the step-state kernels and the
// (O, lse) merge.
//
// The SIMT kernel serves the float32 path, whose tolerance (1e-5) rules out
// the tensor cores, and is the GPU cross-check of the bf16 tensor-core path.
// It follows the same ring scheduler (ring_sched.h), for every split: for a
// 64-row query tile of one head it folds 64-key K/V tiles in the rank's ring
// order into the running (m, l, O) of "Lesson 8: Context Parallelism",
// section 3, then writes
// out = O / l and lse = m + ln l (ring mode) or folds its block result into
// the caller's state (step mode).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ring_sched.h"

namespace ra {

__device__ __forceinline__ float ld_val(const float* p) { return *p; }
__device__ __forceinline__ float ld_val(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_val(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_val(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Fold a block result (m_b, l_b, O_b normalised) into a stored state
// (m, l, O normalised) -- section 3's update applied to a whole block.
// Natural-log units.  A block with no allowed key (m_b = -inf) changes
// nothing.  Returns the new (m, l) and the two weights for O.
struct MergeW {
  float m, l, w_old, w_blk;
};
__device__ __forceinline__ MergeW merge_weights(float m_old, float l_old, float m_b, float l_b) {
  MergeW r;
  if (m_b == -CUDART_INF_F) {
    r.m = m_old; r.l = l_old; r.w_old = 1.f; r.w_blk = 0.f;
    return r;
  }
  const float mn = fmaxf(m_old, m_b);
  const float a = (m_old == -CUDART_INF_F) ? 0.f : expf(m_old - mn) * l_old;
  const float c = expf(m_b - mn) * l_b;
  r.m = mn;
  r.l = a + c;
  r.w_old = a / r.l;
  r.w_blk = c / r.l;
  return r;
}

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(Plan p, const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, T* __restrict__ out,
                                                        float* __restrict__ lse, float* __restrict__ m_st,
                                                        float* __restrict__ l_st, float* __restrict__ O_st,
                                                        float scale) {
  constexpr int BQ = 64, BK = 64, DP = D + 1, PP = BK + 1;
  extern __shared__ float smem[];
  float* Qs = smem;            // [BQ][DP]
  float* Ks = Qs + BQ * DP;    // [BK][DP]
  float* Vs = Ks + BK * DP;    // [BK][D]
  float* Ps = Vs + BK * D;     // [BQ][PP]

  const int tiles = cdiv(p.C, BQ);
  const int qslot = blockIdx.x / tiles;
  const int qt = blockIdx.x - qslot * tiles;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.Hq / p.Hkv);
  const int q_off = qt * BQ;
  const int nrows = imin(BQ, p.C - q_off);
  const int qrow0 = buf_row(p, qslot, q_off);
  const int qpos0 = q_pos_base(p, qslot) + q_off;
  const int qhi = qpos0 + nrows - 1;
  const int tid = threadIdx.x, r = tid >> 2, sub = tid & 3;
  const int qpos = qpos0 + r;

  for (int e = tid; e < BQ * D; e += 256) {
    const int rr = e / D, d = e - rr * D;
    float x = 0.f;
    if (rr < nrows) x = ld_val(q + (((size_t)b * p.Sq + buf_row(p, qslot, q_off + rr)) * p.Hq + h) * D + d);
    Qs[rr * DP + d] = x;
  }

  float m = -CUDART_INF_F, l = 0.f, o[D / 4];
#pragma unroll
  for (int j = 0; j < D / 4; ++j) o[j] = 0.f;

  KvIter it;
  kv_begin(p, qslot, it);
  KvTile t;
  const int tpc = cdiv(p.C, BK);
  while (kv_next(p, qhi, BK, tpc, it, t)) {
    __syncthreads();
    for (int e = tid; e < BK * D; e += 256) {
      const int kk = e / D, d = e - kk * D;
      float xk = 0.f, xv = 0.f;
      if (kk < t.nvalid) {
        const size_t off = (((size_t)b * p.Skv + buf_row(p, t.slot, t.k0 + kk)) * p.Hkv + g) * D + d;
        xk = ld_val(k + off);
        xv = ld_val(v + off);
      }
      Ks[kk * DP + d] = xk;
      Vs[kk * D + d] = xv;
    }
    __syncthreads();

    float s[BK / 4];
    float mx = -CUDART_INF_F;
#pragma unroll
    for (int i = 0; i < BK / 4; ++i) {
      const int key = sub + 4 * i;
      float acc = 0.f;
#pragma unroll 16
      for (int d = 0; d < D; ++d) acc = fmaf(Qs[r * DP + d], Ks[key * DP + d], acc);
      const bool ok = (key < t.nvalid) && (r < nrows) && (!p.causal || t.pos0 + key <= qpos);
      s[i] = ok ? acc * scale : -CUDART_INF_F;
      mx = fmaxf(mx, s[i]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    const float m_base = (m_new == -CUDART_INF_F) ? 0.f : m_new;
    const float alpha = (m == -CUDART_INF_F) ? 0.f : expf(m - m_base);
    float rs = 0.f;
#pragma unroll
    for (int i = 0; i < BK / 4; ++i) {
      const float pe = expf(s[i] - m_base);
      rs += pe;
      Ps[r * PP + sub + 4 * i] = pe;
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l = l * alpha + rs;
    m = m_new;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < D / 4; ++j) {
      const int d = sub + 4 * j;
      float acc = o[j] * alpha;
#pragma unroll 8
      for (int kk = 0; kk < BK; ++kk) acc = fmaf(Ps[r * PP + kk], Vs[kk * D + d], acc);
      o[j] = acc;
    }
  }

  const bool active = r < nrows;
  const int row = buf_row(p, qslot, q_off + r);
  if (p.mode == kModeRing) {
    if (!active) return;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    T* orow = out + (((size_t)b * p.Sq + row) * p.Hq + h) * D;
#pragma unroll
    for (int j = 0; j < D / 4; ++j) st_val(orow + sub + 4 * j, o[j] * inv);
    if (sub == 0) lse[((size_t)b * p.Hq + h) * p.Sq + row] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
  } else {
    const size_t si = ((size_t)b * p.Hq + h) * p.Sq + (active ? row : qrow0);
    const float m_old = m_st[si], l_old = l_st[si];
    const float m_b = (l > 0.f) ? m : -CUDART_INF_F;
    const MergeW w = merge_weights(m_old, l_old, m_b, l);
    float* orow = O_st + (((size_t)b * p.Sq + row) * p.Hq + h) * D;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (active) {
#pragma unroll
      for (int j = 0; j < D / 4; ++j) {
        const int d = sub + 4 * j;
        orow[d] = w.w_old * orow[d] + w.w_blk * (o[j] * inv);
      }
    }
    __syncwarp();  // every lane of the row has read (m, l) before they are replaced
    if (active && sub == 0) {
      m_st[si] = w.m;
      l_st[si] = w.l;
    }
  }
}

template <typename T, int D>
static cudaError_t launch_simt_t(const Plan& p, const void* q, const void* k, const void* v, void* out,
                                 float* lse, float* m, float* l, float* O, float scale, cudaStream_t st) {
  constexpr int BQ = 64, BK = 64;
  const size_t smem = sizeof(float) * ((size_t)BQ * (D + 1) + (size_t)BK * (D + 1) + (size_t)BK * D +
                                       (size_t)BQ * (BK + 1));
  auto kern = attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nqc * cdiv(p.C, BQ), p.Hq, p.B);
  kern<<<grid, 256, smem, st>>>(p, (const T*)q, (const T*)k, (const T*)v, (T*)out, lse, m, l, O, scale);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const Plan& p, bool bf16, const void* q, const void* k, const void* v, void* out,
                             float* lse, float* m, float* l, float* O, float scale, cudaStream_t st) {
  if (bf16) {
    return p.D == 64 ? launch_simt_t<__nv_bfloat16, 64>(p, q, k, v, out, lse, m, l, O, scale, st)
                     : launch_simt_t<__nv_bfloat16, 128>(p, q, k, v, out, lse, m, l, O, scale, st);
  }
  return p.D == 64 ? launch_simt_t<float, 64>(p, q, k, v, out, lse, m, l, O, scale, st)
                   : launch_simt_t<float, 128>(p, q, k, v, out, lse, m, l, O, scale, st);
}

// ---------------------------------------------------------------------------
// step state: initialise and finalise
// ---------------------------------------------------------------------------
__global__ void state_init_kernel(float* m, float* l, float* O, size_t n_ml, size_t n_o) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_ml; i += stride) {
    m[i] = -CUDART_INF_F;
    l[i] = 0.f;
  }
  float4* O4 = reinterpret_cast<float4*>(O);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_o / 4; i += stride)
    O4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

cudaError_t launch_state_init(float* m, float* l, float* O, int B, int Hq, int S_loc, int D, cudaStream_t st) {
  const size_t n_ml = (size_t)B * Hq * S_loc, n_o = n_ml * D;
  state_init_kernel<<<592, 256, 0, st>>>(m, l, O, n_ml, n_o);
  return cudaGetLastError();
}

template <typename T>
__global__ void state_finalize_kernel(const float* __restrict__ m, const float* __restrict__ l,
                                      const float* __restrict__ O, T* __restrict__ out, float* __restrict__ lse,
                                      int B, int Hq, int S, int D) {
  // one warp per (b, row, h)
  const size_t w = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const size_t n = (size_t)B * S * Hq;
  if (w >= n) return;
  const int h = (int)(w % Hq);
  const size_t bs = w / Hq;
  const int s = (int)(bs % S), b = (int)(bs / S);
  const size_t si = ((size_t)b * Hq + h) * S + s;
  const float lv = l[si];
  const bool live = lv > 0.f;
  for (int d = lane; d < D; d += 32) st_val(out + w * D + d, live ? O[w * D + d] : 0.f);
  if (lane == 0) lse[si] = live ? m[si] + logf(lv) : -CUDART_INF_F;
}

cudaError_t launch_state_finalize(const float* m, const float* l, const float* O, void* out, float* lse, int B,
                                  int Hq, int S, int D, bool bf16, cudaStream_t st) {
  const size_t warps = (size_t)B * S * Hq;
  const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
  if (bf16)
    state_finalize_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(m, l, O, (__nv_bfloat16*)out, lse, B, Hq, S, D);
  else
    state_finalize_kernel<float><<<blocks, 256, 0, st>>>(m, l, O, (float*)out, lse, B, Hq, S, D);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// (O, lse) merge, HBM-bound: one warp per (b, hq) row.  Lane j computes the
// weight e^(lse_p - lse) of parts p = j, j+32, ... once per block of 32 parts
// and the accumulation loop broadcasts it by shuffle.  Lanes own 4
// consecutive dims (one 16-byte load per part, a warp reads 512 contiguous
// bytes of a part), and kUnroll parts are loaded before any is used, so each
// lane keeps kUnroll independent loads in flight.  A part whose weight is 0
// (an empty part, lse = -inf) is not read.  The output row leaves as one
// vector store per lane.
// ---------------------------------------------------------------------------
namespace merge {
constexpr int kUnroll = 8;
// Small blocks (4 rows each): as blocks finish, the SMs are refilled a few
// rows at a time, so the last partial wave of a large merge stays short.
constexpr int kThreads = 128;
}

__device__ __forceinline__ void st_vec4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void st_vec4(__nv_bfloat16* p, float4 v) {
  uint2 w;
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  w.x = *reinterpret_cast<uint32_t*>(&lo);
  w.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = w;
}

__device__ __forceinline__ void fma4(float w, const float4& x, float4& acc) {
  acc.x = fmaf(w, x.x, acc.x);
  acc.y = fmaf(w, x.y, acc.y);
  acc.z = fmaf(w, x.z, acc.z);
  acc.w = fmaf(w, x.w, acc.w);
}

template <typename T>
__global__ void __launch_bounds__(merge::kThreads) merge_kernel(const float* __restrict__ part, const float* __restrict__ plse,
                                                    T* __restrict__ out, float* __restrict__ out_lse, int n_rows,
                                                    int P, int D) {
  using merge::kUnroll;
  const int w = (int)(((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= n_rows) return;
  const float* L = plse + (size_t)w * P;
  float mx = -CUDART_INF_F;
  for (int i = lane; i < P; i += 32) mx = fmaxf(mx, L[i]);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const bool live = mx != -CUDART_INF_F;
  const float base = live ? mx : 0.f;
  float z = 0.f;
  for (int i = lane; i < P; i += 32) z += expf(L[i] - base);
#pragma unroll
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float inv_z = live ? 1.f / z : 0.f;
  const float* Ob = part + (size_t)w * P * D;
  for (int d0 = 0; d0 < D; d0 += 128) {
    const int d = d0 + lane * 4;
    const bool mine = d < D;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < P; c += 32) {
      const int nb = min(32, P - c);
      const float wt = lane < nb ? expf(L[c + lane] - base) * inv_z : 0.f;
      const float* src = Ob + (size_t)c * D + d;
      int j = 0;
      for (; j + kUnroll <= nb; j += kUnroll) {
        float wj[kUnroll];
        float4 x[kUnroll];
if (mine) {
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) x[u] = __ldg(reinterpret_cast<const float4*>(src + (size_t)(j + u) * D));
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) wj[u] = __shfl_sync(0xffffffffu, wt, j + u);
        if (mine) {
#pragma unroll
          for (int u = 0; u < kUnroll; ++u)
            if (wj[u] != 0.f) fma4(wj[u], x[u], acc);   // an empty part's O may hold anything
        }
      }
      for (; j < nb; ++j) {
        const float wj = __shfl_sync(0xffffffffu, wt, j);
        if (mine && wj != 0.f) fma4(wj, __ldg(reinterpret_cast<const float4*>(src + (size_t)j * D)), acc);
      }
    }
    if (mine) st_vec4(out + (size_t)w * D + d, acc);
  }
  if (lane == 0 && out_lse) out_lse[w] = live ? mx + logf(z) : -CUDART_INF_F;
}

cudaError_t launch_merge(const float* part, const float* plse, void* out, float* out_lse, int B, int Hq, int P,
                         int D, bool bf16, cudaStream_t st) {
  const int rows = B * Hq;
  const unsigned blocks = (unsigned)(((size_t)rows * 32 + merge::kThreads - 1) / merge::kThreads);
  if (bf16)
    merge_kernel<__nv_bfloat16><<<blocks, merge::kThreads, 0, st>>>(part, plse, (__nv_bfloat16*)out, out_lse, rows,
                                                                    P, D);
  else
    merge_kernel<float><<<blocks, merge::kThreads, 0, st>>>(part, plse, (float*)out, out_lse, rows, P, D);
  return cudaGetLastError();
}

}  // namespace ra
