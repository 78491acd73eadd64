// Split-KV single-token decode on the tensor cores ("NVIDIA unveils Helix
// Parallelism", Phase 1: the KV cache sharded along the sequence; each shard
// yields a partial result that is merged afterwards).
//
// Work unit = (chunk p, batch b, kv head g, sub-split s): RPS consecutive rows
// of one chunk.  A persistent grid (one CTA per SM) walks the units in chunk
// order, so the always-full early chunks come first and the ragged tails of
// the sequences last.  The G query heads of a kv head share every K/V row, so
// a 128-row K/V tile is one pair of small tcgen05 products (the heads padded
// to the smallest N of the instruction, 16):
//   S^T = K Q^T      M = 128 keys,  N = 16 heads, K = 128 dims  (K, Q K-major)
//   O^T += V^T P^T   M = 128 dims,  N = 16 heads, K = 128 keys  (V MN-major)
// with S^T and O^T in tensor memory.  Warp roles:
//   warps 0-3  softmax group: thread t owns tensor-memory lane t, i.e. key
//              row t of S^T and dimension t of O^T; it turns its G scores
//              into weights against a per-head base shared by the whole CTA
//              and writes them (bf16) as P^T, the B operand of O^T, in
//              shared memory;
//   warp 4     TMA producer: the unit's query rows (128-byte swizzle, padded
//              rows stay zero), then K and V tiles into a 3-stage ring;
//   warp 5     MMA issuer and tensor-memory owner: S(j+1) is issued before
//              the O^T update of tile j, so the softmax of tile j+1 overlaps it.
//   warp 6     merge warp (one-launch decode only): counts each chunk whose
//              final partial this CTA wrote and merges on the count that
//              completes the P chunks, off the softmax group's path.
// The online softmax of "Lesson 8: Context Parallelism", section 3, with a
// lazy base: a head's base moves only when one of its scores exceeds it by
// more than 2^8 (a block-wide OR decides, and only then are the tile maxima
// reduced and O^T rescaled), which is exact because l and O share the base.
// Two sums are kept, as in the prefill kernel: the fp32 sum of the weights
// (gives lse) and the sum of their bf16 values (normalises O, so that the
// weights applied to V sum to one).
// At the end of a unit the thread of dimension d holds O[h][d] for the G
// heads.  A chunk covered by one sub-split writes its partial directly;
// otherwise every sub-split writes to the workspace and the last CTA to
// arrive (atomic counter, reset by that CTA) folds them into the chunk's
// partial.  With an output buffer the merge runs in the same launch: the CTA
// that finishes the last of the P chunks of a (sequence, kv head) -- a second
// counter, reset the same way -- combines the P partials into out and lse, in
// its merge warp.
// The valid rows of a chunk come from the sequence length (chunk p holds
// positions [p*C, (p+1)*C)) or, for a cache filled by the round-robin append
// of "NVIDIA unveils Helix Parallelism" (KV cache growth), from the chunk's
// own fill count.  The kernel is HBM-bound: each valid K/V byte is read once.
// Every wait is bounded; the softmax warps leave together (block-wide ORs).
#include <cuda_bf16.h>
#include <type_traits>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ptx.cuh"

namespace ra {

namespace dec {
constexpr int DM = 128;                     // head dimensions a tile row holds (D = 64 uses the first half)
constexpr int BN = 128;                     // K/V rows per tile (the M of S^T)
constexpr int NQ = 16;                      // query heads padded to the smallest N of the product
constexpr int NST = 3;                      // K/V stages
constexpr int RPS = 8192;                   // rows per sub-split (a multiple of BN)
constexpr int SLAB = BN * 64 * 2;           // one 128-row x 64-column bf16 box (16 KB)
constexpr int TILE_BYTES = BN * DM * 2;     // one K or V tile (32 KB)
constexpr int QSLAB = NQ * 128;             // 16 rows x 64 columns of bf16 (2 KB)
constexpr int NSW = 4;                      // softmax warps
constexpr int CT = 32 * NSW;                // softmax threads
constexpr int THREADS = CT + 96;            // + producer warp + MMA warp + merge warp
constexpr uint32_t TMEM_COLS = 64;          // S^T (2 x 16 columns), O^T (16 columns)
constexpr float LAZY = 8.f;                 // log2 of the largest tolerated growth before rescaling
static_assert(RPS % BN == 0, "tiles never straddle two sub-splits");
}  // namespace dec

struct DecGeom {
  int Cd;      // rows per chunk
  int nsub;    // sub-splits per chunk
  int units;
};

// Valid rows of chunk p of sequence b (always in [0, Cd]; out-of-range
// lengths are clamped, never trusted): from the chunk's own fill count
// (kShard) or from the sequence length.
template <bool kShard>
__device__ __forceinline__ int chunk_rows(const DecodeArgs& a, const DecodeExtra& x, int Cd, int b, int p) {
  if constexpr (kShard) return min(max(x.shard_lens[b * a.P + p], 0), Cd);
  const int len = min(max(a.seqlens[b], 0), a.Smax);
  return max(0, min(len - p * Cd, Cd));
}
// One past the last valid row of chunk p (a row index of the whole cache).
template <bool kShard>
__device__ __forceinline__ int chunk_end(const DecodeArgs& a, const DecodeExtra& x, int Cd, int b, int p) {
  if constexpr (kShard) return p * Cd + min(max(x.shard_lens[b * a.P + p], 0), Cd);
  const int len = min(max(a.seqlens[b], 0), a.Smax);
  return min(len, (p + 1) * Cd);
}

// Counts one finished chunk of (b, kv head g) with an acquire-release atomic
// (after a barrier that follows the CTA's writes of that chunk's partial, so
// the release publishes them).  True for the arrival that completes the P
// chunks; that arrival resets the counter for the next call.
__device__ __forceinline__ bool count_chunk(const DecodeArgs& a, const DecodeExtra& x, int b, int g) {
  unsigned int* ctr = x.ws_done + (size_t)b * a.Hkv + g;
  const bool last = atom_add_acq_rel_gpu(ctr, 1u) == (unsigned int)(a.P - 1);
  if (last) atomicExch(ctr, 0u);
  return last;
}

// The merge of the P partials of (b, kv head g) for its G query heads, done
// by one warp of the CTA whose arrival completed the count of finished chunks
// (that arrival's acquire, followed by __syncwarp, makes every chunk's partial
// visible here).  The update of "Lesson 8: Context Parallelism", section 3,
// applied to whole partial states:
//   lse = m* + ln sum_p e^(lse_p - m*),  out = sum_p e^(lse_p - lse) O_p.
// Heads h0 .. h0 + G - 1 of the group (query heads (b, g * Gq + h0 + i)); the
// group is merged in passes of at most 8 heads, so that the per-head values of
// a pass stay in registers (16 heads at once spilled).
template <int G, int DH>
__device__ __noinline__ void merge_heads(const DecodeArgs& a, const DecodeExtra& x, size_t bh0, int lane) {
  constexpr int D = DH;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(x.out);
  // lse of chunk (q0 + lane) of every head; the first 32 chunks stay in registers
  auto lse_at = [&](int h, int q) { return q < a.P ? __ldcg(a.part_lse + (bh0 + h) * a.P + q) : -CUDART_INF_F; };
  float lv[G], mx[G], L[G];
#pragma unroll
  for (int h = 0; h < G; ++h) mx[h] = lv[h] = lse_at(h, lane);
  for (int q0 = 32; q0 < a.P; q0 += 32)
#pragma unroll
    for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], lse_at(h, q0 + lane));
#pragma unroll
  for (int off = 16; off; off >>= 1)
#pragma unroll
    for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], off));
#pragma unroll
  for (int h = 0; h < G; ++h) L[h] = mx[h] == -CUDART_INF_F ? 0.f : expf(lv[h] - mx[h]);
  for (int q0 = 32; q0 < a.P; q0 += 32)
#pragma unroll
    for (int h = 0; h < G; ++h)
      if (mx[h] != -CUDART_INF_F) L[h] += expf(lse_at(h, q0 + lane) - mx[h]);
#pragma unroll
  for (int off = 16; off; off >>= 1)
#pragma unroll
    for (int h = 0; h < G; ++h) L[h] += __shfl_xor_sync(0xffffffffu, L[h], off);
  float inv[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    inv[h] = L[h] > 0.f ? 1.f / L[h] : 0.f;
    if (lane == 0 && x.out_lse) x.out_lse[bh0 + h] = L[h] > 0.f ? mx[h] + logf(L[h]) : -CUDART_INF_F;
  }
  // lane owns dims lane + 32k of every head; the weights of 32 chunks at a time sit
  // one per lane and reach the others by shuffles; the loads of a chunk are independent
  float acc[G][D / 32];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < D / 32; ++k) acc[h][k] = 0.f;
  for (int q0 = 0; q0 < a.P; q0 += 32) {
    float w[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float v = q0 == 0 ? lv[h] : lse_at(h, q0 + lane);
      w[h] = inv[h] > 0.f && v != -CUDART_INF_F ? expf(v - mx[h]) * inv[h] : 0.f;
    }
    const int n = min(32, a.P - q0);
#pragma unroll 4
    for (int j = 0; j < n; ++j) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float wj = __shfl_sync(0xffffffffu, w[h], j);
        const float* row = a.partials + ((bh0 + h) * a.P + q0 + j) * D + lane;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) acc[h][k] = fmaf(wj, __ldcg(row + 32 * k), acc[h][k]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < D / 32; ++k) out[(bh0 + h) * D + lane + 32 * k] = __float2bfloat16_rn(acc[h][k]);
}

template <int G, int DH>
__device__ __forceinline__ void merge_bg(const DecodeArgs& a, const DecodeExtra& x, int b, int g, int lane) {
  constexpr int GP = G > 8 ? 8 : G;   // heads per pass
  __syncwarp();   // lane 0's acquire covers the warp from here on
  for (int h0 = 0; h0 < G; h0 += GP) merge_heads<GP, DH>(a, x, (size_t)b * a.Hq + g * G + h0, lane);
}

// Called by the merge warp (all lanes) for a chunk whose final partial this CTA
// wrote: one lane counts the chunk; the arrival that completes the count of
// (b, g) merges it in this warp.  The softmax group does not wait.
template <int G, int DH>
__device__ __forceinline__ void chunk_final_count(const DecodeArgs& a, const DecodeExtra& x, int b, int g, int lane) {
  int last = 0;
  if (lane == 0) last = count_chunk(a, x, b, g);
  if (__shfl_sync(0xffffffffu, last, 0)) {
    __syncwarp();   // lane 0's acquire covers the warp
    merge_bg<G, DH>(a, x, b, g, lane);
  }
}

template <int G>
struct DecSmem {
  alignas(1024) uint8_t kv[dec::NST][2][dec::TILE_BYTES];   // K, V tiles: 2 slabs of 128 rows x 128 B each
  alignas(1024) uint8_t q[2][2 * dec::QSLAB];                 // padded query rows, by unit parity
  alignas(1024) uint8_t pt[2][2 * dec::QSLAB];                // P^T (16 head rows x 128 keys), by tile parity
  float red[2][dec::NSW][G];                                  // cross-warp reductions
  alignas(8) uint64_t kv_full[dec::NST], kv_empty[dec::NST];
  alignas(8) uint64_t q_full[2], q_empty[2];
  alignas(8) uint64_t s_full[2], s_free[2], p_full[2], o_done[2];
  alignas(8) uint64_t o_full, o_free, teardown;
  // finished chunks handed from the softmax group to the merge warp (kMerge): a ring of 4 slots
  int q_b[4], q_g[4];
  alignas(8) uint64_t q_post[4], q_done[4];
  uint32_t tmem_base;
  int is_last;      // set by one thread between two softmax-group barriers, read by all after the second
  int abort_flag;
};

// Instruction descriptor of kind::f16 (bf16 A and B, f32 accumulation) with
// the major-ness of both operands (bit 15: A, bit 16: B; 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_f16_ab(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// G consecutive 32-bit columns of this warp's 32 lanes (G = 1, 2, 4, 8, 16)
template <int G>
__device__ __forceinline__ void tmem_ld_g(uint32_t taddr, float (&v)[G]) {
  uint32_t r[G];
  if constexpr (G == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
  } else if constexpr (G == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
  } else if constexpr (G == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr));
  } else if constexpr (G == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else {
    static_assert(G == 16, "G");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  }
#pragma unroll
  for (int i = 0; i < G; ++i) v[i] = __uint_as_float(r[i]);
}
template <int G>
__device__ __forceinline__ void tmem_st_g(uint32_t taddr, const float (&v)[G]) {
  uint32_t r[G];
#pragma unroll
  for (int i = 0; i < G; ++i) r[i] = __float_as_uint(v[i]);
  if constexpr (G == 1) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r[0]) : "memory");
  } else if constexpr (G == 2) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1,%2};" ::"r"(taddr), "r"(r[0]), "r"(r[1])
                 : "memory");
  } else if constexpr (G == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
  } else if constexpr (G == 8) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
  } else {
    static_assert(G == 16, "G");
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Unit u -> (b, kv head g, chunk p, sub-split) and its rows [r0, r1) (r0 >= r1: nothing to read).
struct DecUnit {
  int b, g, p, sub, r0, r1, ntiles;
};
template <bool kShard>
__device__ __forceinline__ DecUnit dec_unit(const DecodeArgs& a, const DecodeExtra& x, const DecGeom& geo, int u) {
  DecUnit U;
  int t = u;
  U.sub = t % geo.nsub; t /= geo.nsub;
  U.g = t % a.Hkv; t /= a.Hkv;
  U.b = t % a.B;
  U.p = t / a.B;
  U.r0 = U.p * geo.Cd + U.sub * dec::RPS;
  U.r1 = min(U.r0 + dec::RPS, chunk_end<kShard>(a, x, geo.Cd, U.b, U.p));
  U.ntiles = U.r0 < U.r1 ? (U.r1 - U.r0 + dec::BN - 1) / dec::BN : 0;
  return U;
}

// kMerge: the launch also merges the partials (a.out != null); kShard: valid
// rows come from per-chunk fill counts (a.shard_lens != null).  Separate
// instantiations, so that the plain partial kernel carries none of their code.
template <int G, int DH, bool kMerge, bool kShard>
__global__ void __launch_bounds__(dec::THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, DecodeArgs a, DecGeom geo, DecodeExtra x) {
  using namespace dec;
  extern __shared__ uint8_t smem_raw[];
  DecSmem<G>& sm = *reinterpret_cast<DecSmem<G>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  unsigned int* err = a.err;

  // the padded query rows and the padded P^T rows stay zero (never written again)
  {
    uint4* z = reinterpret_cast<uint4*>(&sm.q[0][0]);
    constexpr int n16 = (int)((sizeof(sm.q) + sizeof(sm.pt)) / 16);
    for (int i = threadIdx.x; i < n16; i += THREADS) z[i] = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (DH == 64) {
      // D = 64: the V tiles' second 64-column block is the zero upper half of the M = 128
      // product O^T += V^T P^T (never written by TMA)
      for (int st = 0; st < NST; ++st) {
        uint4* zv = reinterpret_cast<uint4*>(sm.kv[st][1] + SLAB);
        for (int i = threadIdx.x; i < SLAB / 16; i += THREADS) zv[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&sm.kv_full[s]), 1);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.q_full[i]), 1);
      mbar_init(smem_u32(&sm.q_empty[i]), 1);
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.s_free[i]), CT);
      mbar_init(smem_u32(&sm.p_full[i]), CT);
      mbar_init(smem_u32(&sm.o_done[i]), 1);
    }
    mbar_init(smem_u32(&sm.o_full), 1);
    mbar_init(smem_u32(&sm.o_free), CT);
    mbar_init(smem_u32(&sm.teardown), 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&sm.q_post[i]), 1);
      mbar_init(smem_u32(&sm.q_done[i]), 1);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == NSW + 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == NSW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol_kv = l2_policy_evict_first();
      const uint64_t pol_q = l2_policy_evict_last();
      uint32_t cnt = 0, nq = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < geo.units && ok; u += gridDim.x) {
        const DecUnit U = dec_unit<kShard>(a, x, geo, u);
        if (U.ntiles == 0) continue;
        const int qb = nq & 1;
        if (nq >= 2 && !mbar_wait(smem_u32(&sm.q_empty[qb]), ((nq >> 1) - 1) & 1u, abort_flag, kWaitQEmpty, err)) {
          ok = false;
          break;
        }
        const uint32_t qf = smem_u32(&sm.q_full[qb]);
        mbar_arrive_expect_tx(qf, G * DH * 2);
        for (int sl = 0; sl < DH / 64; ++sl)
          tma_load_4d(smem_u32(sm.q[qb]) + sl * QSLAB, &tmQ, qf, sl * 64, 0, U.b * a.Hq + U.g * G, 0, pol_q);
        ++nq;
        for (int j = 0; j < U.ntiles; ++j) {
          const int s = cnt % NST;
          if (!mbar_wait(smem_u32(&sm.kv_empty[s]), ((cnt / NST) & 1u) ^ 1u, abort_flag, kWaitDecodeEmpty, err)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm.kv_full[s]);
          mbar_arrive_expect_tx(fb, 2 * BN * DH * 2);
          const int row = U.r0 + j * BN;
          for (int sl = 0; sl < DH / 64; ++sl) {
            tma_load_4d(smem_u32(sm.kv[s][0]) + sl * SLAB, &tmK, fb, sl * 64, U.g, row, U.b, pol_kv);
            tma_load_4d(smem_u32(sm.kv[s][1]) + sl * SLAB, &tmV, fb, sl * 64, U.g, row, U.b, pol_kv);
          }
          ++cnt;
        }
      }
      // do not leave while copies are still landing in shared memory
      for (uint32_t c = (cnt > (uint32_t)NST ? cnt - NST : 0); c < cnt; ++c)
        mbar_wait(smem_u32(&sm.kv_full[c % NST]), (c / NST) & 1u, nullptr, kWaitTeardown, err);
      for (uint32_t c = (nq > 2u ? nq - 2u : 0u); c < nq; ++c)
        mbar_wait(smem_u32(&sm.q_full[c & 1]), (c >> 1) & 1u, nullptr, kWaitTeardown, err);
    }
  } else if (warp == NSW + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS[2] = {tmem, tmem + 16}, tO = tmem + 32;
      constexpr uint32_t idS = idesc_f16_ab(BN, NQ, false, false);   // S^T = K Q^T
      constexpr uint32_t idPV = idesc_f16_ab(DM, NQ, true, false);   // O^T += V^T P^T (D = 64: upper half zero)
      uint32_t cnt = 0, nq = 0, tj = 0, nu = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < geo.units && ok; u += gridDim.x) {
        const DecUnit U = dec_unit<kShard>(a, x, geo, u);
        if (U.ntiles == 0) continue;
        const int qb = nq & 1;
        if (!mbar_wait(smem_u32(&sm.q_full[qb]), (nq >> 1) & 1u, abort_flag, kWaitQFull, err)) { ok = false; break; }
        tc_fence_after();
        ++nq;
        const uint64_t qdesc = sw128_desc(smem_u32(sm.q[qb]), 16, 1024);
        for (int j = 0; j <= U.ntiles && ok; ++j) {
          if (j < U.ntiles) {
            // S^T(j) into buffer t & 1, once the softmax has read S^T(t - 2) from it
            const uint32_t c = cnt + j, s = c % NST, t = tj + j, sb = t & 1u;
            if (!mbar_wait(smem_u32(&sm.kv_full[s]), (c / NST) & 1u, abort_flag, kWaitDecodeFull, err)) {
              ok = false;
              break;
            }
            if (t >= 2 && !mbar_wait(smem_u32(&sm.s_free[sb]), ((t >> 1) - 1) & 1u, abort_flag, kWaitSFull, err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kdesc = sw128_desc(smem_u32(sm.kv[s][0]), 16, 1024);
#pragma unroll
            for (int k = 0; k < DH / 16; ++k)
              mma_ss(tS[sb], kdesc + ((((k >> 2) * SLAB) + (k & 3) * 32) >> 4),
                     qdesc + ((((k >> 2) * QSLAB) + (k & 3) * 32) >> 4), idS, k > 0 ? 1u : 0u);
            mma_commit(smem_u32(&sm.s_full[sb]));
            if (j == U.ntiles - 1) mma_commit(smem_u32(&sm.q_empty[qb]));
          }
          if (j > 0) {
            // O^T += V^T(j-1) P^T(j-1)
            const uint32_t c = cnt + j - 1, s = c % NST, t = tj + j - 1, pb = t & 1u;
            if (!mbar_wait(smem_u32(&sm.p_full[pb]), (t >> 1) & 1u, abort_flag, kWaitPFull, err)) {
              ok = false;
              break;
            }
            if (j == 1 && nu > 0 &&
                !mbar_wait(smem_u32(&sm.o_free), (nu - 1) & 1u, abort_flag, kWaitOFinal, err)) {   // O^T was read
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t vdesc = sw128_desc(smem_u32(sm.kv[s][1]), SLAB, 1024);
            const uint64_t pdesc = sw128_desc(smem_u32(sm.pt[pb]), 16, 1024);
#pragma unroll
            for (int k = 0; k < BN / 16; ++k)
              mma_ss(tO, vdesc + ((k * 16 * 128) >> 4), pdesc + ((((k >> 2) * QSLAB) + (k & 3) * 32) >> 4), idPV,
                     (j > 1 || k > 0) ? 1u : 0u);
            mma_commit(smem_u32(&sm.o_done[pb]));
            mma_commit(smem_u32(&sm.kv_empty[s]));
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&sm.o_full));
        cnt += U.ntiles;
        tj += U.ntiles;
        ++nu;
      }
      // every MMA issued so far must be complete before tensor memory is freed
      mma_commit(smem_u32(&sm.teardown));
      mbar_wait(smem_u32(&sm.teardown), 0, nullptr, kWaitTeardown, err);
    }
  } else if (warp < NSW) {
    // ------------------------------------------------------------ softmax group
    const int row = threadIdx.x;                             // key row of S^T, dimension of O^T
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tmem + lane_off + 32;
    const float sl2 = a.scale * 1.4426950408889634f;
    // this thread's P^T entries: row h, key `row` (128-byte swizzle: 16-byte chunk XOR row)
    const uint32_t pt_base = (uint32_t)((row >> 6) * QSLAB + (row & 7) * 2);
    const int kc = (row & 63) >> 3;
    uint32_t tj = 0, nu = 0;
    bool ok = true;
    // kMerge: thread 0 hands each chunk whose final partial this CTA wrote (after the barrier
    // that follows those writes) to the merge warp, which counts it and merges on the count
    // that completes the P chunks; a sentinel (b = -1) ends the merge warp's loop
    uint32_t nposted = 0;
    auto post = [&](int b, int g) {
      const uint32_t k = nposted & 3u;
      if (nposted >= 4 && !mbar_wait(smem_u32(&sm.q_done[k]), ((nposted >> 2) - 1) & 1u, abort_flag, kWaitPFull, err))
        return;
      sm.q_b[k] = b;
      sm.q_g[k] = g;
      mbar_arrive(smem_u32(&sm.q_post[k]));
      ++nposted;
    };
    for (int u = blockIdx.x; u < geo.units; u += gridDim.x) {
      const DecUnit U = dec_unit<kShard>(a, x, geo, u);
      const int nvalid_chunk = chunk_rows<kShard>(a, x, geo.Cd, U.b, U.p);
      const int n_live = (nvalid_chunk + RPS - 1) / RPS;
      if (nvalid_chunk == 0) {
        if (U.sub == 0) {
          for (int e = row; e < G * DH; e += CT) {
            const int h = e / DH, d = e - h * DH;
            a.partials[((size_t)(U.b * a.Hq + U.g * G + h) * a.P + U.p) * DH + d] = 0.f;
          }
          if (row < G) a.part_lse[(size_t)(U.b * a.Hq + U.g * G + row) * a.P + U.p] = -CUDART_INF_F;
          if constexpr (kMerge) {
            named_bar_sync(1, CT);   // the chunk's partial is written before it is counted
            if (row == 0) post(U.b, U.g);
          }
        }
        continue;
      }
      if (U.ntiles == 0) continue;

      // per head: base m (the same in every thread), fp32 sum l and bf16-value sum lt of this thread's rows
      float m[G], l[G], lt[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -CUDART_INF_F;
        l[h] = 0.f;
        lt[h] = 0.f;
      }
      for (int j = 0; j < U.ntiles; ++j) {
        const uint32_t t = tj + j, sb = t & 1u;
        bool good = mbar_wait(smem_u32(&sm.s_full[sb]), (t >> 1) & 1u, abort_flag, kWaitSFull, err);
        // P^T buffer sb is free once O^T has taken P^T(t - 2)
        if (good && t >= 2) good = mbar_wait(smem_u32(&sm.o_done[sb]), ((t >> 1) - 1) & 1u, abort_flag, kWaitPFull, err);
        if (named_bar_any(1, CT, !good || !ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float xs[G];
        tmem_ld_g<G>(tmem + lane_off + 16 * sb, xs);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.s_free[sb]));
        const bool valid = U.r0 + j * BN + row < U.r1;
        if (!valid) {
          // a row past the valid ones (a cache's unwritten rows may hold any bits): its weight is 0,
          // and its V row is zeroed so that the product never meets 0 x NaN
          uint4* vr = reinterpret_cast<uint4*>(sm.kv[t % NST][1] + row * 128);
#pragma unroll
          for (int sl = 0; sl < 2; ++sl)
#pragma unroll
            for (int c = 0; c < 8; ++c) vr[sl * (SLAB / 16) + c] = make_uint4(0u, 0u, 0u, 0u);
        }
        bool exceed = false;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          xs[h] = valid ? xs[h] * sl2 : -CUDART_INF_F;
          exceed |= xs[h] > m[h] + LAZY;
        }
        if (named_bar_any(1, CT, exceed)) {
          // move the base of the heads whose tile maximum exceeds it (always on a unit's first tile)
          const int rb = j & 1;   // reduction buffer: the next use is two barriers away
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float mw = warp_max(xs[h]);
            if (lane == 0) sm.red[rb][warp][h] = mw;
          }
          named_bar_sync(1, CT);
          float alpha[G];
          bool moved = false;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float mt = sm.red[rb][0][h];
#pragma unroll
            for (int w = 1; w < NSW; ++w) mt = fmaxf(mt, sm.red[rb][w][h]);
            alpha[h] = 1.f;
            if (mt > m[h] + LAZY) {
              alpha[h] = m[h] == -CUDART_INF_F ? 0.f : ex2(m[h] - mt);
              m[h] = mt;
              moved = true;
            }
            l[h] *= alpha[h];
            lt[h] *= alpha[h];
          }
          if (j > 0 && moved) {   // the same decision in every thread (from the shared maxima)
            // O^T holds this unit's earlier tiles: rescale its columns once O^T(t - 1) is complete
            const uint32_t tp = t - 1;
            if (!mbar_wait(smem_u32(&sm.o_done[tp & 1u]), (tp >> 1) & 1u, abort_flag, kWaitPFull, err)) ok = false;
            __syncwarp();
            tc_fence_after();
            float o[G];
            tmem_ld_g<G>(tO, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] *= alpha[h];
            tmem_st_g<G>(tO, o);
            tmem_wait_st();
          }
        }
        // weights against the base; P^T(t) in shared memory for the tensor cores
        uint8_t* ptb = sm.pt[sb];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pw = m[h] == -CUDART_INF_F ? 0.f : ex2(xs[h] - m[h]);
          const uint32_t bits = pack_bf16x2(pw, 0.f) & 0xffffu;
          l[h] += pw;
          lt[h] += __uint_as_float(bits << 16);
          *reinterpret_cast<uint16_t*>(ptb + pt_base + (h >> 3) * 1024 + (h & 7) * 128 + ((kc ^ (h & 7)) << 4)) =
              (uint16_t)bits;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.p_full[sb]));
      }
      if (!ok) break;
      tj += U.ntiles;

      // ---- the unit's result: O^T after its last product, sums reduced over the 128 threads
      const bool fin = mbar_wait(smem_u32(&sm.o_full), nu & 1u, abort_flag, kWaitOFinal, err);
      if (named_bar_any(1, CT, !fin)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float o[G];
      tmem_ld_g<G>(tO, o);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.o_free));
      ++nu;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ls = warp_sum(l[h]), lts = warp_sum(lt[h]);
        if (lane == 0) {
          sm.red[0][warp][h] = ls;
          sm.red[1][warp][h] = lts;
        }
      }
      named_bar_sync(1, CT);
      float* ws_unit = a.ws_part + ((((size_t)(U.b * a.Hkv + U.g) * a.P + U.p) * geo.nsub + U.sub) * G) * (DH + 1);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float L = 0.f, LT = 0.f;
#pragma unroll
        for (int w = 0; w < NSW; ++w) {
          L += sm.red[0][w][h];
          LT += sm.red[1][w][h];
        }
        const float od = o[h] / LT;
        const float lse = (m[h] + log2f(L)) * 0.6931471805599453f;
        if (row >= DH) continue;   // D = 64: the upper half of O^T is padding
        if (n_live == 1) {
          a.partials[((size_t)(U.b * a.Hq + U.g * G + h) * a.P + U.p) * DH + row] = od;
          if (row == 0) a.part_lse[(size_t)(U.b * a.Hq + U.g * G + h) * a.P + U.p] = lse;
        } else {
          ws_unit[h * (DH + 1) + row] = od;
          if (row == 0) ws_unit[h * (DH + 1) + DH] = lse;
        }
      }
      named_bar_sync(1, CT);   // sm.red is free again
      if (n_live > 1) {
        if (row == 0) {
          unsigned int* ctr = a.ws_count + (size_t)(U.b * a.Hkv + U.g) * a.P + U.p;
          const unsigned int old = atom_add_acq_rel_gpu(ctr, 1u);
          const int last = (old == (unsigned int)(n_live - 1));
          if (last) atomicExch(ctr, 0u);       // leave the counter at zero for the next call
          sm.is_last = last;
        }
        named_bar_sync(1, CT);
        if (sm.is_last) {
          const float* ws_chunk = a.ws_part + (((size_t)(U.b * a.Hkv + U.g) * a.P + U.p) * geo.nsub) * G * (DH + 1);
          for (int e = row; e < G * DH; e += CT) {
            const int h = e / DH, d = e - h * DH;
            float mx = -CUDART_INF_F;
            for (int s2 = 0; s2 < n_live; ++s2) mx = fmaxf(mx, __ldcg(ws_chunk + (s2 * G + h) * (DH + 1) + DH));
            float Lsum = 0.f, acc = 0.f;
            for (int s2 = 0; s2 < n_live; ++s2) {
              const float* r = ws_chunk + (s2 * G + h) * (DH + 1);
              const float w = expf(__ldcg(r + DH) - mx);
              Lsum += w;
              acc = fmaf(w, __ldcg(r + d), acc);
            }
            a.partials[((size_t)(U.b * a.Hq + U.g * G + h) * a.P + U.p) * DH + d] = acc / Lsum;
            if (d == 0) a.part_lse[(size_t)(U.b * a.Hq + U.g * G + h) * a.P + U.p] = mx + logf(Lsum);
          }
        }
      }
      // this CTA wrote the chunk's final partial: directly, or as the last sub-split to arrive
      const bool chunk_final = n_live == 1 || sm.is_last;
      if (named_bar_any(1, CT, !ok || *abort_flag)) break;
      if constexpr (kMerge)
        if (chunk_final && row == 0) post(U.b, U.g);
    }
    if constexpr (kMerge)
      if (row == 0) post(-1, 0);
  } else if (warp == NSW + 2) {
    // ------------------------------------------------------------ merge warp (kMerge)
    if constexpr (kMerge) {
      for (uint32_t n = 0;; ++n) {
        const uint32_t k = n & 3u;
        const bool got = mbar_wait(smem_u32(&sm.q_post[k]), (n >> 2) & 1u, abort_flag, kWaitPFull, err);
        if (!__all_sync(0xffffffffu, got)) break;
        const int b = sm.q_b[k], g = sm.q_g[k];
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.q_done[k]));   // the slot is free again
        if (b < 0) break;
        chunk_final_count<G, DH>(a, x, b, g, lane);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == NSW + 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Workspace: sub-split results | per-chunk arrival counters | per-(b, kv head)
// finished-chunk counters, each part 256-byte aligned.
static size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Smax, int D, int P) {
  if (B < 1 || Hq < 1 || Hkv < 1 || P < 1 || Smax < P || D < 1 || Hq % Hkv) return 0;
  const int G = Hq / Hkv;
  const int Cd = Smax / P;
  const int nsub = (Cd + dec::RPS - 1) / dec::RPS;
  const size_t chunks = (size_t)B * Hkv * P;
  return round256(chunks * nsub * G * (D + 1) * sizeof(float)) + round256(chunks * sizeof(unsigned int)) +
         round256((size_t)B * Hkv * sizeof(unsigned int));
}

void decode_workspace_split(void* ws, int B, int Hq, int Hkv, int Smax, int D, int P, float** part,
                            unsigned int** count, unsigned int** done) {
  const int G = Hq / Hkv;
  const int Cd = Smax / P;
  const int nsub = (Cd + dec::RPS - 1) / dec::RPS;
  const size_t chunks = (size_t)B * Hkv * P;
  const size_t b_part = round256(chunks * nsub * G * (D + 1) * sizeof(float));
  const size_t b_count = round256(chunks * sizeof(unsigned int));
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  *part = reinterpret_cast<float*>(base);
  *count = reinterpret_cast<unsigned int*>(base + b_part);
  *done = reinterpret_cast<unsigned int*>(base + b_part + b_count);
}

template <int G, int DH, bool kMerge, bool kShard>
static cudaError_t launch_decode_g(const DecodeArgs& a, const DecodeExtra& x, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  // q viewed as B*Hq rows of D; K, V as [B, Smax, Hkv, D]; 64-column boxes, 128-byte swizzle
  if (!make_tmap_bhsd(&tq, a.q, 1, a.B * a.Hq, 1, a.D, 64, G, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_bhsd(&tk, a.k, a.B, a.Smax, a.Hkv, a.D, 64, dec::BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_bhsd(&tv, a.v, a.B, a.Smax, a.Hkv, a.D, 64, dec::BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  DecGeom geo;
  geo.Cd = a.Smax / a.P;
  geo.nsub = (geo.Cd + dec::RPS - 1) / dec::RPS;
  const long long units = (long long)a.P * a.B * a.Hkv * geo.nsub;
  if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
  geo.units = (int)units;
  const size_t smem = sizeof(DecSmem<G>) + 1024;
  auto kern = decode_kernel<G, DH, kMerge, kShard>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = num_sms();
  kern<<<grid, dec::THREADS, smem, st>>>(tq, tk, tv, a, geo, x);
  return cudaGetLastError();
}

cudaError_t launch_decode_partial(const DecodeArgs& a, const DecodeExtra& x, cudaStream_t st) {
  const int G = a.Hq / a.Hkv;
  if (!decode_group_supported(G)) return cudaErrorNotSupported;
  const int mode = (x.out != nullptr ? 2 : 0) + (x.shard_lens != nullptr ? 1 : 0);
  auto pick_d = [&](auto g, auto d) -> cudaError_t {
    constexpr int GG = decltype(g)::value, DD = decltype(d)::value;
    switch (mode) {
      case 0: return launch_decode_g<GG, DD, false, false>(a, x, st);
      case 1: return launch_decode_g<GG, DD, false, true>(a, x, st);
      case 2: return launch_decode_g<GG, DD, true, false>(a, x, st);
      default: return launch_decode_g<GG, DD, true, true>(a, x, st);
    }
  };
  auto pick = [&](auto g) -> cudaError_t {
    if (a.D == 64) return pick_d(g, std::integral_constant<int, 64>{});
    return pick_d(g, std::integral_constant<int, 128>{});
  };
  switch (G) {
    case 1: return pick(std::integral_constant<int, 1>{});
    case 2: return pick(std::integral_constant<int, 2>{});
    case 4: return pick(std::integral_constant<int, 4>{});
    case 8: return pick(std::integral_constant<int, 8>{});
    default: return pick(std::integral_constant<int, 16>{});
  }
}

}  // namespace ra

// ---------------------------------------------------------------------------
// ring_attn_decode_partial_noalloc: the same decode, with its scratch (the
// sub-split results and the per-chunk arrival counters) in a fixed array of
// this library instead of a caller-provided workspace.
//
// It is for callers that cannot call cudaMalloc or hand this call a
// workspace: host programs whose own allocator owns all device memory (a
// fixed budget or a caching pool that must not be bypassed), and code on a
// latency-critical path where an allocation, which may synchronise the
// device, is not acceptable.  The array below is reserved on every GPU that
// loads this library and held until the process exits.
// ---------------------------------------------------------------------------
#include <mutex>

#include "../../include/ring_attn.h"

namespace ra {

static __device__ __align__(256) unsigned char g_decode_scratch[RING_DECODE_NOALLOC_SCRATCH_BYTES];

// Device address of g_decode_scratch on the current device.  Host code must
// not pass the symbol itself to a kernel: on the host it only names a
// stand-in.  Looked up once per device (with that device current) on the
// first call made on it.
static cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static void* cache[64] = {nullptr};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    cache[dev] = p;
  }
  *out = cache[dev];
  return cudaSuccess;
}

}  // namespace ra

extern "C" ring_status ring_attn_decode_partial_noalloc(const void* q, const void* k, const void* v,
                                                        const int32_t* seqlens, float* partials, float* part_lse,
                                                        int B, int Hq, int Hkv, int Smax, int D, int P, float scale,
                                                        int dtype, void* stream) {
  using namespace ra;
  auto a16 = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(q) || !a16(k) || !a16(v) || !seqlens || !a16(partials) || !a16(part_lse)) return RING_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || Smax < 1 || P < 1 || D < 1 || Hq % Hkv || Smax % P) return RING_EINVAL;
  if (!(scale > 0.f) || scale != scale || scale == __builtin_huge_valf()) return RING_EINVAL;
  if (dtype != RING_BF16 && dtype != RING_FP32) return RING_EINVAL;
  if ((long long)B * Smax * Hkv * D >= (1LL << 42)) return RING_EINVAL;
  if (dtype != RING_BF16 || (D != 64 && D != 128)) return RING_EUNSUPPORTED;
  const int G = Hq / Hkv;
  if (!decode_group_supported(G)) return RING_EUNSUPPORTED;
  const size_t need = decode_workspace_bytes(B, Hq, Hkv, Smax, D, P);
  if (need == 0 || need > (size_t)RING_DECODE_NOALLOC_SCRATCH_BYTES) return RING_EINVAL;
  void* ws = nullptr;
  if (noalloc_scratch(&ws) != cudaSuccess) return RING_ECUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a{};
  a.q = q; a.k = k; a.v = v; a.seqlens = seqlens;
  a.partials = partials; a.part_lse = part_lse;
  DecodeExtra x{};
  decode_workspace_split(ws, B, Hq, Hkv, Smax, D, P, &a.ws_part, &a.ws_count, &x.ws_done);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Smax = Smax; a.D = D; a.P = P; a.scale = scale;
  a.err = error_word();
  // the arrival counters must start at zero; the previous call may have been cut short
  if (cudaMemsetAsync(a.ws_count, 0, (size_t)B * Hkv * P * sizeof(unsigned int), st) != cudaSuccess)
    return RING_ECUDA;
  const cudaError_t e = launch_decode_partial(a, x, st);
  if (e == cudaSuccess) return RING_OK;
  return e == cudaErrorNotSupported ? RING_EUNSUPPORTED : RING_ECUDA;
}
