// Split-KV single-token decode ("NVIDIA unveils Helix Parallelism", Phase 1:
// the KV cache sharded along the sequence; each shard yields a partial result
// that is merged afterwards).
//
// Work unit = (chunk p, batch b, kv head g, sub-split s): RPS consecutive rows
// of one chunk.  A persistent grid (one CTA per SM) walks the units in chunk
// order, so the always-full early chunks come first and the ragged tails of
// the sequences last.  Per CTA:
//   warp 0       TMA producer: 96-row K and V boxes into a 4-stage ring of
//                shared memory (bounded waits on the stage barriers);
//   warps 1..12  consumers: a half warp owns one K/V row per pass; a lane
//                holds 8 of the 128 dims of every query head of the kv head
//                (scaled by scale*log2 e), so each K/V element is widened to
//                fp32 once; partial dot products (packed f32x2 FMA) are
//                reduced by a transposing half-warp butterfly that leaves each
//                lane the score of one head; that head's lanes fold the row
//                into the running (m, l) -- the online-softmax update of
//                "Lesson 8: Context Parallelism", section 3 -- keeping a stale
//                max until a score exceeds it by 2^8 (exact: the same base
//                scales l and O), and broadcast the weight to the other lanes
//                for the PV update.
// At the end of a unit the 32 group states are folded (shuffles, then shared
// memory).  A chunk covered by one sub-split writes its partial directly;
// otherwise every sub-split writes to the workspace and the last CTA to
// arrive (atomic counter, reset by that CTA) folds them into the chunk's
// partial.  With an output buffer the merge runs in the same launch: the CTA
// that finishes the last of the P chunks of a (sequence, kv head) -- a second
// counter, reset the same way -- combines the P partials into out and lse.
// The valid rows of a chunk come from the sequence length (chunk p holds
// positions [p*C, (p+1)*C)) or, for a cache filled by the round-robin append
// of "NVIDIA unveils Helix Parallelism" (KV cache growth), from the chunk's
// own fill count.  The kernel is HBM-bound: each valid K/V byte is read once.
#include <cuda_bf16.h>
#include <type_traits>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kernels.h"
#include "ptx.cuh"

namespace ra {

namespace dec {
constexpr int D = 128;
constexpr int ROWS = 96;                    // rows per stage
constexpr int NST = 4;                      // stages
constexpr int RPS = 4032;                   // rows per sub-split (a multiple of ROWS)
constexpr int STAGE_BYTES = 2 * ROWS * D * 2;
constexpr int NCW = 12;                     // consumer warps
constexpr int UPI = 4;                      // rows per half warp handled together
constexpr int THREADS = 32 * (1 + NCW);
static_assert(ROWS % (2 * UPI * NCW) == 0, "a stage is covered by whole iterations of all consumer warps");
static_assert(RPS % ROWS == 0, "stages never straddle two sub-splits");
constexpr float LAZY = 8.f;                 // log2 of the largest tolerated growth before rescaling
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

__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float* f) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

// 8 bf16 -> 4 packed pairs of float (exact widening)
__device__ __forceinline__ void bf16x8_to_f32x2(const uint4 w, uint64_t* f2) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) f2[i] = pack2(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
}

// Each lane keeps its G heads in a lane-dependent order (slot i holds head
// head_of_slot(lane, i)) chosen so that the transposing half-warp sum below
// needs no selects: at each of the first log2(G) butterfly levels a lane keeps
// the first half of its remaining slots and sends the second half, which its
// partner holds, in the same head order, in its own second half.
template <int G>
__device__ __forceinline__ int head_of_slot(int lane, int i) {
  const int hi = (lane >> 3) & 1, odd = (lane >> 2) & 1;
  if constexpr (G == 4) {
    const int pair = (i >> 1) ? 1 - hi : hi;
    const int mem = (i & 1) ? 1 - odd : odd;
    return 2 * pair + mem;
  } else if constexpr (G == 2) {
    return i ? 1 - hi : hi;
  } else {
    return 0;
  }
}

// Sum over the 16 lanes of a half warp of the G per-head partial sums (slot
// order), leaving in every lane the full sum of head own_head(lane) = the head
// of its slot 0.  G = 4 takes 5 shuffles instead of 16.
template <int G>
__device__ __forceinline__ float half_warp_transpose_sum(const float (&v)[G]) {
  if constexpr (G == 4) {
    const float k0 = v[0] + __shfl_xor_sync(0xffffffffu, v[2], 8);
    const float k1 = v[1] + __shfl_xor_sync(0xffffffffu, v[3], 8);
    float x = k0 + __shfl_xor_sync(0xffffffffu, k1, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
  } else if constexpr (G == 2) {
    float x = v[0] + __shfl_xor_sync(0xffffffffu, v[1], 8);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x;
  } else {
    float x = v[0];
#pragma unroll
    for (int off = 8; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
  }
}

// Lane (xor distance) in the same half warp whose slot 0 holds the head of
// this lane's slot i: the reduced score of a head is replicated in every lane
// whose slot 0 is that head, so a butterfly shuffle reaches it.
template <int G>
__device__ __forceinline__ constexpr int slot_xor(int i) {
  return G == 4 ? (i << 2) : G == 2 ? (i << 3) : 0;
}

template <int G>
struct DecSmem {
  alignas(1024) uint8_t stage[dec::NST][dec::STAGE_BYTES];
  float wpart[dec::NCW][G][dec::D];
  float wm[dec::NCW][G];
  float wl[dec::NCW][G];
  alignas(8) uint64_t full[dec::NST];
  alignas(8) uint64_t empty[dec::NST];
  int is_last;      // set by one thread between two consumer barriers, read by all after the second
  int abort_flag;
};

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
template <int G>
__device__ __noinline__ void merge_bg(const DecodeArgs& a, const DecodeExtra& x, int b, int g, int lane) {
  constexpr int D = dec::D;
  __syncwarp();   // lane 0's acquire covers the warp from here on
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(x.out);
  const size_t bh0 = (size_t)b * a.Hq + g * G;
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

// Called by consumer warp 0 (all lanes) after the CTA's writes of a chunk's
// final partial and a consumer barrier: one lane counts the chunk; the warp
// that completes the count of (b, g) merges it.  The other consumer warps do
// not wait.
template <int G>
__device__ __forceinline__ void chunk_final_count(const DecodeArgs& a, const DecodeExtra& x, int b, int g, int lane) {
  int last = 0;
  if (lane == 0) last = count_chunk(a, x, b, g);
  if (__shfl_sync(0xffffffffu, last, 0)) {
    __syncwarp();   // lane 0's acquire covers the warp
    merge_bg<G>(a, x, b, g, lane);
  }
}

// kMerge: the launch also merges the partials (a.out != null); kShard: valid
// rows come from per-chunk fill counts (a.shard_lens != null).  Separate
// instantiations, so that the plain partial kernel carries none of their code.
template <int G, bool kMerge, bool kShard>
__global__ void __launch_bounds__(dec::THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, DecodeArgs a,
                  DecGeom geo, DecodeExtra x) {
  using namespace dec;
  extern __shared__ uint8_t smem_raw[];
  DecSmem<G>& sm = *reinterpret_cast<DecSmem<G>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), NCW);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t pol = l2_policy_evict_first();
      uint32_t cnt = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < geo.units && ok; u += gridDim.x) {
        int t = u;
        const int sub = t % geo.nsub; t /= geo.nsub;
        const int g = t % a.Hkv; t /= a.Hkv;
        const int b = t % a.B;
        const int p = t / a.B;
        const int r0 = p * geo.Cd + sub * RPS;
        const int r1 = min(r0 + RPS, chunk_end<kShard>(a, x, geo.Cd, b, p));
        for (int row = r0; row < r1; row += ROWS) {
          const int s = cnt % NST;
          const uint32_t ph = (cnt / NST) & 1u;
          if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1u, abort_flag, kWaitDecodeEmpty, a.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&sm.full[s]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          const uint32_t dst = smem_u32(sm.stage[s]);
          tma_load_4d(dst, &tmK, fb, 0, g, row, b, pol);
          tma_load_4d(dst + ROWS * D * 2, &tmV, fb, 0, g, row, b, pol);
          ++cnt;
        }
      }
      // do not leave while copies are still landing in shared memory
      for (uint32_t c = (cnt > (uint32_t)NST ? cnt - NST : 0); c < cnt; ++c) {
        const int s = c % NST;
        mbar_wait(smem_u32(&sm.full[s]), (c / NST) & 1u, nullptr, kWaitTeardown, a.err);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // Lane layout: each half warp (16 lanes) owns one K/V row per pass; lane
  // (dh, j) holds dims [dh*64 + 8j, dh*64 + 8j + 8) of every one of the G
  // query heads and of their output rows (the 16 lanes read the row's 256
  // contiguous bytes).  Per row: partial dot products, a transposing
  // half-warp reduction that leaves each lane the full score of one head,
  // the online-softmax update done by that head's lanes, and a broadcast of
  // the G weights p_h for the PV update.  Each K/V element is widened once.
  const int cw = warp - 1;                 // consumer warp 0..NCW-1
  const int ctid = threadIdx.x - 32;       // 0..32*NCW-1
  const int half = lane >> 4;
  const int dcol = ((lane >> 3) & 1) * 64 + (lane & 7) * 8;   // first dim of this lane
  const int oh = head_of_slot<G>(lane, 0);   // the head whose running (m, l) this lane keeps
  const float qscale = a.scale * 1.4426950408889634f;
  uint32_t cnt = 0;
  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(a.q);
  constexpr int CT = 32 * NCW;

  for (int u = blockIdx.x; u < geo.units; u += gridDim.x) {
    int t = u;
    const int sub = t % geo.nsub; t /= geo.nsub;
    const int g = t % a.Hkv; t /= a.Hkv;
    const int b = t % a.B;
    const int p = t / a.B;
    const int c0 = p * geo.Cd;
    const int nvalid_chunk = chunk_rows<kShard>(a, x, geo.Cd, b, p);
    const int n_live = (nvalid_chunk + RPS - 1) / RPS;
    const int r0 = c0 + sub * RPS;
    const int r1 = min(r0 + RPS, c0 + nvalid_chunk);

    if (nvalid_chunk == 0) {
      if (sub == 0) {
        for (int e = ctid; e < G * D; e += CT) {
          const int h = e / D, d = e - h * D;
          a.partials[((size_t)(b * a.Hq + g * G + h) * a.P + p) * D + d] = 0.f;
        }
        if (ctid < G) a.part_lse[(size_t)(b * a.Hq + g * G + ctid) * a.P + p] = -CUDART_INF_F;
        if constexpr (kMerge) {
          named_bar_sync(1, CT);   // the chunk's partial is written before it is counted
          if (cw == 0) chunk_final_count<G>(a, x, b, g, lane);
        }
      }
      continue;
    }
    if (r0 >= r1) continue;

    // this lane's 8 dims of the G query heads, scaled by scale * log2(e)
    uint64_t q2[G][4];   // slot order (see head_of_slot)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float f[8];
      const int head = head_of_slot<G>(lane, h);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(qb + ((size_t)b * a.Hq + g * G + head) * D + dcol), f);
#pragma unroll
      for (int i = 0; i < 4; ++i) q2[h][i] = pack2(f[2 * i] * qscale, f[2 * i + 1] * qscale);
    }
    // running state: m, l of head oh (this lane's owned head); O rows of all heads
    float m = -CUDART_INF_F, l = 0.f;
    uint64_t o2[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 4; ++i) o2[h][i] = 0ull;

    bool ok = true;
    for (int row = r0; row < r1 && ok; row += ROWS) {
      const int s = cnt % NST;
      const uint32_t ph = (cnt / NST) & 1u;
      if (!mbar_wait(smem_u32(&sm.full[s]), ph, abort_flag, kWaitDecodeFull, a.err)) { ok = false; break; }
      const uint8_t* Ks = sm.stage[s];
      const uint8_t* Vs = Ks + ROWS * D * 2;
      // UPI passes per iteration: their reductions and broadcasts interleave
#pragma unroll
      for (int pass = 0; pass < ROWS / (2 * NCW); pass += UPI) {
        int rr[UPI];
        bool valid[UPI];
        uint64_t x2[UPI][4];
        float part[UPI][G];
#pragma unroll
        for (int u = 0; u < UPI; ++u) {
          rr[u] = (pass + u) * 2 * NCW + cw * 2 + half;
          valid[u] = row + rr[u] < r1;
          bf16x8_to_f32x2(*reinterpret_cast<const uint4*>(Ks + rr[u] * 256 + dcol * 2), x2[u]);
        }
#pragma unroll
        for (int u = 0; u < UPI; ++u)
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const uint64_t acc = ffma2(q2[h][1], x2[u][1], ffma2(q2[h][0], x2[u][0], 0ull));
            part[u][h] = hsum2(ffma2(q2[h][3], x2[u][3], ffma2(q2[h][2], x2[u][2], acc)));
          }
#pragma unroll
        for (int u = 0; u < UPI; ++u)
          bf16x8_to_f32x2(*reinterpret_cast<const uint4*>(Vs + rr[u] * 256 + dcol * 2), x2[u]);
        float sc[UPI];
#pragma unroll
        for (int u = 0; u < UPI; ++u) {
          sc[u] = half_warp_transpose_sum<G>(part[u]);
          if (!valid[u]) sc[u] = -CUDART_INF_F;
        }
        // online update with the UPI rows (the base moves at most once per iteration)
        float smax = sc[0];
#pragma unroll
        for (int u = 1; u < UPI; ++u) smax = fmaxf(smax, sc[u]);
        const bool moved = smax > m + LAZY;
        if (__any_sync(0xffffffffu, moved)) {
          float f = 1.f;
          if (moved) {
            f = (m == -CUDART_INF_F) ? 0.f : ex2(m - smax);
            m = smax;
            l *= f;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float fh = __shfl_xor_sync(0xffffffffu, f, slot_xor<G>(h));
            const uint64_t f2 = pack2(fh, fh);
#pragma unroll
            for (int i = 0; i < 4; ++i) o2[h][i] = fmul2(o2[h][i], f2);
          }
        }
        const bool live = m != -CUDART_INF_F;
        float pw[UPI];
#pragma unroll
        for (int u = 0; u < UPI; ++u) {
          pw[u] = (valid[u] && live) ? ex2(sc[u] - m) : 0.f;
          l += pw[u];
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
          for (int u = 0; u < UPI; ++u) {
            const float pu = __shfl_xor_sync(0xffffffffu, pw[u], slot_xor<G>(h));
            const uint64_t p2 = pack2(pu, pu);
#pragma unroll
            for (int i = 0; i < 4; ++i) o2[h][i] = ffma2(p2, x2[u][i], o2[h][i]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));   // this warp is done with the stage
      ++cnt;
    }
    // (after an expired wait the unit still runs through every named barrier
    // below, so that all consumer warps leave the loop together)

    // fold the two half warps (same heads and dims, different rows)
    {
      const float mc = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      const float f = (m == -CUDART_INF_F) ? 0.f : ex2(m - mc);
      l *= f;
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      m = mc;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float fh = __shfl_xor_sync(0xffffffffu, f, slot_xor<G>(h));
        const uint64_t f2 = pack2(fh, fh);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float x, y;
          unpack2(fmul2(o2[h][i], f2), x, y);
          x += __shfl_xor_sync(0xffffffffu, x, 16);
          y += __shfl_xor_sync(0xffffffffu, y, 16);
          o2[h][i] = pack2(x, y);
        }
      }
    }
    if (half == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int head = head_of_slot<G>(lane, h);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          unpack2(o2[h][i], sm.wpart[cw][head][dcol + 2 * i], sm.wpart[cw][head][dcol + 2 * i + 1]);
      }
      if ((lane & 3) == 0) {
        sm.wm[cw][oh] = m;
        sm.wl[cw][oh] = l;
      }
    }
    named_bar_sync(1, CT);

    // fold the consumer warps: thread -> (head, dim) pairs; natural-log lse at the end
    float* ws_unit = a.ws_part + ((((size_t)(b * a.Hkv + g) * a.P + p) * geo.nsub + sub) * G) * (D + 1);
    for (int e = ctid; e < G * D; e += CT) {
      const int h = e / D, d = e - h * D;
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < NCW; ++w) mx = fmaxf(mx, sm.wm[w][h]);
      float Lsum = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float f = (sm.wm[w][h] == -CUDART_INF_F) ? 0.f : ex2(sm.wm[w][h] - mx);
        Lsum = fmaf(sm.wl[w][h], f, Lsum);
        acc = fmaf(sm.wpart[w][h][d], f, acc);
      }
      const float od = acc / Lsum;
      const float lse = (mx + log2f(Lsum)) * 0.6931471805599453f;
      if (n_live == 1) {
        a.partials[((size_t)(b * a.Hq + g * G + h) * a.P + p) * D + d] = od;
        if (d == 0) a.part_lse[(size_t)(b * a.Hq + g * G + h) * a.P + p] = lse;
      } else {
        ws_unit[h * (D + 1) + d] = od;
        if (d == 0) ws_unit[h * (D + 1) + D] = lse;
      }
    }
    if (n_live > 1) {
      named_bar_sync(1, CT);
      if (ctid == 0) {
        unsigned int* ctr = a.ws_count + (size_t)(b * a.Hkv + g) * a.P + p;
        const unsigned int old = atom_add_acq_rel_gpu(ctr, 1u);
        const int last = (old == (unsigned int)(n_live - 1));
        if (last) atomicExch(ctr, 0u);       // leave the counter at zero for the next call
        sm.is_last = last;
      }
      named_bar_sync(1, CT);
      if (sm.is_last) {
        const float* ws_chunk = a.ws_part + (((size_t)(b * a.Hkv + g) * a.P + p) * geo.nsub) * G * (D + 1);
        for (int e = ctid; e < G * D; e += CT) {
          const int h = e / D, d = e - h * D;
          float mx = -CUDART_INF_F;
          for (int s2 = 0; s2 < n_live; ++s2) mx = fmaxf(mx, __ldcg(ws_chunk + (s2 * G + h) * (D + 1) + D));
          float Lsum = 0.f, acc = 0.f;
          for (int s2 = 0; s2 < n_live; ++s2) {
            const float* r = ws_chunk + (s2 * G + h) * (D + 1);
            const float w = expf(__ldcg(r + D) - mx);
            Lsum += w;
            acc = fmaf(w, __ldcg(r + d), acc);
          }
          a.partials[((size_t)(b * a.Hq + g * G + h) * a.P + p) * D + d] = acc / Lsum;
          if (d == 0) a.part_lse[(size_t)(b * a.Hq + g * G + h) * a.P + p] = mx + logf(Lsum);
        }
      }
    }
    // this CTA wrote the chunk's final partial: directly, or as the last sub-split to arrive
    const bool chunk_final = n_live == 1 || sm.is_last;
    // shared fold buffers are free again; leave together if any wait expired
    if (named_bar_any(1, CT, !ok || *abort_flag)) break;
    if constexpr (kMerge)
      if (chunk_final && cw == 0) chunk_final_count<G>(a, x, b, g, lane);
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

template <int G, bool kMerge, bool kShard>
static cudaError_t launch_decode_g(const DecodeArgs& a, const DecodeExtra& x, cudaStream_t st) {
  CUtensorMap tk, tv;
  if (!make_tmap_bhsd(&tk, a.k, a.B, a.Smax, a.Hkv, a.D, dec::D, dec::ROWS, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_bhsd(&tv, a.v, a.B, a.Smax, a.Hkv, a.D, dec::D, dec::ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  DecGeom geo;
  geo.Cd = a.Smax / a.P;
  geo.nsub = (geo.Cd + dec::RPS - 1) / dec::RPS;
  const long long units = (long long)a.P * a.B * a.Hkv * geo.nsub;
  if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
  geo.units = (int)units;
  const size_t smem = sizeof(DecSmem<G>) + 1024;
  auto kern = decode_kernel<G, kMerge, kShard>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = num_sms();
  kern<<<grid, dec::THREADS, smem, st>>>(tk, tv, a, geo, x);
  return cudaGetLastError();
}

cudaError_t launch_decode_partial(const DecodeArgs& a, const DecodeExtra& x, cudaStream_t st) {
  const int G = a.Hq / a.Hkv;
  if (G != 1 && G != 2 && G != 4) return cudaErrorNotSupported;
  const int mode = (x.out != nullptr ? 2 : 0) + (x.shard_lens != nullptr ? 1 : 0);
  auto pick = [&](auto g) -> cudaError_t {
    constexpr int GG = decltype(g)::value;
    switch (mode) {
      case 0: return launch_decode_g<GG, false, false>(a, x, st);
      case 1: return launch_decode_g<GG, false, true>(a, x, st);
      case 2: return launch_decode_g<GG, true, false>(a, x, st);
      default: return launch_decode_g<GG, true, true>(a, x, st);
    }
  };
  if (G == 1) return pick(std::integral_constant<int, 1>{});
  if (G == 2) return pick(std::integral_constant<int, 2>{});
  return pick(std::integral_constant<int, 4>{});
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
  if (dtype != RING_BF16 || D != 128) return RING_EUNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4) return RING_EUNSUPPORTED;
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
