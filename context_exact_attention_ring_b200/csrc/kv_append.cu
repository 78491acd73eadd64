// Round-robin KV append ("NVIDIA unveils Helix Parallelism", the KV cache as
// it grows during decoding): tokens generated after the prompt are dealt to
// the KV-parallel ranks block by block -- the first `block` appended tokens of
// a sequence go to rank 0, the next `block` to rank 1, and so on, wrapping
// after rank P-1 -- so that every rank's shard grows evenly instead of one
// rank taking every new token.
//
// Rank p's shard is rows [p*C, (p+1)*C) of the cache (C = Smax/P) and holds
// shard_lens[b][p] valid rows; a token is written at the shard's fill count,
// which then advances.  One CTA per sequence; each warp copies whole token
// rows with 16-byte loads and stores.  A token whose shard is full is not
// written: the kernel records kFaultCapacity in the device error word, never
// writes outside the shard, and leaves that shard's count at C.
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace ra {

// Append indices i in [0, x) that the round-robin rule sends to rank p.
__device__ __forceinline__ long long rr_count(long long x, int p, int block, int P) {
  const long long cycle = (long long)block * P;
  const long long full = x / cycle, rem = x - full * cycle;
  const long long part = rem - (long long)p * block;
  return full * block + (part < 0 ? 0 : part > block ? block : part);
}

__global__ void __launch_bounds__(256) kv_append_kernel(AppendArgs a) {
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int C = a.Smax / a.P;
  const long long n0 = a.n_appended[b] > 0 ? a.n_appended[b] : 0;
  const size_t row_bytes = (size_t)a.Hkv * a.D * a.elem_bytes;
  const int nvec = (int)(row_bytes / 16);
  for (int j = warp; j < a.T; j += nwarps) {
    const long long n = n0 + j;
    const int p = (int)((n / a.block) % a.P);
    const int len0 = min(max(a.shard_lens[b * a.P + p], 0), C);
    const long long row = len0 + rr_count(n, p, a.block, a.P) - rr_count(n0, p, a.block, a.P);
    if (row >= C) {
      if (lane == 0) atomicCAS(a.err, 0u, kFaultCapacity);
      continue;
    }
    const size_t src = ((size_t)b * a.T + j) * row_bytes;
    const size_t dst = ((size_t)b * a.Smax + (size_t)p * C + (size_t)row) * row_bytes;
    const uint4* ks = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.k_new) + src);
    const uint4* vs = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.v_new) + src);
    uint4* kd = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.k_cache) + dst);
    uint4* vd = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.v_cache) + dst);
    for (int e = lane; e < nvec; e += 32) {
      kd[e] = __ldg(ks + e);
      vd[e] = __ldg(vs + e);
    }
  }
  __syncthreads();   // every copy has read the old counts
  for (int p = threadIdx.x; p < a.P; p += blockDim.x) {
    const int len0 = min(max(a.shard_lens[b * a.P + p], 0), C);
    const long long len1 = len0 + rr_count(n0 + a.T, p, a.block, a.P) - rr_count(n0, p, a.block, a.P);
    a.shard_lens[b * a.P + p] = (int)(len1 < C ? len1 : C);
  }
  if (threadIdx.x == 0) {
    const long long n1 = n0 + a.T;
    a.n_appended[b] = n1 < 0x7fffffffLL ? (int)n1 : 0x7fffffff;
  }
}

cudaError_t launch_kv_append(const AppendArgs& a, cudaStream_t st) {
  if (a.B < 1 || a.T < 1) return cudaSuccess;
  kv_append_kernel<<<a.B, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace ra
