// Host-side launchers of the library's kernels (internal; the public ABI is
// include/ring_attn.h).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "ring_sched.h"

namespace ra {

// CUDA-core ring attention (ring or step mode, fp32 or bf16 inputs).
cudaError_t launch_attn_simt(const Plan& p, bool bf16, const void* q, const void* k, const void* v, void* out,
                             float* lse, float* m, float* l, float* O, float scale, cudaStream_t st);

// Tensor-core (tcgen05) ring attention, bf16 in / fp32 accumulate.
struct TcArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;            // ring mode: [B,Sq,Hq,D] bf16
  float* lse;           // ring mode: [B,Hq,Sq]
  float* m;             // step mode state
  float* l;
  float* O;
  unsigned long long* counters;  // optional [2 + P]
  float scale;
  unsigned int* err;             // device error word
};
cudaError_t launch_attn_tc(const Plan& p, const TcArgs& a, cudaStream_t st);
// The same on CTA pairs (tcgen05 cta_group::2, M = 256), D = 128 only.
cudaError_t launch_attn_tc_pair(const Plan& p, const TcArgs& a, cudaStream_t st);

// Backward (CUDA cores).  Ring mode writes dq, dk, dv (input dtype); step
// mode adds into the float32 sums dq_acc, dk_acc, dv_acc instead.
struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;     // [B,Sq,Hq,D]
  const float* lse;     // [B,Hq,Sq] of the forward
  const float* delta;   // [B,Hq,Sq] = rowsum(dout * out)
  void* dq;             // [B,Sq,Hq,D]
  void* dk;             // [B,Skv,Hkv,D]
  void* dv;
  float* dq_acc;        // step mode
  float* dk_acc;
  float* dv_acc;
  float scale;
};
cudaError_t launch_bwd_delta(const void* out, const void* dout, float* delta, int B, int Hq, int S, int D, bool bf16,
                             cudaStream_t st);
cudaError_t launch_bwd_simt(const Plan& p, const BwdArgs& a, bool bf16, cudaStream_t st);
// Backward on the tensor cores (bf16): a K/V-major launch (dK, dV) then a
// Q-major launch (dQ).
cudaError_t launch_bwd_tc(const Plan& p, const BwdArgs& a, unsigned int* err, cudaStream_t st);

cudaError_t launch_state_init(float* m, float* l, float* O, int B, int Hq, int S_loc, int D, cudaStream_t st);
cudaError_t launch_state_finalize(const float* m, const float* l, const float* O, void* out, float* lse, int B,
                                  int Hq, int S, int D, bool bf16, cudaStream_t st);
cudaError_t launch_merge(const float* part, const float* plse, void* out, float* out_lse, int B, int Hq, int P,
                         int D, bool bf16, cudaStream_t st);

// Split-KV decode.
struct DecodeArgs {
  const void* q;        // [B,Hq,D] bf16
  const void* k;        // [B,Smax,Hkv,D] bf16; chunk p = rows [p*Smax/P, (p+1)*Smax/P)
  const void* v;
  const int32_t* seqlens;  // [B]: rows < seqlens[b] are valid (unless DecodeExtra::shard_lens)
  float* partials;      // [B,Hq,P,D]
  float* part_lse;      // [B,Hq,P]
  float* ws_part;       // sub-split results
  unsigned int* ws_count;  // per-chunk arrival counters (zero between calls)
  int B, Hq, Hkv, Smax, D, P;
  float scale;
  unsigned int* err;    // device error word
};
// Arguments of the fused / shard-length decode, kept out of DecodeArgs (a
// separate kernel parameter leaves the register allocation of the plain
// partial kernel as it was).
struct DecodeExtra {
  const int32_t* shard_lens;  // [B,P] or null: the first shard_lens[b,p] rows of chunk p are valid
  void* out;                  // null, or [B,Hq,D] bf16: merge the P partials in the same launch
  float* out_lse;             // [B,Hq] or null (with out)
  unsigned int* ws_done;      // per-(b, kv head) finished-chunk counters (zero between calls)
};
// Query heads per kv head the decode kernel is built for (the heads are the N of
// its tensor-core products, padded to 16).
inline bool decode_group_supported(int G) { return G == 1 || G == 2 || G == 4 || G == 8 || G == 16; }
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Smax, int D, int P);
void decode_workspace_split(void* ws, int B, int Hq, int Hkv, int Smax, int D, int P, float** part,
                            unsigned int** count, unsigned int** done);
cudaError_t launch_decode_partial(const DecodeArgs& a, const DecodeExtra& x, cudaStream_t st);

// Round-robin KV append (one CTA per sequence).
struct AppendArgs {
  void* k_cache;        // [B,Smax,Hkv,D]
  void* v_cache;
  const void* k_new;    // [B,T,Hkv,D]
  const void* v_new;
  int32_t* shard_lens;  // [B,P], read and advanced
  int32_t* n_appended;  // [B], read and advanced
  int B, T, Hkv, Smax, D, P, block, elem_bytes;
  unsigned int* err;    // device error word (capacity overflow)
};
cudaError_t launch_kv_append(const AppendArgs& a, cudaStream_t st);

// Driver entry point for building TMA descriptors (resolved at run time, so
// the library does not link libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

// 4-D bf16 tensor map over a [B, rows, heads, D] tensor with box
// {box_d, 1, box_rows, 1}.
bool make_tmap_bhsd(CUtensorMap* m, const void* base, int B, int rows, int heads, int D, int box_d, int box_rows,
                    CUtensorMapSwizzle swz);

// 5-D bf16 tensor map over a [B, S, heads, D] tensor viewed as
// [B, S/P, P, heads, D] (token x*P + c at coordinates (c, x)) with box
// {box_d, 1, 1, box_rows, 1}: one box holds box_rows tokens of stripe c.
bool make_tmap_striped(CUtensorMap* m, const void* base, int B, int S, int P, int heads, int D, int box_d,
                       int box_rows, CUtensorMapSwizzle swz);

int num_sms();

// Device address of the library's error word on the current device.
unsigned int* error_word();

}  // namespace ra
