// C ABI of the library (declared in include/ring_attn.h): argument checks,
// TMA descriptor construction and kernel dispatch.  No memory is allocated
// here; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/ring_attn.h"
#include "kernels.h"
#include "ptx.cuh"
#include "ring_sched.h"

namespace ra {

__device__ unsigned int g_error_word = 0;

unsigned int* error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  static unsigned int* cache[64] = {nullptr};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess) cache[dev] = static_cast<unsigned int*>(p);
  }
  return cache[dev];
}

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_tmap_bhsd(CUtensorMap* m, const void* base, int B, int rows, int heads, int D, int box_d, int box_rows,
                    CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2, (cuuint64_t)rows * heads * D * 2};
  const cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_striped(CUtensorMap* m, const void* base, int B, int S, int P, int heads, int D, int box_d,
                       int box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc || P < 1 || S % P) return false;
  const cuuint64_t row = (cuuint64_t)heads * D * 2;   // bytes per token
  const cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)P, (cuuint64_t)(S / P), (cuuint64_t)B};
  const cuuint64_t strides[4] = {(cuuint64_t)D * 2, row, row * P, row * S};
  const cuuint32_t box[5] = {(cuuint32_t)box_d, 1, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  static int cache[64] = {0};
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  int n = 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

// One thread waits on an mbarrier that nothing will ever complete, with a
// short limit: exercises the bounded-wait error path without any fault.
__global__ void selftest_wait_kernel(unsigned int* err, unsigned long long limit_ns) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    mbar_wait_for(smem_u32(&bar), 0, &abort_flag, kWaitSelftest, err, limit_ns);
  }
}

}  // namespace ra

using namespace ra;

namespace {

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ring_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return RING_OK;
  if (e == cudaErrorNotSupported) return RING_EUNSUPPORTED;
  if (e == cudaErrorInvalidValue) return RING_EINVAL;
  return RING_ECUDA;
}

bool good_scale(float s) { return std::isfinite(s) && s > 0.f; }

// Split code of the `layout` argument: low byte the split, next byte the
// chunks per rank (0 = the split's default).  Returns false if out of range.
bool decode_layout(int layout, int* kind, int* cpr) {
  if (layout < 0 || (layout >> 16)) return false;
  const int kd = layout & 0xff, k = (layout >> 8) & 0xff;
  if (kd == RING_CONTIGUOUS) {
    *cpr = k ? k : 1;
    if (*cpr > RING_MAX_CHUNKS_PER_RANK) return false;
  } else if (kd == RING_ZIGZAG) {
    *cpr = k ? k : 2;
    if (*cpr < 2 || *cpr > RING_MAX_CHUNKS_PER_RANK) return false;
  } else if (kd == RING_STRIPED) {
    if (k > 1) return false;
    *cpr = 1;
  } else {
    return false;
  }
  *kind = kd == RING_ZIGZAG ? kLayoutZigzag : kd == RING_STRIPED ? kLayoutStriped : kLayoutContiguous;
  return true;
}

// Ring-mode plan of a split (no pointers, no shapes beyond the sequence).
bool ring_split(int S, int P, int layout, Plan* pl) {
  int kind = 0, cpr = 1;
  if (S < 1 || P < 1 || !decode_layout(layout, &kind, &cpr)) return false;
  const long long nchunks = (long long)P * cpr;
  if (nchunks > (1LL << 30) || S % nchunks) return false;
  pl->mode = kModeRing;
  pl->layout = kind;
  pl->P = P;
  pl->cpr = cpr;
  pl->striped = kind == kLayoutStriped;
  pl->strided = pl->striped;
  pl->nqc = pl->nkc = (int)nchunks;
  pl->C = (int)(S / nchunks);
  pl->Sq = pl->Skv = S;
  return true;
}

// Shared checks of the prefill entry points; fills the ring-mode plan.
ring_status ring_plan(const void* q, const void* k, const void* v, const void* out, const void* lse, int B, int Hq,
                      int Hkv, int S, int D, int P, int causal, int layout, float scale, int dtype, Plan* p) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse)) return RING_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || P < 1 || D < 1) return RING_EINVAL;
  if (Hq % Hkv) return RING_EINVAL;
  if (dtype != RING_BF16 && dtype != RING_FP32) return RING_EINVAL;
  if (!good_scale(scale)) return RING_EINVAL;
  Plan pl{};
  if (!ring_split(S, P, layout, &pl)) return RING_EINVAL;
  if ((long long)B * S * Hq * D >= (1LL << 40)) return RING_EINVAL;
  if (D != 64 && D != 128) return RING_EUNSUPPORTED;
  pl.B = B; pl.Hq = Hq; pl.Hkv = Hkv; pl.D = D;
  pl.causal = causal ? 1 : 0;
  *p = pl;
  return RING_OK;
}

// Shared checks of the decode entry points; fills the kernel arguments.
ring_status decode_args(const void* q, const void* k, const void* v, const int32_t* seqlens,
                        const int32_t* shard_lens, float* partials, float* part_lse, int B, int Hq, int Hkv,
                        int Smax, int D, int P, float scale, int dtype, void* workspace, size_t workspace_bytes,
                        DecodeArgs* out, DecodeExtra* extra) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !(seqlens || shard_lens) || !aligned16(partials) ||
      !aligned16(part_lse))
    return RING_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || Smax < 1 || P < 1 || D < 1 || Hq % Hkv || Smax % P) return RING_EINVAL;
  if (!good_scale(scale)) return RING_EINVAL;
  if (dtype != RING_BF16 && dtype != RING_FP32) return RING_EINVAL;
  if ((long long)B * Smax * Hkv * D >= (1LL << 42)) return RING_EINVAL;
  if (dtype != RING_BF16 || (D != 64 && D != 128)) return RING_EUNSUPPORTED;
  const int G = Hq / Hkv;
  if (!decode_group_supported(G)) return RING_EUNSUPPORTED;
  const size_t need = decode_workspace_bytes(B, Hq, Hkv, Smax, D, P);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need) return RING_EINVAL;
  DecodeArgs a{};
  DecodeExtra x{};
  a.q = q; a.k = k; a.v = v; a.seqlens = seqlens;
  x.shard_lens = shard_lens;
  a.partials = partials; a.part_lse = part_lse;
  decode_workspace_split(workspace, B, Hq, Hkv, Smax, D, P, &a.ws_part, &a.ws_count, &x.ws_done);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Smax = Smax; a.D = D; a.P = P; a.scale = scale;
  a.err = error_word();
  *out = a;
  *extra = x;
  return RING_OK;
}

// Shared checks of the step entry points; fills the step-mode plan.
ring_status step_plan(const void* q_shard, const void* kchunk, const void* vchunk, const ring_chunk_ids* ids, int B,
                      int Hq, int Hkv, int D, float scale, int dtype, Plan* out) {
  if (!ids) return RING_EINVAL;
  if (!aligned16(q_shard) || !aligned16(kchunk) || !aligned16(vchunk)) return RING_EINVAL;
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || Hq % Hkv) return RING_EINVAL;
  if (ids->n_q < 1 || ids->n_q > RING_MAX_CHUNKS_PER_RANK || ids->n_kv < 1 ||
      ids->n_kv > RING_MAX_CHUNKS_PER_RANK || ids->chunk_len < 1 || ids->stripes < 0)
    return RING_EINVAL;
  for (int i = 0; i < ids->n_q; ++i)
    if (ids->q[i] < 0) return RING_EINVAL;
  for (int i = 0; i < ids->n_kv; ++i)
    if (ids->kv[i] < 0) return RING_EINVAL;
  if (dtype != RING_BF16 && dtype != RING_FP32) return RING_EINVAL;
  if (!good_scale(scale)) return RING_EINVAL;
  if (ids->stripes > 0) {
    // striped split: one stripe of queries against one stripe of keys
    if (ids->n_q != 1 || ids->n_kv != 1 || ids->q[0] >= ids->stripes || ids->kv[0] >= ids->stripes)
      return RING_EINVAL;
  } else {
    const long long maxgid = 2147483647LL / ids->chunk_len;
    for (int i = 0; i < ids->n_q; ++i)
      if (ids->q[i] + 1LL > maxgid) return RING_EINVAL;
    for (int i = 0; i < ids->n_kv; ++i)
      if (ids->kv[i] + 1LL > maxgid) return RING_EINVAL;
  }
  if ((long long)ids->n_q * ids->chunk_len > 2147483647LL || (long long)ids->n_kv * ids->chunk_len > 2147483647LL)
    return RING_EINVAL;
  if (D != 64 && D != 128) return RING_EUNSUPPORTED;
  Plan p{};
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.D = D;
  p.causal = ids->causal ? 1 : 0;
  p.mode = kModeStep;
  p.layout = ids->stripes > 0 ? kLayoutStriped : kLayoutContiguous;
  p.P = ids->stripes > 0 ? ids->stripes : 1;
  p.cpr = 1;
  p.striped = ids->stripes > 0;
  p.strided = 0;   // the buffers are the shards themselves
  p.C = ids->chunk_len;
  p.nqc = ids->n_q;
  p.nkc = ids->n_kv;
  for (int i = 0; i < p.nqc; ++i) p.qid[i] = ids->q[i];
  for (int i = 0; i < p.nkc; ++i) p.kid[i] = ids->kv[i];
  // Q slots by decreasing chunk id (the longest rows first)
  for (int i = 0; i < p.nqc; ++i) p.qorder[i] = i;
  for (int i = 1; i < p.nqc; ++i)
    for (int j = i; j > 0 && p.qid[p.qorder[j]] > p.qid[p.qorder[j - 1]]; --j) {
      const int t = p.qorder[j];
      p.qorder[j] = p.qorder[j - 1];
      p.qorder[j - 1] = t;
    }
  p.Sq = p.nqc * p.C;
  p.Skv = p.nkc * p.C;
  *out = p;
  return RING_OK;
}

}  // namespace

extern "C" {

ring_status ring_attn_fwd_counted(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                                  int Hkv, int S, int D, int P, int causal, int layout, float scale, int dtype,
                                  unsigned long long* counters, void* stream) {
  Plan p;
  ring_status rs = ring_plan(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, &p);
  if (rs != RING_OK) return rs;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == RING_FP32)
    return from_cuda(launch_attn_simt(p, false, q, k, v, out, lse, nullptr, nullptr, nullptr, scale, st));
  TcArgs a{q, k, v, out, lse, nullptr, nullptr, nullptr, counters, scale, error_word()};
  return from_cuda(launch_attn_tc(p, a, st));
}

ring_status ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                          int S, int D, int P, int causal, int layout, float scale, int dtype, void* stream) {
  return ring_attn_fwd_counted(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, nullptr,
                               stream);
}

ring_status ring_attn_fwd_simt(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                               int Hkv, int S, int D, int P, int causal, int layout, float scale, int dtype,
                               void* stream) {
  Plan p;
  ring_status rs = ring_plan(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, &p);
  if (rs != RING_OK) return rs;
  return from_cuda(launch_attn_simt(p, dtype == RING_BF16, q, k, v, out, lse, nullptr, nullptr, nullptr, scale,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

size_t ring_attn_bwd_workspace_bytes(int B, int Hq, int S) {
  if (B < 1 || Hq < 1 || S < 1) return 0;
  return ((size_t)B * Hq * S * sizeof(float) + 255) & ~size_t(255);
}

ring_status ring_attn_bwd_delta(const void* out, const void* dout, float* delta, int B, int Hq, int S, int D,
                                int dtype, void* stream) {
  if (!aligned16(out) || !aligned16(dout) || !aligned16(delta)) return RING_EINVAL;
  if (B < 1 || Hq < 1 || S < 1 || D < 1) return RING_EINVAL;
  if (dtype != RING_BF16 && dtype != RING_FP32) return RING_EINVAL;
  return from_cuda(launch_bwd_delta(out, dout, delta, B, Hq, S, D, dtype == RING_BF16,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

static ring_status bwd_impl(const void* q, const void* k, const void* v, const void* out, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S, int D,
                            int P, int causal, int layout, float scale, int dtype, void* workspace,
                            size_t workspace_bytes, void* stream, bool simt) {
  Plan p;
  ring_status rs = ring_plan(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, &p);
  if (rs != RING_OK) return rs;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return RING_EINVAL;
  const size_t need = ring_attn_bwd_workspace_bytes(B, Hq, S);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need) return RING_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* delta = static_cast<float*>(workspace);
  cudaError_t e = launch_bwd_delta(out, dout, delta, B, Hq, S, D, dtype == RING_BF16, st);
  if (e != cudaSuccess) return from_cuda(e);
  BwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.lse = lse; a.delta = delta;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.scale = scale;
  if (dtype == RING_BF16 && !simt) return from_cuda(launch_bwd_tc(p, a, error_word(), st));
  return from_cuda(launch_bwd_simt(p, a, dtype == RING_BF16, st));
}

ring_status ring_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S, int D, int P,
                          int causal, int layout, float scale, int dtype, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, workspace,
                  workspace_bytes, stream, false);
}

ring_status ring_attn_bwd_simt(const void* q, const void* k, const void* v, const void* out, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S, int D,
                               int P, int causal, int layout, float scale, int dtype, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, workspace,
                  workspace_bytes, stream, true);
}

ring_status ring_attn_step_bwd(const void* q_shard, const void* kchunk, const void* vchunk, const void* dout_shard,
                               const float* lse, const float* delta, float* dq_acc, float* dk_acc, float* dv_acc,
                               const ring_chunk_ids* ids, int B, int Hq, int Hkv, int D, float scale, int dtype,
                               void* stream) {
  Plan p;
  ring_status rs = step_plan(q_shard, kchunk, vchunk, ids, B, Hq, Hkv, D, scale, dtype, &p);
  if (rs != RING_OK) return rs;
  if (!aligned16(dout_shard) || !aligned16(lse) || !aligned16(delta) || !aligned16(dq_acc) || !aligned16(dk_acc) ||
      !aligned16(dv_acc))
    return RING_EINVAL;
  BwdArgs a{};
  a.q = q_shard; a.k = kchunk; a.v = vchunk; a.dout = dout_shard; a.lse = lse; a.delta = delta;
  a.dq_acc = dq_acc; a.dk_acc = dk_acc; a.dv_acc = dv_acc;
  a.scale = scale;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == RING_BF16) return from_cuda(launch_bwd_tc(p, a, error_word(), st));
  return from_cuda(launch_bwd_simt(p, a, false, st));
}

ring_status ring_attn_state_init(float* m, float* l, float* O, int B, int Hq, int S_loc, int D, void* stream) {
  if (!aligned16(m) || !aligned16(l) || !aligned16(O)) return RING_EINVAL;
  if (B < 1 || Hq < 1 || S_loc < 1 || D < 1 || D % 4) return RING_EINVAL;
  return from_cuda(launch_state_init(m, l, O, B, Hq, S_loc, D, reinterpret_cast<cudaStream_t>(stream)));
}

ring_status ring_attn_step(const void* q_shard, const void* kchunk, const void* vchunk, float* m, float* l, float* O,
                           const ring_chunk_ids* ids, int B, int Hq, int Hkv, int D, float scale, int dtype,
                           void* stream) {
  Plan p;
  ring_status rs = step_plan(q_shard, kchunk, vchunk, ids, B, Hq, Hkv, D, scale, dtype, &p);
  if (rs != RING_OK) return rs;
  if (!aligned16(m) || !aligned16(l) || !aligned16(O)) return RING_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == RING_FP32)
    return from_cuda(launch_attn_simt(p, false, q_shard, kchunk, vchunk, nullptr, nullptr, m, l, O, scale, st));
  TcArgs a{q_shard, kchunk, vchunk, nullptr, nullptr, m, l, O, nullptr, scale, error_word()};
  return from_cuda(launch_attn_tc(p, a, st));
}

ring_status ring_attn_state_finalize(const float* m, const float* l, const float* O, void* out, float* lse, int B,
                                     int Hq, int S_loc, int D, int dtype, void* stream) {
  if (!aligned16(m) || !aligned16(l) || !aligned16(O) || !aligned16(out) || !aligned16(lse)) return RING_EINVAL;
  if (B < 1 || Hq < 1 || S_loc < 1 || D < 1) return RING_EINVAL;
  if (dtype != RING_BF16 && dtype != RING_FP32) return RING_EINVAL;
  return from_cuda(launch_state_finalize(m, l, O, out, lse, B, Hq, S_loc, D, dtype == RING_BF16,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

size_t ring_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Smax, int D, int P) {
  if (P < 1 || Smax % P) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, Smax, D, P);
}

ring_status ring_attn_decode_partial(const void* q, const void* k, const void* v, const int32_t* seqlens,
                                     float* partials, float* part_lse, int B, int Hq, int Hkv, int Smax, int D, int P,
                                     float scale, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  DecodeArgs a{};
  DecodeExtra x{};
  ring_status rs = decode_args(q, k, v, seqlens, nullptr, partials, part_lse, B, Hq, Hkv, Smax, D, P, scale, dtype,
                               workspace, workspace_bytes, &a, &x);
  if (rs != RING_OK) return rs;
  return from_cuda(launch_decode_partial(a, x, reinterpret_cast<cudaStream_t>(stream)));
}

ring_status ring_attn_decode_fused(const void* q, const void* k, const void* v, const int32_t* seqlens,
                                   const int32_t* shard_lens, float* partials, float* part_lse, void* out,
                                   float* out_lse, int B, int Hq, int Hkv, int Smax, int D, int P, float scale,
                                   int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if ((seqlens == nullptr) == (shard_lens == nullptr)) return RING_EINVAL;   // exactly one source of lengths
  if (!aligned16(out)) return RING_EINVAL;
  if (out_lse && (reinterpret_cast<uintptr_t>(out_lse) & 3u)) return RING_EINVAL;
  DecodeArgs a{};
  DecodeExtra x{};
  ring_status rs = decode_args(q, k, v, seqlens, shard_lens, partials, part_lse, B, Hq, Hkv, Smax, D, P, scale,
                               dtype, workspace, workspace_bytes, &a, &x);
  if (rs != RING_OK) return rs;
  x.out = out;
  x.out_lse = out_lse;
  return from_cuda(launch_decode_partial(a, x, reinterpret_cast<cudaStream_t>(stream)));
}

ring_status ring_attn_kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                                int32_t* shard_lens, int32_t* n_appended, int B, int T, int Hkv, int Smax, int D,
                                int P, int block, int dtype, void* stream) {
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new) || !shard_lens ||
      !n_appended)
    return RING_EINVAL;
  if (B < 1 || T < 1 || Hkv < 1 || Smax < 1 || D < 1 || P < 1 || block < 1 || Smax % P) return RING_EINVAL;
  if (dtype != RING_BF16 && dtype != RING_FP32) return RING_EINVAL;
  const int eb = dtype == RING_BF16 ? 2 : 4;
  if (((long long)Hkv * D * eb) % 16) return RING_EUNSUPPORTED;   // rows are copied in 16-byte pieces
  if ((long long)B * Smax * Hkv * D >= (1LL << 42) || (long long)B * T * Hkv * D >= (1LL << 42)) return RING_EINVAL;
  AppendArgs a{};
  a.k_cache = k_cache; a.v_cache = v_cache; a.k_new = k_new; a.v_new = v_new;
  a.shard_lens = shard_lens; a.n_appended = n_appended;
  a.B = B; a.T = T; a.Hkv = Hkv; a.Smax = Smax; a.D = D; a.P = P; a.block = block; a.elem_bytes = eb;
  a.err = error_word();
  return from_cuda(launch_kv_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

ring_status ring_attn_merge(const float* partials, const float* part_lse, void* out, float* out_lse, int B, int Hq,
                            int P, int D, int out_dtype, void* stream);

ring_status ring_attn_decode(const void* q, const void* k, const void* v, const int32_t* seqlens, float* partials,
                             float* part_lse, void* out, float* out_lse, int B, int Hq, int Hkv, int Smax, int D,
                             int P, float scale, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  ring_status s = ring_attn_decode_partial(q, k, v, seqlens, partials, part_lse, B, Hq, Hkv, Smax, D, P, scale, dtype,
                                           workspace, workspace_bytes, stream);
  if (s != RING_OK) return s;
  return ring_attn_merge(partials, part_lse, out, out_lse, B, Hq, P, D, RING_BF16, stream);
}

ring_status ring_attn_merge(const float* partials, const float* part_lse, void* out, float* out_lse, int B, int Hq,
                            int P, int D, int out_dtype, void* stream) {
  if (!aligned16(partials) || !part_lse || !aligned16(out)) return RING_EINVAL;
  if (out_lse && (reinterpret_cast<uintptr_t>(out_lse) & 3u)) return RING_EINVAL;
  if (B < 1 || Hq < 1 || P < 1 || D < 1) return RING_EINVAL;
  if (out_dtype != RING_BF16 && out_dtype != RING_FP32) return RING_EINVAL;
  if (D % 4 || D > 1024) return RING_EUNSUPPORTED;
  return from_cuda(launch_merge(partials, part_lse, out, out_lse, B, Hq, P, D, out_dtype == RING_BF16,
                                reinterpret_cast<cudaStream_t>(stream)));
}

ring_status ring_attn_sched_stats(int S, int P, int causal, int layout, int tile_q, int tile_k,
                                  int64_t* per_rank_pairs, int64_t* full, int64_t* partial, int64_t* skipped) {
  if (S < 1 || P < 1 || tile_q < 1 || tile_k < 1) return RING_EINVAL;
  Plan p{};
  if (!ring_split(S, P, layout, &p)) return RING_EINVAL;
  p.B = 1; p.Hq = 1; p.Hkv = 1; p.D = 128;
  p.causal = causal ? 1 : 0;
  int64_t f = 0, pa = 0, sk = 0;
  if (per_rank_pairs)
    for (int r = 0; r < P; ++r) per_rank_pairs[r] = 0;
  const int tq = cdiv(p.C, tile_q), tk = cdiv(p.C, tile_k);
  for (int qs = 0; qs < p.nqc; ++qs) {
    const int r = chunk_owner(p, qs);
    const int qb = q_pos_base(p, qs);
    // pairs: the visiting order of rank r, filtered by the causal rule on chunks
    KvIter it;
    kv_begin(p, qs, it);
    for (; it.idx < p.nkc; kv_next_chunk(p, it)) {
      const int kb = kv_pos_base(p, it.qg, kv_cur_slot(p, it));
      if (!p.causal || kb <= qb + p.C - 1) {
        if (per_rank_pairs) per_rank_pairs[r]++;
      }
      for (int a = 0; a < tq; ++a) {
        const int q0 = qb + a * tile_q, q1 = qb + imin((a + 1) * tile_q, p.C) - 1;
        for (int b = 0; b < tk; ++b) {
          const int k0 = kb + b * tile_k, k1 = kb + imin((b + 1) * tile_k, p.C) - 1;
          const int c = tile_class(p.causal, q0, q1, k0, k1);
          if (c == 0) ++f; else if (c == 1) ++pa; else ++sk;
        }
      }
    }
  }
  if (full) *full = f;
  if (partial) *partial = pa;
  if (skipped) *skipped = sk;
  return RING_OK;
}

ring_status ring_attn_device_error(int* where) {
  if (where) *where = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return RING_ECUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return RING_ECUDA;
  if (word) {
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return RING_ECUDA;
    if (where) *where = (int)word;
    return word == kFaultCapacity ? RING_ECAPACITY : RING_ETIMEOUT;
  }
  return RING_OK;
}

ring_status ring_attn_selftest_wait(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return RING_EINVAL;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(error_word(),
                                                                           (unsigned long long)limit_us * 1000ull);
  return from_cuda(cudaGetLastError());
}

const char* ring_attn_strerror(ring_status s) {
  switch (s) {
    case RING_OK: return "ok";
    case RING_EINVAL: return "invalid argument";
    case RING_EUNSUPPORTED: return "unsupported configuration";
    case RING_ECUDA: return "CUDA error";
    case RING_ETIMEOUT: return "a bounded wait inside a kernel expired";
    case RING_ECAPACITY: return "a KV append found its shard full";
  }
  return "unknown status";
}

int ring_attn_version(void) { return 1; }
int ring_attn_built_arch(void) { return 100; }

}  // extern "C"
