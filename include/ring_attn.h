/*
 * ring_attn.h -- C ABI of a B200 (sm_100a) library for exact ring attention
 * emulated on one GPU.
 *
 * What is computed.  A sequence of S tokens is cut into chunks and dealt to P
 * virtual ranks ("Lesson 8: Context Parallelism", section 1 and Fig. 8-2).
 * Each rank keeps its query shard fixed and meets the K/V blocks of every
 * rank in ring order -- at step t the block that started on rank (r-t) mod P
 * (section 2, Fig. 8-3) -- folding each block into a running state (m, l, O)
 * with the online-softmax update of section 3.  After the full loop each
 * query has seen every allowed key, so the result is exact attention
 * softmax(scale * Q K^T) V (section 1; "Sequence parallelism and ring
 * attention", FAQ).  Causal masking follows section 4 (query i sees keys
 * j <= i, global positions); the contiguous split is section 4A, the zig-zag
 * split (2P chunks, rank r owns chunks r and 2P-1-r) section 4B, with k
 * chunks per rank and the striped split as variants (see ring_layout).  The decode
 * entry points shard the KV cache of one-token queries along the sequence
 * ("NVIDIA unveils Helix Parallelism", Phase 1, KV parallelism) and merge the
 * per-shard partial results.
 *
 * Conventions shared by every entry point.
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no memory and keeps no state except one device error word and
 *     the fixed scratch array of ring_attn_decode_partial_noalloc (reserved
 *     when the library is loaded; see that entry).
 *   - Row-major layouts, last index contiguous:
 *       q, out        [B, S, Hq, D]        k, v  [B, S, Hkv, D]
 *       lse           [B, Hq, S]  float, natural log: lse = m + ln l
 *     Query head h reads K/V head h / (Hq / Hkv) (grouped-query attention).
 *   - dtype RING_BF16: q, k, v, out are bfloat16, accumulation is float32 on
 *     the tensor cores (tcgen05, accumulators in tensor memory).
 *     dtype RING_FP32: q, k, v, out are float32, float32 FMA on CUDA cores.
 *   - Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *     default stream) and does not synchronise the host.
 *   - Pointers must be 16-byte aligned.  Errors are returned, never printed;
 *     nothing aborts.
 *   - RING_ETIMEOUT is reported by ring_attn_device_error(): every wait inside
 *     a kernel is bounded; a wait that expires sets the device error word and
 *     the kernel returns early (its outputs are then undefined).
 */
#ifndef RING_ATTN_H_
#define RING_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RING_OK = 0,
  RING_EINVAL = -1,        /* bad argument: null/misaligned pointer, shape not divisible, ... */
  RING_EUNSUPPORTED = -2,  /* valid but not built: head dim, dtype combination */
  RING_ECUDA = -3,         /* a CUDA runtime / driver call or a launch failed */
  RING_ETIMEOUT = -4,      /* a bounded wait inside a kernel expired */
  RING_ECAPACITY = -5      /* a KV append found its shard full (see ring_attn_kv_append) */
} ring_status;

/*
 * How the sequence is split among the P virtual ranks (the `layout` argument):
 *   RING_CONTIGUOUS  P*k chunks; rank r owns chunks r*k .. r*k+k-1 (section 4A
 *                    of "Lesson 8" for k = 1; the worked example's sequential
 *                    assignment for k > 1).
 *   RING_ZIGZAG      P*k chunks; slot j of rank r is chunk (j/2)*P + r for
 *                    even j and P*k-1-(j/2)*P-r for odd j (section 4B for
 *                    k = 2, chunks r and 2P-1-r; the code exercise for any k).
 *   RING_STRIPED     token t belongs to rank t mod P ("Sequence parallelism and
 *                    ring attention", outlook, which names the striped variant;
 *                    the token rule is this library's reading).
 * The low byte selects the split; RING_SPLIT(split, k) adds the chunks per
 * rank k (1..RING_MAX_CHUNKS_PER_RANK; zig-zag needs k >= 2, striped k = 1).
 * A bare RING_CONTIGUOUS means k = 1, a bare RING_ZIGZAG k = 2.
 */
typedef enum { RING_CONTIGUOUS = 0, RING_ZIGZAG = 1, RING_STRIPED = 2 } ring_layout;
#define RING_MAX_CHUNKS_PER_RANK 8
#define RING_SPLIT(split, k) ((int)(split) | ((int)(k) << 8))
typedef enum { RING_BF16 = 0, RING_FP32 = 1 } ring_dtype;

/* The chunks carried by one ring step (see ring_attn_step). */
typedef struct {
  int32_t n_q;        /* query chunks in the shard: 1..RING_MAX_CHUNKS_PER_RANK  */
  int32_t q[RING_MAX_CHUNKS_PER_RANK];   /* their chunk indices, in shard order  */
  int32_t n_kv;       /* K/V chunks in the block: 1..RING_MAX_CHUNKS_PER_RANK    */
  int32_t kv[RING_MAX_CHUNKS_PER_RANK];  /* their chunk indices, in buffer order */
  int32_t chunk_len;  /* rows per chunk (all chunks have this length)            */
  int32_t causal;     /* 1: key at position j is allowed for query i iff j <= i  */
  int32_t stripes;    /* 0: chunked split, row x of chunk c is position c*chunk_len + x.
                         P > 0: striped split over P ranks; q[0] and kv[0] are
                         ranks (< P), row x of rank c's stripe is position
                         x*P + c, and n_q = n_kv = 1.                           */
} ring_chunk_ids;

/*
 * ring_attn_fwd -- the whole ring loop of every virtual rank, fused in one
 * persistent launch ("Lesson 8", sections 2-4).
 *
 * q [B,S,Hq,D], k/v [B,S,Hkv,D] in natural token order; out [B,S,Hq,D] (same
 * dtype as q), lse [B,Hq,S] float.  The sequence is split into P chunks
 * (layout RING_CONTIGUOUS, chunk length S/P), 2P chunks (RING_ZIGZAG, chunk
 * length S/(2P)), P*k chunks (RING_SPLIT(..., k)) or P stripes of S/P
 * tokens (RING_STRIPED).  For every rank and every query tile the kernel folds
 * K/V tiles into the on-chip (m, l, O) state in the rank's ring order,
 * skipping tiles that the causal mask removes entirely; the state never
 * leaves the chip between ring steps.
 *
 * Returns RING_EINVAL for a null or misaligned pointer, B/Hq/Hkv/S/P < 1,
 * Hq % Hkv != 0, S not divisible by the number of chunks (or stripes), layout
 * or dtype out of range, or a non-finite / non-positive scale; RING_EUNSUPPORTED for
 * D not in {64, 128}; RING_ECUDA if a launch fails.
 */
ring_status ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                          int B, int Hq, int Hkv, int S, int D, int P, int causal, int layout,
                          float scale, int dtype, void* stream);

/*
 * ring_attn_fwd_counted -- ring_attn_fwd that also counts, on the device, the
 * work the scheduler actually issued.  `counters` is a device array of
 * (2 + P) uint64 that the call ADDS to (zero it first):
 *   counters[0]      128x128 tiles computed without a mask, summed over (b, hq)
 *   counters[1]      128x128 tiles computed with the causal / ragged mask
 *   counters[2 + r]  causal chunk pairs (query chunk, K/V chunk) with at least
 *                    one allowed key met by virtual rank r, summed over (b, hq)
 * Tiles are 128 query rows x 128 keys cut inside each chunk pair (the last
 * tile of a chunk may be shorter).  Only dtype RING_BF16 counts; other
 * arguments and errors as ring_attn_fwd.
 * Instrumentation of the scheduler: the per-rank pair counts are those of
 * "Lesson 8", section 4B (2P+1 per zig-zag rank) and section 4A (r+1 per
 * contiguous rank).
 */
ring_status ring_attn_fwd_counted(const void* q, const void* k, const void* v, void* out, float* lse,
                                  int B, int Hq, int Hkv, int S, int D, int P, int causal, int layout,
                                  float scale, int dtype, unsigned long long* counters, void* stream);

/*
 * ring_attn_fwd_simt -- the same computation as ring_attn_fwd on CUDA cores
 * with float32 FMA for both dtypes (bf16 inputs are widened exactly).  Slow;
 * it exists to cross-check the tensor-core path on the GPU.  Arguments and
 * errors as ring_attn_fwd.
 * The computation is that of "Lesson 8", sections 2-4.
 */
ring_status ring_attn_fwd_simt(const void* q, const void* k, const void* v, void* out, float* lse,
                               int B, int Hq, int Hkv, int S, int D, int P, int causal, int layout,
                               float scale, int dtype, void* stream);

/*
 * ring_attn_state_init -- set a ring state to its starting value
 * m = -inf, l = 0, O = 0 ("Lesson 8", section 3, before the first block).
 * m, l [B,Hq,S_loc] float; O [B,S_loc,Hq,D] float.  Returns RING_EINVAL for
 * null/misaligned pointers, sizes < 1 or D % 4 != 0; RING_ECUDA on launch
 * failure.
 */
ring_status ring_attn_state_init(float* m, float* l, float* O, int B, int Hq, int S_loc, int D,
                                 void* stream);

/*
 * ring_attn_step -- one hop of the ring for one rank ("Lesson 8", section 2:
 * local attention of the fixed Q_r against the K/V block currently held,
 * merged into O_r with the section-3 update).
 *
 * q_shard [B, n_q*C, Hq, D]: the rank's query chunks ids->q[0..n_q) stacked in
 * that order (C = ids->chunk_len); kchunk, vchunk [B, n_kv*C, Hkv, D]: the
 * held K/V chunks ids->kv[0..n_kv) stacked in that order.  For the striped
 * split (ids->stripes = P) the shard is rank ids->q[0]'s stripe in token
 * order and the block is rank ids->kv[0]'s stripe.  State, read and written
 * in place:  m, l [B, Hq, n_q*C] float (m is the running max of the scaled
 * scores, natural units; l = sum exp(s - m)) and O [B, n_q*C, Hq, D] float,
 * normalised (O = sum exp(s - m) v / l), as in section 3.  Rows whose block
 * has no allowed key keep their state.  Fully masked tiles are skipped.
 * A bf16 step may begin while the previous kernel on the stream is finishing
 * (programmatic dependent launch); it reads the state only after that kernel
 * has completed, so consecutive steps on one stream need no synchronisation.
 *
 * Returns RING_EINVAL for null/misaligned pointers, ids == NULL, n_q or n_kv
 * outside 1..RING_MAX_CHUNKS_PER_RANK, chunk_len < 1, negative chunk ids,
 * stripes < 0, a striped step with n_q or n_kv != 1 or a rank >= stripes,
 * Hq % Hkv != 0, bad dtype or scale; RING_EUNSUPPORTED for D not in {64,128};
 * RING_ECUDA on launch failure.
 */
ring_status ring_attn_step(const void* q_shard, const void* kchunk, const void* vchunk,
                           float* m, float* l, float* O, const ring_chunk_ids* ids,
                           int B, int Hq, int Hkv, int D, float scale, int dtype, void* stream);

/*
 * ring_attn_state_finalize -- out = O (cast to dtype), lse = m + ln l, for a
 * state produced by ring_attn_step.  out [B,S_loc,Hq,D]; lse [B,Hq,S_loc].
 * A row with l == 0 gets out = 0 and lse = -inf.  Returns RING_EINVAL for
 * null/misaligned pointers, sizes < 1 or a dtype out of range; RING_ECUDA on
 * launch failure.
 * "Lesson 8", section 3 keeps (m, l); lse = m + ln l is this library's
 * reading of the log-sum-exp of that state.
 */
ring_status ring_attn_state_finalize(const float* m, const float* l, const float* O, void* out,
                                     float* lse, int B, int Hq, int S_loc, int D, int dtype,
                                     void* stream);

/*
 * Backward pass.  The pages use the ring for training but give no backward;
 * the gradients are the calculus of the forward (L = sum(dout * out)):
 *   P = exp(scale * Q K^T - lse),  dP = dout V^T,  delta_i = dout_i . out_i,
 *   dS = P o (dP - delta),  dV = P^T dout,  dK = scale * dS^T Q,
 *   dQ = scale * dS K   (dK, dV summed over the query heads of a group).
 * P is recomputed from the forward's lse, tile by tile, in the ring's order:
 * a K/V block gathers dK, dV from the query chunks it meets as it travels
 * round the ring ("Lesson 8", section 2); each rank's dQ gathers from the
 * blocks it meets.  bf16: tensor cores (bf16 products, fp32 accumulation);
 * float32: CUDA cores.
 */

/* Bytes of workspace ring_attn_bwd needs (the delta rows); 0 on bad sizes. */
size_t ring_attn_bwd_workspace_bytes(int B, int Hq, int S);

/*
 * ring_attn_bwd_delta -- delta[b,h,i] = sum_d dout[b,i,h,d] * out[b,i,h,d]
 * for out, dout [B,S,Hq,D] of `dtype`; delta [B,Hq,S] float.  Returns
 * RING_EINVAL for null/misaligned pointers, sizes < 1 or a dtype out of
 * range; RING_ECUDA on launch failure.
 * The pages give no backward (see the backward pass above).
 */
ring_status ring_attn_bwd_delta(const void* out, const void* dout, float* delta, int B, int Hq, int S, int D,
                                int dtype, void* stream);

/*
 * ring_attn_bwd -- gradients of the whole ring of ring_attn_fwd.
 * q, out, dout, dq [B,S,Hq,D]; k, v, dk, dv [B,S,Hkv,D], all of `dtype`;
 * lse [B,Hq,S] float as written by the forward.  Split, causal rule, scale and
 * errors as ring_attn_fwd; workspace (ring_attn_bwd_workspace_bytes bytes,
 * 256-byte aligned) receives delta.  dq, dk, dv are overwritten; the results
 * do not depend on the launch order of tiles (no atomics).
 * The pages give no backward (see the backward pass above).
 */
ring_status ring_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S, int D,
                          int P, int causal, int layout, float scale, int dtype, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * ring_attn_bwd_simt -- ring_attn_bwd on CUDA cores with float32 FMA for both
 * dtypes (the bf16 ring_attn_bwd runs on the tensor cores: tcgen05 products
 * of 128 x 128 tiles, fp32 accumulation in tensor memory).  Slow; it exists
 * to cross-check the tensor-core path.  Arguments and errors as ring_attn_bwd.
 * The pages give no backward (see the backward pass above).
 */
ring_status ring_attn_bwd_simt(const void* q, const void* k, const void* v, const void* out, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S, int D,
                               int P, int causal, int layout, float scale, int dtype, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * ring_attn_step_bwd -- one hop of the backward ring for one rank: the
 * gradients of attention of the rank's query shard against the K/V block it
 * holds.  q_shard, dout_shard [B, n_q*C, Hq, D] and kchunk, vchunk
 * [B, n_kv*C, Hkv, D] as in ring_attn_step; lse, delta [B, Hq, n_q*C] float of
 * the WHOLE forward (lse of the full attention, delta from its output).
 * Adds, in place: dq_acc [B, n_q*C, Hq, D] float (this block's share of the
 * shard's dQ) and dk_acc, dv_acc [B, n_kv*C, Hkv, D] float (the shard's share
 * of the block's dK, dV, which travel with the block).  Errors as
 * ring_attn_step.
 * The pages give no backward; the hop mirrors the forward's ring step
 * ("Lesson 8", section 2).
 */
ring_status ring_attn_step_bwd(const void* q_shard, const void* kchunk, const void* vchunk, const void* dout_shard,
                               const float* lse, const float* delta, float* dq_acc, float* dk_acc, float* dv_acc,
                               const ring_chunk_ids* ids, int B, int Hq, int Hkv, int D, float scale, int dtype,
                               void* stream);

/*
 * ring_attn_decode_partial -- split-KV single-token decode, the KV cache
 * sharded along the sequence into P chunks ("Helix Parallelism", Phase 1).
 *
 * q [B,Hq,D] bf16 (one query token per sequence); k, v [B,Smax,Hkv,D] bf16;
 * seqlens [B] int32 on the device (keys j < seqlens[b] are valid; 0 <= seqlens
 * <= Smax, checked by the kernel: out-of-range entries are clamped and raise
 * no fault).  Chunk p covers rows [p*Smax/P, (p+1)*Smax/P).  Writes, per
 * (b, hq, p), the normalised partial output partials[B,Hq,P,D] float and
 * part_lse[B,Hq,P] float; a chunk with no valid key gives O = 0 and
 * lse = -inf.  Inside a chunk the rows are further split across CTAs and
 * recombined with the same update; `workspace` (device, at least
 * ring_attn_decode_workspace_bytes(...) bytes, 256-byte aligned) holds those
 * sub-results and per-chunk arrival counters.  The counters must be zero
 * before the first call on a workspace; every call that completes leaves them
 * zero again.  A call cut short by an expired wait (ring_attn_device_error
 * returns RING_ETIMEOUT) may leave them non-zero: zero the workspace again
 * before its next use.  Calls that share a workspace must not overlap on the
 * GPU.
 *
 * Returns RING_EINVAL for null/misaligned pointers, Smax % P != 0, shapes < 1,
 * Hq % Hkv != 0, workspace too small; RING_EUNSUPPORTED unless dtype ==
 * RING_BF16, D is 64 or 128 and Hq / Hkv is 1, 2, 4, 8 or 16 (the query heads
 * of a kv head are the columns of the kernel's tensor-core products, padded to
 * 16);
 * RING_ECUDA on launch failure.
 */
ring_status ring_attn_decode_partial(const void* q, const void* k, const void* v,
                                     const int32_t* seqlens, float* partials, float* part_lse,
                                     int B, int Hq, int Hkv, int Smax, int D, int P, float scale,
                                     int dtype, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Bytes of workspace ring_attn_decode_partial needs for these sizes (0 on bad sizes).
 * A library helper; the pages have no counterpart. */
size_t ring_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Smax, int D, int P);

/*
 * ring_attn_decode_partial_noalloc -- ring_attn_decode_partial without a
 * workspace argument and without any allocation.  (The pages have no
 * counterpart: this is an interface convenience of the library.)
 *
 * For callers that cannot call cudaMalloc or pass a workspace: a host program
 * whose own allocator owns all device memory (a fixed budget, or a caching
 * pool that must not be bypassed), or code on a latency-critical path where an
 * allocation, which may synchronise the device, is not acceptable.
 *
 * The scratch lives in one fixed array of RING_DECODE_NOALLOC_SCRATCH_BYTES
 * bytes inside the library, reserved on every GPU that loads the library and
 * held until the process exits.  Sizes whose scratch need
 * (ring_attn_decode_workspace_bytes) exceeds that maximum are rejected with
 * RING_EINVAL before anything is launched; the B8 Hq32 Hkv8 D128 2^20-token,
 * 32-chunk decode needs about 17 MB.  The first call on a device looks up the
 * array's device address (with that device current); make that first call
 * before any stream capture.  Each call clears the array's arrival counters
 * on `stream`, then launches the same kernel as ring_attn_decode_partial.
 * No call allocates: no cudaMalloc, cudaFree or allocating library routine.
 * All calls share the one array, so calls that overlap on the GPU (other
 * streams, other host threads) race and give wrong results: serialise them.
 * Other arguments, outputs and errors as ring_attn_decode_partial.
 */
#define RING_DECODE_NOALLOC_SCRATCH_BYTES (40u << 20)
ring_status ring_attn_decode_partial_noalloc(const void* q, const void* k, const void* v,
                                             const int32_t* seqlens, float* partials, float* part_lse,
                                             int B, int Hq, int Hkv, int Smax, int D, int P, float scale,
                                             int dtype, void* stream);

/*
 * ring_attn_merge -- combine P normalised partial results per (b, hq):
 *   lse = m* + ln sum_p exp(lse_p - m*),  m* = max_p lse_p
 *   out = sum_p exp(lse_p - lse) O_p
 * (the section-3 update of "Lesson 8" applied to whole partial states).
 * partials [B,Hq,P,D] float, part_lse [B,Hq,P] float; out [B,Hq,D] of
 * out_dtype (RING_BF16 or RING_FP32), out_lse [B,Hq] float (may be NULL).
 * If every part is empty: out = 0, lse = -inf.
 * Returns RING_EINVAL / RING_EUNSUPPORTED (D not a multiple of 4 or > 1024) /
 * RING_ECUDA.
 */
ring_status ring_attn_merge(const float* partials, const float* part_lse, void* out, float* out_lse,
                            int B, int Hq, int P, int D, int out_dtype, void* stream);

/*
 * ring_attn_decode -- the whole split-KV decode: ring_attn_decode_partial
 * followed by ring_attn_merge on the same stream.  partials / part_lse are
 * the caller's buffers for the per-chunk results (as above); out [B,Hq,D]
 * bf16 and out_lse [B,Hq] float (may be NULL) receive attention over all
 * seqlens[b] keys.  Errors as the two calls.
 * The split-KV decode of "NVIDIA unveils Helix Parallelism", Phase 1.
 */
ring_status ring_attn_decode(const void* q, const void* k, const void* v, const int32_t* seqlens, float* partials,
                             float* part_lse, void* out, float* out_lse, int B, int Hq, int Hkv, int Smax, int D,
                             int P, float scale, int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * ring_attn_decode_fused -- the whole split-KV decode in ONE launch: the
 * per-chunk partials of ring_attn_decode_partial, and the merge of
 * ring_attn_merge done by the CTA that finishes the last of the P chunks of
 * each (sequence, kv head) ("NVIDIA unveils Helix Parallelism", Phase 1: the
 * KV-parallel partial results are combined once per token; the combine is
 * the section-3 update of "Lesson 8" applied to whole partial states).
 *
 * Valid rows come from exactly one of:
 *   seqlens [B] int32     rows j < seqlens[b] of the whole cache (chunk p
 *                         covers rows [p*Smax/P, (p+1)*Smax/P)), as in
 *                         ring_attn_decode_partial;
 *   shard_lens [B,P] int32  the first shard_lens[b*P+p] rows of chunk p (a
 *                         cache filled shard by shard, e.g. by
 *                         ring_attn_kv_append); other rows are ignored.
 * Pass the other pointer as NULL.  Lengths outside their range are clamped.
 * partials [B,Hq,P,D] / part_lse [B,Hq,P] float receive the per-chunk results
 * as in ring_attn_decode_partial (caller buffers, also read by the merge);
 * out [B,Hq,D] bf16 and out_lse [B,Hq] float (may be NULL) the merged
 * result.  The workspace is ring_attn_decode_workspace_bytes(...) bytes,
 * 256-byte aligned; its counters must be zero before the first call on it and
 * every call that completes leaves them zero (after RING_ETIMEOUT, zero it
 * again).  Calls that share a workspace must not overlap on the GPU.  Errors
 * as ring_attn_decode_partial, plus RING_EINVAL unless
 * exactly one of seqlens / shard_lens is given, or for a null or misaligned
 * out.
 */
ring_status ring_attn_decode_fused(const void* q, const void* k, const void* v, const int32_t* seqlens,
                                   const int32_t* shard_lens, float* partials, float* part_lse, void* out,
                                   float* out_lse, int B, int Hq, int Hkv, int Smax, int D, int P, float scale,
                                   int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * ring_attn_kv_append -- append T new tokens per sequence to a KV cache
 * sharded over P KV-parallel ranks, round-robin by blocks ("NVIDIA unveils
 * Helix Parallelism", on growing the KV cache: successive blocks of new
 * tokens go to successive ranks, wrapping after the last, so every rank's
 * share grows at the same pace).
 *
 * k_cache, v_cache [B,Smax,Hkv,D]: rank p's shard is rows [p*C, (p+1)*C),
 * C = Smax/P, of which the first shard_lens[b*P+p] are filled.  k_new, v_new
 * [B,T,Hkv,D] hold the new tokens in order.  n_appended [B] counts the tokens
 * appended to each sequence so far (0 after the prompt).  Token j of sequence
 * b has append index n = n_appended[b] + j and goes to rank (n / block) mod P,
 * at row shard_lens[b*P+p] of that shard (after the earlier tokens of this
 * call that went there).  On return shard_lens and n_appended have advanced.
 * All of these are device buffers; lengths outside [0, C] (counts below 0)
 * are clamped.  A token whose shard is full is not written, the shard's
 * count stays at C, and the next ring_attn_device_error() reports
 * RING_ECAPACITY; nothing is written outside the shard.
 * dtype RING_BF16 or RING_FP32 (the element type of cache and tokens).
 * Returns RING_EINVAL for null/misaligned pointers, sizes < 1, Smax % P != 0,
 * block < 1; RING_EUNSUPPORTED if a token row (Hkv*D elements) is not a
 * multiple of 16 bytes; RING_ECUDA on launch failure.
 */
ring_status ring_attn_kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                                int32_t* shard_lens, int32_t* n_appended, int B, int T, int Hkv, int Smax,
                                int D, int P, int block, int dtype, void* stream);

/*
 * ring_attn_sched_stats -- the scheduler's host-side view of one (batch, head)
 * of a causal or full ring, without running anything: per-rank unmasked
 * chunk pairs (a diagonal pair counts once; "Lesson 8", section 4B: 2P+1 per
 * zig-zag rank, section 4A: r+1 per contiguous rank; a striped pair counts
 * if any key precedes a query) and tile classes for tile_q x tile_k tiles
 * cut inside each chunk pair (full: no mask needed; partial: masked;
 * skipped: fully masked, never issued).  `layout` as for ring_attn_fwd.
 * per_rank_pairs has room for P values.  Any output pointer may be NULL.
 * Returns RING_EINVAL for S, P, tile_q or tile_k < 1, or a split out of range
 * or not dividing S; it touches no device.
 */
ring_status ring_attn_sched_stats(int S, int P, int causal, int layout, int tile_q, int tile_k,
                                  int64_t* per_rank_pairs, int64_t* full, int64_t* partial,
                                  int64_t* skipped);

/*
 * ring_attn_device_error -- synchronise the current device and read-and-clear
 * the library's device error word.  Returns RING_ETIMEOUT if a bounded wait
 * in any kernel expired since the last call, RING_ECAPACITY if a KV append
 * dropped a token because its shard was full, RING_ECUDA if the device
 * reports an error, else RING_OK.  `where` (may be NULL) receives the code
 * of the site that recorded the error (0 if none).  Code 12 (reported as
 * RING_ETIMEOUT: the kernel unwound without results) means a CTA pair of the
 * prefill kernel found its cluster ranks numbered otherwise than the blocks
 * 2c, 2c+1 it assumes.
 * A library helper; the pages have no counterpart.
 */
ring_status ring_attn_device_error(int* where);

/*
 * ring_attn_selftest_wait -- launch one thread that waits on an mbarrier no
 * one completes, giving up after limit_us microseconds (1..1e6) exactly as
 * every wait inside the library's kernels gives up after its own limit.  The
 * next ring_attn_device_error() then reports RING_ETIMEOUT.  No fault, trap
 * or hang is involved; it exists to test the error path.
 * A library helper; the pages have no counterpart.
 */
ring_status ring_attn_selftest_wait(int limit_us, void* stream);

/* A static, human-readable name for a status code; an unknown code gives
 * "unknown status".  Never fails.
 * A library helper; the pages have no counterpart. */
const char* ring_attn_strerror(ring_status status);

/* Library version and the SM architecture it was compiled for (e.g. 100).
 * Both are constants of the build and never fail.
 * Library helpers; the pages have no counterpart. */
int ring_attn_version(void);
int ring_attn_built_arch(void);

#ifdef __cplusplus
}
#endif

#endif /* RING_ATTN_H_ */
