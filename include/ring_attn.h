/*
 * ring_attn.h -- C ABI of the exact blockwise (ring) attention library for
 * NVIDIA B200 (sm_100a).  Shared object: libringattn.so.
 *
 * The operation (attention definition on "Billion-token context window
 * engineering", core-challenge paragraph, and "Ring Attention: the secret of
 * million-token context" §2.3): for every batch b, query head h and query
 * row t,
 *     out[b,t,h,:] = sum_j softmax_j(scale * q[b,t,h,:] . k[b,j,hk,:]) v[b,j,hk,:]
 *     lse[b,h,t]   = ln sum_j exp(scale * q[b,t,h,:] . k[b,j,hk,:])
 * over the keys j visible to row t, computed blockwise: the KV sequence is
 * cut into P chunks ("Ring Attention..." §2.1) and each query chunk i visits
 * KV chunk (i+s) mod P at step s (§2.2 figure), folding each visit into
 * running (max, sum, output) statistics (§3.1 two-level loop) that are
 * normalised once over all keys ("From hundreds of milliseconds to a million
 * tokens", system layer 4: global softmax normalisation).
 *
 * Conventions shared by every entry point
 *   - Layouts are row-major and contiguous, token-major:
 *       q, out        [B, N_q,  Hq,  d]
 *       k, v          [B, N_kv, Hkv, d]
 *       lse           [B, Hq, N_q]           float32, natural log
 *       acc           [B, Hq, Lq, d]         float32 running numerator
 *       m, l          [B, Hq, Lq]            float32 running max / sum
 *       o_parts       [S, B, N_q, Hq, d]     float32, each part normalised
 *       lse_parts     [S, B, Hq, N_q]        float32
 *   - GQA: query head h reads KV head h / (Hq / Hkv); Hq % Hkv == 0.
 *   - Causal masking is per token: key position p_k is visible to query
 *     position p_q iff p_k <= p_q ("RingAttention inference: using
 *     cache_idx", basic configuration: causal_block_size = 1).
 *   - d must be 64 or 128.  bf16 entry points need every pointer 16-byte
 *     aligned (the tensor-memory-access unit reads them).
 *   - Every pointer named q, k, v, out, lse, acc, m, l, o_parts, lse_parts
 *     is DEVICE memory owned by the caller; the library keeps no reference
 *     after the call returns and frees nothing it did not allocate.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work
 *     is enqueued asynchronously on it; no call synchronises unless the
 *     environment variable RINGATTN_DEBUG=1 is set (then each call
 *     synchronises and also reports the device status word).
 *   - RINGATTN_NVTX=1 wraps every compute entry point in an NVTX range named
 *     after it, for profilers; with no profiler attached it does nothing.
 *   - Every call returns a ring_attn_status.  Arguments are validated on the
 *     host before anything is launched; an invalid call launches nothing.
 *     ring_attn_error_string() turns a status into text; after
 *     RA_ERR_CUDA, ring_attn_last_error() holds the CUDA message.
 *   - A row with no visible key (possible only through block_step or
 *     lse_merge inputs that cover no key for it) gives out = 0, lse = -inf.
 */
#ifndef RING_ATTN_H_
#define RING_ATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, bad d, Hq % Hkv != 0, N_kv != P*chunk, ... */
  RA_ERR_UNSUPPORTED = 2,    /* the current device is not sm_100 */
  RA_ERR_CUDA = 3,           /* a CUDA call or kernel launch failed; see ring_attn_last_error() */
  RA_ERR_DEVICE_TIMEOUT = 4, /* a kernel's bounded wait expired; its outputs are undefined */
  RA_ERR_OOM = 5             /* stream-ordered workspace allocation failed */
} ring_attn_status;

#define RA_DTYPE_BF16 0
#define RA_DTYPE_F32 1

/*
 * ring_attn_fwd -- full forward pass, bf16 q/k/v/out, float32 lse.
 *
 * The sequence of N_kv keys is cut into P chunks of `chunk` tokens
 * ("Ring Attention..." §2.1); N_kv == P * chunk is required (a length that is
 * not a multiple of P is rejected, the pitfall listed in "RingAttention and
 * RAG compared", §2.3).
 *   cache_idx == -1: prefill.  N_q == N_kv; query row t sits at position t
 *       and belongs to query chunk i = t / chunk, which visits KV chunk
 *       (i+s) mod P at step s.
 *   cache_idx >= 0: incremental query ("RingAttention inference: using
 *       cache_idx", how cache_idx works).  Query row t sits at position
 *       cache_idx + t; cache_idx + N_q <= N_kv is required; the block of
 *       queries is homed at chunk cache_idx / chunk.  The KV cache holds the
 *       new tokens' own keys.  This path splits the KV range over several
 *       CTAs and merges their partials (a stream-ordered workspace of
 *       about S*B*N_q*Hq*(d+1)*4 bytes is allocated and freed on `stream`).
 * scale multiplies q.k (1/sqrt(d) for standard attention).  The result does
 * not depend on P or chunk except through rounding.
 * Returns RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_CUDA or
 * RA_ERR_OOM.
 */
int ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                  int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d,
                  int causal, int64_t chunk, int P, int64_t cache_idx, float scale,
                  void* stream);

/*
 * ring_attn_fwd_host -- ring_attn_fwd for inputs and results in HOST memory,
 * with the copies overlapped with the compute.
 *
 * Attention heads are independent problems (in the definition above, every
 * (b, h) has its own softmax over its own keys), so the call cuts the KV
 * heads into groups of `kv_heads_per_group` (with their
 * Hq / Hkv query heads each) and streams them through two device staging
 * slots: while group g is computed, group g + 1 is copied in and group g - 1
 * copied out.  A step then costs about its host-to-device transfer instead
 * of transfer + compute + transfer back.
 *
 * q, k, v, out, lse: HOST pointers with the layouts of ring_attn_fwd
 * ([B, N, H, d] bf16, lse [B, Hq, N_q] float32), owned by the caller.
 * Page-locked memory (cudaHostAlloc / pinned tensors) is needed for the
 * copies to overlap; pageable memory gives the same result without overlap.
 * Other arguments as ring_attn_fwd; each group is computed exactly as
 * ring_attn_fwd computes it (the split-KV count of an incremental query is
 * chosen per group).
 * kv_heads_per_group: 0 = the fewest KV heads per group that give at most
 * sixteen groups; else it must divide Hkv (RA_ERR_INVALID_ARG otherwise).
 *
 * Asynchronous like ring_attn_fwd: the pipeline starts after the work queued
 * on `stream` and `stream` waits for all of it, so out and lse are complete
 * once `stream` has been synchronised (ring_attn_sync_status).  The caller
 * keeps q, k, v, out and lse allocated and unmodified until then.  The library
 * uses four internal streams per device, created on the first call, and a
 * stream-ordered staging allocation on `stream` of
 * 2 x (2 B N_q hg d 2 + 2 B N_kv kvg d 2 + B hg N_q 4) bytes (hg, kvg: query
 * and KV heads per group), freed on `stream` when the pipeline ends.
 * Returns as ring_attn_fwd; RA_ERR_OOM when the staging allocation fails.
 */
int ring_attn_fwd_host(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d,
                       int causal, int64_t chunk, int P, int64_t cache_idx, float scale,
                       int kv_heads_per_group, void* stream);

/*
 * ring_attn_fwd_f32 -- the same operation with float32 q/k/v/out, computed
 * in float32 on CUDA cores (no TF32 tensor cores: the float32 path is held
 * to 1e-4 absolute error).  Same arguments, conventions and statuses.
 */
int ring_attn_fwd_f32(const float* q, const float* k, const float* v, float* out, float* lse,
                      int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d,
                      int causal, int64_t chunk, int P, int64_t cache_idx, float scale,
                      void* stream);

/*
 * ring_attn_block_step -- one ring visit ("Ring Attention..." §3.1: the
 * flash-attention call on one received KV chunk).  Folds the attention of
 * q_chunk [B, Lq, Hq, d] (global positions q_off + t) against
 * k_chunk/v_chunk [B, Lk, Hkv, d] (global positions k_off + j) into the
 * caller's running state, in place:
 *     m'   = max(m, max_j s_j)             s_j = scale * q . k_j (masked: -inf)
 *     l'   = exp(m - m') l + sum_j exp(s_j - m')
 *     acc' = exp(m - m') acc + sum_j exp(s_j - m') v_j
 * m is in natural-log units.  The empty state is acc = 0, m = -inf, l = 0;
 * a visit whose keys are all masked leaves a row unchanged.
 * dtype selects the element type of q/k/v chunks: RA_DTYPE_BF16 or
 * RA_DTYPE_F32.  acc/m/l are always float32 and are read and written.
 */
int ring_attn_block_step(const void* q_chunk, const void* k_chunk, const void* v_chunk,
                         int64_t q_off, int64_t k_off, float* acc, float* m, float* l,
                         int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d,
                         int causal, float scale, int dtype, void* stream);

/*
 * ring_attn_finalize -- out = acc / l, lse = m + ln l (rows with l == 0 give
 * out = 0, lse = -inf).  acc [B, Hq, Lq, d], m/l [B, Hq, Lq] in; out
 * [B, Lq, Hq, d] of type out_dtype (RA_DTYPE_BF16 or RA_DTYPE_F32) and lse
 * [B, Hq, Lq] out.  This is the global normalisation step of "From hundreds
 * of milliseconds to a million tokens", system layer 4.
 */
int ring_attn_finalize(const float* acc, const float* m, const float* l, void* out, float* lse,
                       int B, int Hq, int64_t Lq, int d, int out_dtype, void* stream);

/*
 * lse_merge -- merge S normalised partial results by their log-sum-exp
 * weights (the same global normalisation, applied to partials that each
 * cover a disjoint key range):
 *     M = max_s lse_s,  w_s = exp(lse_s - M),  lse = M + ln sum_s w_s,
 *     out = sum_s w_s O_s / sum_s w_s
 * o_parts [S, B, N_q, Hq, d] float32, lse_parts [S, B, Hq, N_q] float32 in;
 * out [B, N_q, Hq, d] (out_dtype) and lse [B, Hq, N_q] out.  A partial with
 * lse = -inf carries no weight; a row whose partials are all -inf gives
 * out = 0, lse = -inf.  S >= 1.
 */
int lse_merge(const float* o_parts, const float* lse_parts, int S, void* out, float* lse,
              int B, int Hq, int64_t N_q, int d, int out_dtype, void* stream);

/*
 * ring_attn_bwd -- gradients of ring_attn_fwd (bf16), for training.  The
 * pages define the forward only (and use it for training: Ring Attention
 * with FSDP in "Billion-token context window engineering", production
 * parameters); the backward is the gradient of that definition:
 *     D_t = dout_t . out_t,  p_tj = exp(scale q_t . k_j - lse_t) on visible pairs,
 *     ds_tj = p_tj (dout_t . v_j - D_t),
 *     dq_t = scale sum_j ds_tj k_j,  dk_j = scale sum_t ds_tj q_t,
 *     dv_j = sum_t p_tj dout_t   (dk, dv summed over a GQA group's heads).
 * q, out, dout, dq: [B, N_q, Hq, d] bf16; k, v, dk, dv: [B, N_kv, Hkv, d]
 * bf16; lse: [B, Hq, N_q] float32 as returned by ring_attn_fwd (out too).
 * causal / cache_idx / scale as in ring_attn_fwd.  Every element of dq, dk
 * and dv is written (zero for rows with no visible partner).  A stream-
 * ordered workspace of 2 * B * Hq * ceil(N_q / 128) * 128 floats is
 * allocated and freed on `stream`.  Returns RA_OK, RA_ERR_INVALID_ARG,
 * RA_ERR_UNSUPPORTED, RA_ERR_CUDA or RA_ERR_OOM.
 */
int ring_attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv,
                  int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d,
                  int causal, int64_t cache_idx, float scale, void* stream);

/*
 * ring_attn_fwd_fp8kv -- ring_attn_fwd over a KV cache stored as FP8 E4M3
 * codes (the pages' quantised KV cache for serving: "Billion-token context
 * window engineering", production parameters; "RingAttention vs RAG" §2.3;
 * "From hundreds of milliseconds to a million tokens", KV-cache
 * compression).  k8, v8: [B, N_kv, Hkv, d] E4M3 codes (one byte each);
 * k_scale, v_scale: [B, Hkv] float32.  The keys and values attended to are
 *     k[b, j, h, :] = e4m3(k8[b, j, h, :]) * k_scale[b, h]   (v likewise),
 * and out / lse are exact attention over them, as ring_attn_fwd computes
 * them (q, out bf16; lse float32; same shapes, causal, chunk, P, cache_idx
 * and scale rules; incremental queries use split-KV partials and a stream-
 * ordered workspace).  Decode-shaped blocks (d = 128, at most 16 packed
 * query rows per KV head) use the tensor cores' 8-bit path with the codes as
 * operands (the bf16 queries and the probabilities each split exactly into
 * two E4M3 planes); other shapes read the codes decoded to bf16, which is
 * exact for every E4M3 value.  Scales must be finite with
 * |k_scale| * scale < 177 (any usable logit range).  All pointers are device memory
 * owned by the caller; q, k8, v8, out 16-byte aligned.  Returns RA_OK,
 * RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_CUDA or RA_ERR_OOM.
 */
int ring_attn_fwd_fp8kv(const void* q, const void* k8, const void* v8, const float* k_scale,
                        const float* v_scale, void* out, float* lse, int B, int Hq, int Hkv,
                        int64_t N_q, int64_t N_kv, int d, int causal, int64_t chunk, int P,
                        int64_t cache_idx, float scale, void* stream);

/*
 * ring_attn_fwd_window_anchor -- ring_attn_fwd (bf16, square prefill,
 * N_q == N_kv == N) under the sparse mask of "Ring Attention: the secret of
 * million-token context" §4.3 instead of the causal one: query i attends to
 * its local window, keys max(0, i - window) .. i, and to the anchors of its
 * period A = anchor_period: with a = floor(i / A) * A, the keys a, a - 1
 * (a > 0) and a + A (when a < N - A; that key lies after i).  Tiles that
 * hold none of a row block's keys are skipped.  The result is exact
 * attention under that mask (approximate attention with respect to the
 * full causal one).  window in [0, N]; anchor_period > 0 and a multiple of
 * 256.  Layouts, chunk / P, scale, ownership and status codes as
 * ring_attn_fwd.
 */
int ring_attn_fwd_window_anchor(const void* q, const void* k, const void* v, void* out, float* lse,
                                int B, int Hq, int Hkv, int64_t N, int d, int64_t chunk, int P,
                                int64_t window, int64_t anchor_period, float scale, void* stream);

/*
 * ring_attn_fwd_window_anchor_host -- ring_attn_fwd_window_anchor for inputs
 * and results in HOST memory, with the copies overlapped with the compute
 * exactly as ring_attn_fwd_host (KV-head groups of `kv_heads_per_group`,
 * 0 = at most sixteen groups, streamed through two device staging slots).
 * The mask is per (query, key) position, so each group is computed exactly as
 * ring_attn_fwd_window_anchor computes those heads.  Pointers, lifetimes,
 * staging and returns as ring_attn_fwd_host.
 */
int ring_attn_fwd_window_anchor_host(const void* q, const void* k, const void* v, void* out, float* lse,
                                     int B, int Hq, int Hkv, int64_t N, int d, int64_t chunk, int P,
                                     int64_t window, int64_t anchor_period, float scale,
                                     int kv_heads_per_group, void* stream);

/*
 * ring_attn_bwd_host -- ring_attn_bwd for inputs and results in HOST memory,
 * with the copies overlapped with the compute, as ring_attn_fwd_host: the
 * KV heads are cut into groups of `kv_heads_per_group` (0 = at most sixteen
 * groups) with their query heads, and each group's q, k, v, out, dout, lse
 * are copied in, its three backward kernels run, and its dq, dk, dv are
 * copied out while the neighbouring groups are copied.  Each group is
 * computed exactly as ring_attn_bwd computes those heads.
 *
 * Pointers: HOST memory with the layouts of ring_attn_bwd, owned by the
 * caller, kept allocated and unmodified until `stream` has been
 * synchronised; page-locked memory for overlap.  Staging on the device:
 * 2 x (4 B N_q hg d 2 + 4 B N_kv kvg d 2 + B hg N_q 4) bytes plus the
 * backward's own workspace, stream-ordered on `stream`.
 * Returns as ring_attn_bwd; RA_ERR_INVALID_ARG also when kv_heads_per_group
 * does not divide Hkv.
 */
int ring_attn_bwd_host(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d, int causal,
                       int64_t cache_idx, float scale, int kv_heads_per_group, void* stream);

/*
 * ring_attn_bwd_block_step -- the backward of one ring visit: adds, in
 * place, the share of dq, dk, dv that comes from the pairs of query chunk
 * q_chunk [B, Lq, Hq, d] (global positions q_off + t) and KV chunk
 * k_chunk / v_chunk [B, Lk, Hkv, d] (positions k_off + j).  With the query
 * rows' final lse (over the whole sequence, as ring_attn_finalize or
 * ring_attn_fwd return it) and D_t = dout_t . out_t:
 *     p_tj = exp(scale q_t . k_j - lse_t)       on visible pairs, else 0
 *     ds_tj = p_tj (dout_t . v_j - D_t)
 *     dq_acc_t += scale sum_j ds_tj k_j
 *     dk_acc_j += scale sum_t ds_tj q_t,   dv_acc_j += sum_t p_tj dout_t
 * (dk, dv summed over a GQA group's heads).  Summed over every visit of a
 * ring this is ring_attn_bwd's result: the gradient of the Ring Attention
 * page's blockwise loop (§3.1), whose dk / dv travel with their KV chunk.
 * q/k/v/out/dout chunks bf16 (out_chunk and dout_chunk [B, Lq, Hq, d]);
 * lse_chunk [B, Hq, Lq] float32; dq_acc [B, Lq, Hq, d] and dk_acc / dv_acc
 * [B, Lk, Hkv, d] float32, read and written (start them at zero).  All
 * device pointers owned by the caller; tensors 16-byte aligned.  A stream-
 * ordered workspace of 2 * B * Hq * ceil(Lq / 128) * 128 floats is
 * allocated and freed on `stream`.  Returns RA_OK, RA_ERR_INVALID_ARG,
 * RA_ERR_UNSUPPORTED, RA_ERR_CUDA or RA_ERR_OOM.
 */
int ring_attn_bwd_block_step(const void* q_chunk, const void* k_chunk, const void* v_chunk,
                             const void* out_chunk, const void* dout_chunk, const float* lse_chunk,
                             int64_t q_off, int64_t k_off, float* dq_acc, float* dk_acc, float* dv_acc,
                             int B, int Hq, int Hkv, int64_t Lq, int64_t Lk, int d,
                             int causal, float scale, void* stream);

/*
 * ring_attn_fwd_noalloc -- ring_attn_fwd for incremental queries
 * (cache_idx >= 0) that allocates no device memory.  The pages have no
 * counterpart; this exists for callers that cannot let a library allocate:
 * serving stacks whose own pool owns all device memory, and latency-critical
 * loops where an allocation could fail, fragment that budget or stall.
 * Same arguments, layouts and result as ring_attn_fwd.  The split-KV
 * partials go to a fixed 16 MiB device array inside the library instead of a
 * workspace:
 *   - every GPU that loads the library holds those 16 MiB until the process
 *     exits;
 *   - a call whose partials need more than 16 MiB (about
 *     S * B * N_q * Hq * (d + 1) * 4 bytes, S chosen as in ring_attn_fwd) is
 *     rejected with RA_ERR_INVALID_ARG and a message in
 *     ring_attn_last_error(); cache_idx == -1 is rejected the same way;
 *   - the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture;
 *   - the looked-up address is kept for the life of the process, so a
 *     device reset (cudaDeviceReset) after the first call on that device is
 *     not supported;
 *   - all calls share the one array and it keeps the last call's contents:
 *     calls that may overlap on the GPU (different streams, or different
 *     host threads on the same device) race and must be serialised by the
 *     caller;
 *   - when ring_attn_sync_status() reports RA_ERR_DEVICE_TIMEOUT for the
 *     stream, out and lse of the calls before it are undefined: a split
 *     that gave up writes no partial, and the merge may then read the
 *     previous call's partials from the shared array.
 */
int ring_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                          int B, int Hq, int Hkv, int64_t N_q, int64_t N_kv, int d,
                          int causal, int64_t chunk, int P, int64_t cache_idx, float scale,
                          void* stream);

/*
 * ring_attn_add_and_clear -- acc[i] += part[i], then part[i] = 0, for n
 * float32 elements: folds one ring visit's dk / dv share, computed by
 * ring_attn_bwd_block_step into a zeroed buffer `part`, into the
 * accumulators that travel the ring with their KV chunk (the Ring Attention
 * page's blockwise loop, §3.1, whose KV moves while the current block is
 * computed, §3.2).  Computing the share into `part` lets a visit run while
 * the accumulators it will add into are still in flight; the clear leaves
 * `part` ready for the next visit.  acc and part: distinct device buffers
 * owned by the caller, 4-byte aligned (16-byte alignment of both takes the
 * vector path).  n = 0 is a no-op.  Returns RA_OK, RA_ERR_INVALID_ARG
 * (null or equal pointers, n < 0, misalignment), RA_ERR_UNSUPPORTED or
 * RA_ERR_CUDA.
 */
int ring_attn_add_and_clear(float* acc, float* part, int64_t n, void* stream);

/*
 * ring_attn_sync_status -- synchronise `stream`, then read and clear the
 * device status word that kernels set when a bounded wait expires.  Returns
 * RA_OK, RA_ERR_DEVICE_TIMEOUT or RA_ERR_CUDA.
 */
int ring_attn_sync_status(void* stream);

/*
 * ring_attn_exp2_poly -- y[i] = 2^x[i] on FMA units instead of the
 * special-function unit, the polynomial exp2 the bf16 forward can use for a
 * compile-time share of its softmax exponentials (none by default, since
 * every share measured was slower): x = n + f (n = round(x)), 2^f by a degree-3
 * minimax polynomial on [-1/2, 1/2] (max relative error 7.5e-5), 2^n by an
 * exponent-field add; inputs below -125 are clamped to -125.  Valid for
 * x <= 127.  Exposed so the polynomial can be checked against the
 * hardware exp2.  x, y: n floats of device memory.
 */
int ring_attn_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* Static description of a status code. Never NULL. */
const char* ring_attn_error_string(int status);

/* Text of the most recent CUDA failure seen by this thread ("" if none). */
const char* ring_attn_last_error(void);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int ring_attn_version(void);

/* Number of CUDA kernels this process has launched through the library
 * (all devices, all threads).  Diagnostic: lets a caller count the launches
 * inside a timed region. */
int64_t ring_attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* RING_ATTN_H_ */
