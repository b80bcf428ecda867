/*
 * sconv_kv.h -- C ABI of the B200 (sm_100a) fused ShortConv K/V step.
 *
 * The step (Inkling architecture; "SGLang and Miles announce day-0 Inkling
 * support", aib.vote English news item, paragraphs 1-2; "Inkling" model
 * article on axbrief.com, SConv section):
 *
 *   for every token t of sequence i, separately for K and for V:
 *     y[t,c]   = sum_{j=0}^{W-1} w[j,c] * x[t-W+1+j, c]       causal depthwise
 *                (rows before the sequence's first token come from the
 *                 sequence's conv_state, oldest first; w[W-1] meets the
 *                 current token)
 *     z[t,h,d] = y[t,h,d] * gamma[d] / sqrt(mean_d y[t,h,:]^2 + eps)
 *                (RMSNorm over head_dim; the pages only say "normalization",
 *                 RMSNorm with a learned gamma shared by all heads is the
 *                 stated reading)
 *     cache[slot_mapping[t], h, d] = bf16_rne(z[t,h,d])   (skipped if slot < 0)
 *   and the sequence's conv_state becomes the last W-1 raw input rows of
 *   (old state ++ the sequence's rows), so the window carries across chunks
 *   and decode steps (per-request "Mamba/sconv" state pool: Inkling-Small
 *   SGLang cookbook, section 2 memory-pool paragraph and section 3.5).
 *
 * All of it -- conv, norm, cache write, state update -- happens in ONE
 * kernel pass over HBM.  Arithmetic is fp32 with one rounding to bf16 at the
 * cache store; state rows are bit copies.
 *
 * Conventions for every entry point:
 *   - tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates nothing, keeps no state between calls and never synchronises;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream); work is enqueued on it and the call returns at once;
 *   - bf16 tensors are raw 16-bit storage (`void*`); element strides are in
 *     elements, not bytes;
 *   - the return value is SCONV_KV_OK or a negative SCONV_KV_ERR_* code; on
 *     error nothing has been enqueued;
 *   - problems only visible on the device (a slot beyond the cache, a state
 *     index beyond the pool, an inconsistent cu_seqlens) never trap: the
 *     offending token or sequence is skipped and the matching
 *     SCONV_KV_FLAG_* bit is OR-ed into *err_flag (if err_flag is not NULL);
 *     the caller clears *err_flag and reads it after synchronising.
 *
 * Cache behaviour: the fused kernels read each k/v row (and, in decode,
 * each old conv_state row) exactly once and load them with an L2
 * evict-first policy, so later kernels find the cache rows just written
 * in L2 rather than these inputs.
 *
 * Preconditions the library cannot check without synchronising (results are
 * unspecified when they are violated): non-negative slots are unique within
 * a call; state indices are unique within a call; k/v do not alias the
 * caches or the state; calls that touch the same conv_state or cache rows
 * are ordered on one stream.
 */
#ifndef SCONV_KV_H_
#define SCONV_KV_H_

#include <stdint.h>

#if defined(__GNUC__)
#define SCONV_KV_API __attribute__((visibility("default")))
#else
#define SCONV_KV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
#define SCONV_KV_OK 0
#define SCONV_KV_ERR_NULL (-1)        /* a required pointer is NULL          */
#define SCONV_KV_ERR_SHAPE (-2)       /* W, head_dim, heads, counts, strides  */
#define SCONV_KV_ERR_ALIGN (-3)       /* pointer or stride not 16-byte aligned */
#define SCONV_KV_ERR_UNSUPPORTED (-4) /* valid but not implemented combination */
#define SCONV_KV_ERR_CUDA (-5)        /* CUDA reported an error at launch     */
#define SCONV_KV_ERR_SCRATCH (-6)     /* call needs more than the static scratch */

/* ---------------------------------------------------- device-side flag bits */
#define SCONV_KV_FLAG_SLOT_RANGE 1   /* slot >= num_pages*page_size: skipped  */
#define SCONV_KV_FLAG_STATE_INDEX 2  /* state index outside the pool: sequence
                                        skipped (no cache write, no state)   */
#define SCONV_KV_FLAG_CU_SEQLENS 4   /* cu_seqlens not a partition of
                                        [0, num_tokens): bad sequences skipped */
#define SCONV_KV_FLAG_TIMEOUT 8      /* an internal pipeline wait gave up after
                                        its time limit (about 1 s): the CTA
                                        stopped early, output incomplete      */

/* ------------------------------------------------------------- limits */
#define SCONV_KV_MAX_W 8             /* conv width W in [1, SCONV_KV_MAX_W]   */

/*
 * Paged KV cache layout.  Element (slot, h, d) of k_cache (and of v_cache)
 * lives at
 *     (slot / page_size) * stride_page + (slot % page_size) * stride_slot
 *       + h * stride_head + d
 * elements from the cache base pointer (dim stride 1).  A cache is
 * num_pages * page_size slots; pages are handed to sequences by the caller
 * ("prefix pages" of the serving runtime's radix cache, Inkling-Small
 * cookbook section 3.5), so slot_mapping is an arbitrary scatter.
 */
typedef struct sconv_kv_cache_layout_t {
  int64_t num_pages;
  int64_t page_size;
  int64_t num_kv_heads;
  int64_t head_dim;
  int64_t stride_page;     /* elements */
  int64_t stride_slot;     /* elements */
  int64_t stride_head;     /* elements */
  int64_t bytes_per_cache; /* bytes spanned by ONE cache (k or v) */
} sconv_kv_cache_layout_t;

/*
 * Fill *out with the dense layout [num_pages, page_size, num_kv_heads,
 * head_dim] (stride_head = head_dim, stride_slot = num_kv_heads*head_dim,
 * stride_page = page_size*stride_slot).  Callers with another layout (e.g.
 * K and V interleaved per page) fill the struct themselves.
 * Host-only; touches no GPU.  Errors: SCONV_KV_ERR_NULL (out == NULL),
 * SCONV_KV_ERR_SHAPE (a count < 0, page_size < 1, heads < 1, head_dim < 1).
 */
SCONV_KV_API int sconv_kv_cache_layout(int64_t num_pages, int64_t page_size,
                          int num_kv_heads, int head_dim,
                          sconv_kv_cache_layout_t* out);

/*
 * Fused ShortConv K/V step over a packed varlen batch (prefill or chunked
 * prefill; sequences are packed back to back as in flash-attention's varlen
 * interface).
 *
 *  k, v           bf16, token t's row at k + t*row_stride: Hkv*D channels
 *                 (head-major, then head_dim).  row_stride >= Hkv*D, a
 *                 multiple of 8 elements; lets k and v be column slices of
 *                 a fused qkv projection output.  16-byte aligned.
 *  num_tokens     T, rows of k/v and entries of slot_mapping (>= 0).
 *  cu_seqlens     int32 [num_seqs+1] on the device: cu[0]=0, non-decreasing,
 *                 cu[num_seqs]=T.  Sequence i is rows [cu[i], cu[i+1]).
 *  num_seqs       S >= 0.
 *  conv_w_k/v     bf16 [W, Hkv*D] taps, row j = tap j (j = W-1 meets the
 *                 current token).  16-byte aligned.
 *  gamma_k/v      fp32 [head_dim], shared by all heads.  16-byte aligned.
 *  eps            RMSNorm epsilon (inside the square root).
 *  W              conv width, 1..SCONV_KV_MAX_W.
 *  num_kv_heads   Hkv >= 1.
 *  head_dim       D in {64, 128, 256}.
 *  conv_state     bf16 [state_pool_size, W-1, 2*Hkv*D], in/out: raw input
 *                 rows, oldest first, K channels then V channels.  May be
 *                 NULL only when W == 1.  16-byte aligned.  New sequences
 *                 must start from zeroed rows (the caller zeroes them).
 *  state_indices  int32 [num_seqs] on the device: pool row of sequence i;
 *                 NULL means sequence i uses pool row i.
 *  state_pool_size rows in the pool (bounds for state_indices).
 *  slot_mapping   int64 [T] on the device: cache slot of each token; < 0
 *                 means "do not write" (padding).
 *  k_cache, v_cache  bf16 caches described by *layout (host pointer to the
 *                 struct).  16-byte aligned; stride_head, stride_slot and
 *                 stride_page multiples of 8 elements; the element offset
 *                 of the last slot's row, (num_pages-1)*stride_page +
 *                 (page_size-1)*stride_slot, below 8 * (2^32 - 1) (about
 *                 34 G elements; SCONV_KV_ERR_SHAPE otherwise).
 *  err_flag       optional device int; SCONV_KV_FLAG_* bits are OR-ed in.
 *  stream         cudaStream_t as void*.
 *
 * Errors: SCONV_KV_ERR_NULL, _SHAPE, _ALIGN, _UNSUPPORTED, _CUDA as above.
 * A call with T == 0 or S == 0 enqueues nothing and returns SCONV_KV_OK
 * without examining the pointers (empty tensors may have NULL data).
 */
SCONV_KV_API int sconv_kv_prefill_varlen(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream);

/*
 * Decode specialisation: exactly one new token per sequence (batch
 * sequences; token b belongs to sequence b, as if cu_seqlens = 0..batch).
 * Arguments mean what they mean for sconv_kv_prefill_varlen; k and v are
 * [batch] rows of Hkv*D channels at row_stride.  The sequence's state is
 * read, the new row is convolved with it, normalised, written to
 * cache[slot_mapping[b]] and the state is shifted by one row in place.
 * A call with batch == 0 enqueues nothing and returns SCONV_KV_OK without
 * examining the pointers.
 */
SCONV_KV_API int sconv_kv_decode(
    const void* k, const void* v, int64_t row_stride, int batch,
    const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
    const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
    void* conv_state, const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream);

/*
 * MXFP8 cache store ("Inkling-Small" SGLang cookbook, section 3.6 Long
 * Context: KV entries stored as block-scaled MXFP8 instead of BF16, about
 * twice the tokens per pool).  The page gives no block size or scale
 * format; this follows the OCP Microscaling (MX) format:
 *   - each head's D channels form D/32 blocks of 32 consecutive channels;
 *   - a block stores one E8M0 scale byte s + 127, X = 2^s with
 *     s = floor(log2(max |z| over the block)) - 8 (8 = exponent of E4M3's
 *     largest normal, 448 = 1.75 * 2^8), s = -127 for an all-zero or
 *     subnormal block;
 *   - each element stores the FP8 E4M3 code of z / X, rounded to nearest
 *     even, magnitudes beyond 448 saturated to 448;
 *   - z is the normalised value of the bf16 entry points, in binary32; the
 *     rounding decisions are taken on it.
 *
 * Arguments are those of sconv_kv_prefill_varlen / sconv_kv_decode, except
 * the caches:
 *   k_data, v_data    uint8 E4M3 codes; element (slot, h, d) at the element
 *                     offset given by *layout (1 byte per element).
 *                     16-byte aligned.
 *   k_scale, v_scale  uint8 E8M0 scales; block (slot, h, b) at
 *                     (page*stride_page + off*stride_slot + h*stride_head)/32
 *                     + b.  The layout's strides must be multiples of 32.
 * Errors and flags as for the bf16 entry points (SCONV_KV_ERR_ALIGN also
 * when a stride is not a multiple of 32).
 */
SCONV_KV_API int sconv_kv_prefill_varlen_mxfp8(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_data, uint8_t* k_scale, void* v_data,
    uint8_t* v_scale, const sconv_kv_cache_layout_t* layout, int* err_flag,
    void* stream);

SCONV_KV_API int sconv_kv_decode_mxfp8(
    const void* k, const void* v, int64_t row_stride, int batch,
    const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
    const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
    void* conv_state, const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_data, uint8_t* k_scale, void* v_data,
    uint8_t* v_scale, const sconv_kv_cache_layout_t* layout, int* err_flag,
    void* stream);

/*
 * Layout variants (the _ex entry points; NULL options = the defaults of the
 * entry points above).
 *
 *  gamma_head_stride  elements between consecutive heads' gammas: 0 (the
 *                     default) = gamma_k/v are [head_dim], shared by every
 *                     head; head_dim = per-head gammas [num_kv_heads,
 *                     head_dim].  Other values: SCONV_KV_ERR_SHAPE.
 *  state_positions    NULL (default): conv_state holds each sequence's last
 *                     W-1 raw rows oldest first, all rewritten by every
 *                     call.  Otherwise device int64 [num_seqs] (decode:
 *                     [batch]), the number of tokens sequence i has seen
 *                     before this call, and conv_state is a ring: the raw
 *                     row of position p lives in row p mod (W-1).  A call
 *                     then writes only the rows of its sequence's last
 *                     min(L, W-1) positions (one row per decode step instead
 *                     of W-1); a new sequence starts at position 0 with
 *                     zeroed rows, as in the linear layout.  A negative
 *                     position skips the sequence and sets
 *                     SCONV_KV_FLAG_STATE_INDEX.
 *
 *  wait_timeout_ns    longest time a pipeline wait inside the kernels may
 *                     take before the kernel gives up, lets the copies it
 *                     has issued land, sets SCONV_KV_FLAG_TIMEOUT and
 *                     returns with its output incomplete (<= 0: 1 s).  A
 *                     short limit exercises that path without any fault.
 *  withhold_first_copy  testing only (0 in normal use): nonzero makes every
 *                     CTA skip the copy of its first chunk (decode: of its
 *                     first sequence), so the waits on it run out after
 *                     wait_timeout_ns and the timeout path above runs: a
 *                     wait on something that nothing completes, with no
 *                     fault.  The output of such a call is incomplete.
 *  state_only_dependency  prefill only (decode ignores it).  Nonzero is a
 *                     promise by the caller: the kernel enqueued just
 *                     before this call on `stream` writes none of this
 *                     call's inputs except conv_state, and none of the
 *                     cache slots this call writes -- as when consecutive
 *                     chunks of one long sequence are prefilled back to
 *                     back (1M-token context: aib.vote English news item,
 *                     paragraph 1; Inkling-Small cookbook, section 3.6).
 *                     The call's CTAs are launched early (programmatic
 *                     dependent launch) as usual, but only a CTA that
 *                     reads or writes a conv_state row waits for that
 *                     previous kernel to complete before it does so; every
 *                     other CTA streams its rows and writes its cache slots
 *                     at once, overlapping the previous kernel's tail.
 *                     Every CTA still waits for the previous kernel before
 *                     it lets the next one launch and before it exits, so
 *                     ordering along the stream is kept.  0 (default): every
 *                     CTA waits before its first global access.  Inputs
 *                     produced by the previous kernel (e.g. a projection
 *                     launched right before this call) break the promise:
 *                     leave it 0 then.
 *  independent_state  decode only (prefill ignores it).  Nonzero is a
 *                     promise by the caller: the kernel enqueued just
 *                     before this call on `stream` writes none of this
 *                     call's inputs except k and v -- as when that kernel is
 *                     the K/V projection of this very decode step -- and
 *                     neither reads nor writes the conv_state rows or cache
 *                     slots this call writes.  Each CTA then reads its
 *                     index tables and requests its first sequence's W-1
 *                     state rows before it waits for that kernel
 *                     (programmatic dependent launch); only the K/V rows
 *                     wait.  Every CTA waits before anything is written,
 *                     before the next kernel may launch and before it
 *                     exits.  0 (default): every CTA waits before its first
 *                     global access.
 *
 * The pages fix neither of the two layouts (their norm is only
 * "normalization" and the state pool's layout is not given); both are
 * layouts a serving runtime may use.
 */
typedef struct sconv_kv_options_t {
  int64_t gamma_head_stride;
  const int64_t* state_positions;
  int64_t wait_timeout_ns;
  int64_t withhold_first_copy;
  int64_t state_only_dependency;
  int64_t independent_state;
} sconv_kv_options_t;

SCONV_KV_API int sconv_kv_prefill_varlen_ex(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, const sconv_kv_options_t* options,
    int* err_flag, void* stream);

SCONV_KV_API int sconv_kv_decode_ex(
    const void* k, const void* v, int64_t row_stride, int batch,
    const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
    const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
    void* conv_state, const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, const sconv_kv_options_t* options,
    int* err_flag, void* stream);

SCONV_KV_API int sconv_kv_prefill_varlen_mxfp8_ex(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_data, uint8_t* k_scale, void* v_data,
    uint8_t* v_scale, const sconv_kv_cache_layout_t* layout,
    const sconv_kv_options_t* options, int* err_flag, void* stream);

SCONV_KV_API int sconv_kv_decode_mxfp8_ex(
    const void* k, const void* v, int64_t row_stride, int batch,
    const void* conv_w_k, const void* conv_w_v, const float* gamma_k,
    const float* gamma_v, float eps, int W, int num_kv_heads, int head_dim,
    void* conv_state, const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_data, uint8_t* k_scale, void* v_data,
    uint8_t* v_scale, const sconv_kv_cache_layout_t* layout,
    const sconv_kv_options_t* options, int* err_flag, void* stream);

/*
 * Unfused stages.  The same step as four separate passes over HBM, each
 * with its intermediate in bf16: the chain that the fused entry points
 * replace ("SGLang and Miles announce day-0 Inkling support", aib.vote
 * English news item, paragraph 2: K/V conv, normalisation and KV-cache
 * write fused, against an unfused chain).  Run in order on one stream:
 *
 *   sconv_kv_stage_conv          k, v, old state  -> y
 *   sconv_kv_stage_rmsnorm       y                -> z
 *   sconv_kv_stage_scatter       z, slot_mapping  -> k_cache, v_cache
 *   sconv_kv_stage_state_update  k, v, old state  -> new state
 *
 * the result equals the fused step's except that y is rounded to bf16
 * before the normalisation.  Each stage is also usable alone.
 *
 * Intermediates y and z: bf16 [num_tokens, 2*num_kv_heads*head_dim]
 * (K channels, then V), device memory owned by the caller, 16-byte
 * aligned.  Other arguments mean what they mean for
 * sconv_kv_prefill_varlen, with the same layouts, alignment rules and
 * flag bits.  Calls with num_tokens == 0 (or num_seqs == 0) enqueue nothing
 * and succeed without looking at the pointers.
 *
 * sconv_kv_stage_conv: y[t] = sum_j w[j] * x[t-W+1+j] per channel, rows
 *   before a sequence's first token taken from its conv_state (read only).
 *   A bad state index or a malformed cu_seqlens skips the token (y not
 *   written) and sets the flag bit.
 * sconv_kv_stage_rmsnorm: z = y / sqrt(mean over the head of y^2 + eps) *
 *   gamma[d] per (token, head), rounded to bf16.
 * sconv_kv_stage_scatter: cache[slot_mapping[t]] = z[t] (K half into
 *   k_cache, V half into v_cache); slot < 0 skips the token; a slot past
 *   the cache is skipped and flagged.  cu_seqlens (with num_seqs >= 1, W
 *   and the state pool as given to the other stages) is optional: when it
 *   is not NULL, the tokens of a sequence that the other stages skip (a
 *   malformed cu_seqlens entry, or for W > 1 a state index outside the
 *   pool) are not written either, so the chain leaves the same cache slots
 *   untouched as the fused step; when it is NULL every token is written.
 * sconv_kv_stage_state_update: each sequence's state = the last W-1 raw
 *   rows of (old state ++ its rows), in place; must run after every reader
 *   of the old state (sconv_kv_stage_conv).  W == 1 has no state: no-op.
 */
SCONV_KV_API int sconv_kv_stage_conv(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, int W, int num_kv_heads, int head_dim,
    const void* conv_state, const int32_t* state_indices,
    int64_t state_pool_size, void* y, int* err_flag, void* stream);

SCONV_KV_API int sconv_kv_stage_rmsnorm(
    const void* y, int64_t num_tokens, const float* gamma_k,
    const float* gamma_v, float eps, int num_kv_heads, int head_dim, void* z,
    void* stream);

SCONV_KV_API int sconv_kv_stage_scatter(
    const void* z, int64_t num_tokens, int num_kv_heads, int head_dim,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, const int32_t* cu_seqlens,
    int num_seqs, int W, const int32_t* state_indices,
    int64_t state_pool_size, int* err_flag, void* stream);

SCONV_KV_API int sconv_kv_stage_state_update(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, int W, int num_kv_heads,
    int head_dim, void* conv_state, const int32_t* state_indices,
    int64_t state_pool_size, int* err_flag, void* stream);

/*
 * The unfused chain in one call, with no allocation: the same four stages
 * (conv, rmsnorm, scatter, state update, in that order on `stream`), their
 * bf16 intermediates y and z placed in a scratch buffer that the library
 * holds in static device memory (SCONV_KV_NOALLOC_SCRATCH_BYTES per device,
 * reserved when the library's module loads; every call looks up its
 * address in the current context, a host-side lookup that allocates
 * nothing).  The library allocates nothing on any call.
 *
 * Arguments and results as for sconv_kv_prefill_varlen (bf16 caches), and
 * the results equal those of the four sconv_kv_stage_* calls (scatter given
 * cu_seqlens, so a skipped sequence leaves its cache slots untouched).
 * Every argument of all four stages is checked before the first launch:
 * an argument error returns with nothing enqueued.  Only a CUDA launch
 * failure (SCONV_KV_ERR_CUDA) can come after earlier stages were enqueued.
 * The call needs 2 * round_up_256(num_tokens * 2 * num_kv_heads * head_dim
 * * 2) bytes of scratch; a larger call returns SCONV_KV_ERR_SCRATCH before
 * enqueueing anything.  Calls share the one scratch buffer, which keeps
 * whatever the last call left in it: calls that overlap on the GPU race,
 * so they must be ordered (one stream, or streams ordered by events).
 *
 * The source pages have no counterpart to this entry point: it is a
 * convenience of this library.
 */
#define SCONV_KV_NOALLOC_SCRATCH_BYTES (64ll << 20)

SCONV_KV_API int sconv_kv_unfused_step_noalloc(
    const void* k, const void* v, int64_t row_stride, int64_t num_tokens,
    const int32_t* cu_seqlens, int num_seqs, const void* conv_w_k,
    const void* conv_w_v, const float* gamma_k, const float* gamma_v,
    float eps, int W, int num_kv_heads, int head_dim, void* conv_state,
    const int32_t* state_indices, int64_t state_pool_size,
    const int64_t* slot_mapping, void* k_cache, void* v_cache,
    const sconv_kv_cache_layout_t* layout, int* err_flag, void* stream);

/* Static text for a status code (never NULL). */
SCONV_KV_API const char* sconv_kv_strerror(int status);

/* Text of the last CUDA error seen by an entry point on this host thread
 * ("" if none).  Valid until the next call on the same thread. */
SCONV_KV_API const char* sconv_kv_last_cuda_error(void);

/* Library version as major*10000 + minor*100 + patch. */
SCONV_KV_API int sconv_kv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SCONV_KV_H_ */
