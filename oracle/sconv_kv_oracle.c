/*
 * Oracle for the fused ShortConv K/V step -- TEST INFRASTRUCTURE ONLY.
 *
 * This file is the plain, slow, obviously-correct CPU statement of what the
 * fused ShortConv K/V step computes.  It exists so that the CUDA path can be
 * checked against something written straight from the method's definition.
 * Only the test suite, the package's smoke check and the benchmark's CPU
 * baseline leg may load it; the product path never does.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Sources (web pages about the Inkling architecture):
 *  - "SGLang and Miles announce day-0 Inkling support" (aib.vote, English
 *    news item), paragraph 1: ShortConv is a causal convolution over the
 *    token dimension.
 *  - same item, paragraph 2: the fused ShortConv kernel does the K/V
 *    convolution, then the normalisation, then the KV-cache write, in that
 *    order, in one kernel.
 *  - "Inkling: 1-trillion-parameter multimodal model with 1M context"
 *    (axbrief.com), section "SConv, MoE and per-modality embedding towers":
 *    SConv reads the current token and the previous W-1 hidden states,
 *    W being the window size.
 *  - "Inkling-Small" SGLang cookbook (data-sketchers.com), section 2
 *    "configuration tips", memory-pool paragraph, and section 3.5 (HiCache):
 *    the conv ("Mamba/sconv") state of each request lives in a state pool
 *    and is carried between calls.
 *
 * Readings taken where the pages are silent (the pages give no formula):
 *  - the normalisation is RMSNorm over head_dim with a learned gamma[D]
 *    shared by all heads, eps inside the square root, no mean subtraction;
 *  - tap w[W-1] multiplies the current token, w[0] the oldest one; no bias,
 *    no activation; K and V each have their own taps, depthwise over the
 *    C = Hkv*D channels;
 *  - conv_state holds the last W-1 raw (pre-conv) bf16 input rows of a
 *    sequence, oldest first, K channels [0,C) then V channels [C,2C);
 *  - a negative slot means "do not write this token";
 *  - all arithmetic is in double precision; the cache receives one
 *    round-to-nearest-even rounding to bf16 of the normalised value.
 *
 * Every function below performs one step of the method with plain loops and
 * no blocking, fusion or reordering.  Index conventions:
 *   x rows:        x[row * row_stride + c],            c in [0, C)
 *   state rows:    s[r * state_row_stride + c],         r in [0, W-1)
 *   cache element: base + page*stride_page + off*stride_slot
 *                       + h*stride_head + d,
 *                  page = slot / page_size, off = slot % page_size.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_SLOT_RANGE -2
#define ORACLE_ERR_SLOT_DUP -3
#define ORACLE_ERR_STATE_INDEX -4
#define ORACLE_ERR_CU_SEQLENS -5
#define ORACLE_ERR_NOMEM -6

/* bf16 is the top half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits, exponent range of
 * binary32), ties to even, in one rounding step.  rint() rounds to nearest
 * even under the default rounding mode. */
uint16_t oracle_double_to_bf16(double x) {
  if (isnan(x)) return (uint16_t)0x7FC0;
  double ax = fabs(x);
  double r;
  if (ax == 0.0) {
    r = x; /* keeps the sign of zero */
  } else {
    int e;
    frexp(ax, &e); /* ax = m * 2^e, m in [0.5, 1) */
    /* quantum of the bf16 grid around ax: 2^(e-8) for normal numbers,
     * 2^-133 below the smallest normal 2^-126 */
    int q = e - 8;
    if (q < -133) q = -133;
    r = ldexp(rint(ldexp(ax, -q)), q);
    /* largest finite bf16 is (2 - 2^-7) * 2^127; anything that rounds
     * beyond it is infinity */
    if (r > ldexp(255.0, 120)) r = INFINITY;
    if (x < 0) r = -r;
  }
  float f = (float)r; /* exact: r is on the bf16 grid */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/*
 * Step a1+a2: window assembly and causal depthwise convolution of ONE
 * sequence of ONE tensor (K or V).
 *   y[p][c] = sum_{j=0}^{W-1} w[j][c] * xrow(p-W+1+j)[c]
 * where xrow(q) = x[q] for q >= 0 and the old state row s[W-1+q] for q < 0.
 * (Causal conv over tokens: aib.vote news item, paragraph 1; current token
 * plus the previous W-1 states: axbrief.com SConv section.)
 * The sum runs over j in increasing order.
 */
void oracle_conv(const uint16_t* x, int64_t row_stride, int64_t L,
                 const uint16_t* s, int64_t state_row_stride,
                 const uint16_t* w, int W, int C, double* y) {
  for (int64_t p = 0; p < L; ++p) {
    for (int c = 0; c < C; ++c) {
      double acc = 0.0;
      for (int j = 0; j < W; ++j) {
        int64_t q = p - (W - 1) + j;
        uint16_t xv = (q >= 0) ? x[q * row_stride + c]
                               : s[(W - 1 + q) * state_row_stride + c];
        acc += oracle_bf16_to_double(w[(int64_t)j * C + c]) *
               oracle_bf16_to_double(xv);
      }
      y[p * C + c] = acc;
    }
  }
}

/*
 * Step a3: RMSNorm of every (token, head) over head_dim with gamma[D]
 * shared by all heads (the pages only say "normalization"; this reading is
 * the stated assumption).
 *   r = 1 / sqrt( (sum_d y[d]^2) / D + eps ),   z[d] = (y[d] * r) * gamma[d]
 */
void oracle_rmsnorm_strided(const double* y, int64_t L, int num_heads, int D,
                            const float* gamma, int64_t gamma_head_stride, double eps,
                            double* z) {
  for (int64_t p = 0; p < L; ++p) {
    for (int h = 0; h < num_heads; ++h) {
      const double* yh = y + (p * num_heads + h) * (int64_t)D;
      const float* gh = gamma + (int64_t)h * gamma_head_stride;
      double ss = 0.0;
      for (int d = 0; d < D; ++d) ss += yh[d] * yh[d];
      double r = 1.0 / sqrt(ss / (double)D + eps);
      double* zh = z + (p * num_heads + h) * (int64_t)D;
      for (int d = 0; d < D; ++d) zh[d] = (yh[d] * r) * (double)gh[d];
    }
  }
}

/* gamma shared by all heads (gamma_head_stride 0) */
void oracle_rmsnorm(const double* y, int64_t L, int num_heads, int D,
                    const float* gamma, double eps, double* z) {
  oracle_rmsnorm_strided(y, L, num_heads, D, gamma, 0, eps, z);
}

/* Address (in elements) of slot `slot`, head h, dim 0 of a paged cache. */
static int64_t cache_offset(int64_t slot, int h, int64_t page_size,
                            int64_t stride_page, int64_t stride_slot,
                            int64_t stride_head) {
  int64_t page = slot / page_size;
  int64_t off = slot % page_size;
  return page * stride_page + off * stride_slot + (int64_t)h * stride_head;
}

/*
 * Step a4: round to bf16 and write token p's normalised row to
 * cache[slots[p]]; a negative slot is skipped.  Out-of-range slots are an
 * error (nothing is written for them, the error is reported).
 * (KV-cache write inside the fused step: aib.vote news item, paragraph 2.)
 */
int oracle_scatter(const double* z, int64_t L, int num_heads, int D,
                   const int64_t* slots, int64_t num_slots, int64_t page_size,
                   int64_t stride_page, int64_t stride_slot,
                   int64_t stride_head, uint16_t* cache) {
  int status = ORACLE_OK;
  for (int64_t p = 0; p < L; ++p) {
    int64_t slot = slots[p];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      status = ORACLE_ERR_SLOT_RANGE;
      continue;
    }
    for (int h = 0; h < num_heads; ++h) {
      int64_t base = cache_offset(slot, h, page_size, stride_page,
                                  stride_slot, stride_head);
      for (int d = 0; d < D; ++d)
        cache[base + d] =
            oracle_double_to_bf16(z[(p * num_heads + h) * (int64_t)D + d]);
    }
  }
  return status;
}

/*
 * Step a5: the new state of one tensor of one sequence is the last W-1 rows
 * of (old state rows ++ the sequence's L input rows), oldest first, copied
 * as raw bf16.  With L = 0 the state is unchanged.
 * (Per-request conv state carried in a pool: Inkling-Small cookbook,
 * section 2 memory-pool paragraph and section 3.5.)
 */
void oracle_state_update(const uint16_t* x, int64_t row_stride, int64_t L,
                         uint16_t* s, int64_t state_row_stride, int C, int W) {
  int n = W - 1;
  if (n <= 0 || L == 0) return;
  /* copy the old rows first so the update reads only old values */
  uint16_t* old = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n * (size_t)C);
  if (!old) return;
  for (int r = 0; r < n; ++r)
    for (int c = 0; c < C; ++c) old[r * C + c] = s[r * state_row_stride + c];
  for (int j = 0; j < n; ++j) {
    /* combined index: old rows are -n..-1, new rows 0..L-1 */
    int64_t q = L - n + j;
    for (int c = 0; c < C; ++c)
      s[j * state_row_stride + c] =
          (q >= 0) ? x[q * row_stride + c] : old[(n + q) * C + c];
  }
  free(old);
}

/*
 * Step a5 with a ring-buffer state (a layout variant): the raw input row of
 * position p of the sequence lives in state row p mod (W-1).  The sequence
 * has seen pos0 tokens before this call, so its L new rows are positions
 * pos0 .. pos0+L-1; the rows of the last min(L, W-1) of them are written,
 * every other state row keeps its value (it still holds one of the last W-1
 * positions).
 */
void oracle_state_update_ring(const uint16_t* x, int64_t row_stride, int64_t L,
                              uint16_t* s, int64_t state_row_stride, int C, int W,
                              int64_t pos0) {
  const int64_t n = W - 1;
  if (n <= 0) return;
  const int64_t first = L > n ? L - n : 0;
  for (int64_t q = first; q < L; ++q) {
    const int64_t row = (pos0 + q) % n;
    for (int c = 0; c < C; ++c) s[row * state_row_stride + c] = x[q * row_stride + c];
  }
}

/* The W-1 rows in front of position pos0 (oldest first) from a ring state:
 * position pos0-(W-1)+j sits in row (pos0-(W-1)+j) mod (W-1) = (pos0+j)
 * mod (W-1); rows for positions before 0 are the zero rows a new sequence
 * starts with. */
static void ring_to_linear(const uint16_t* ring, int64_t state_row_stride, int W, int C2,
                           int64_t pos0, uint16_t* lin) {
  const int64_t n = W - 1;
  for (int64_t j = 0; j < n; ++j) {
    const int64_t row = (pos0 + j) % n;
    memcpy(lin + j * C2, ring + row * state_row_stride, sizeof(uint16_t) * (size_t)C2);
  }
}

/*
 * The whole step over a varlen batch: for each sequence i in order, for K
 * then V: conv (a1+a2) -> RMSNorm (a3) -> bf16 scatter (a4) -> state
 * update (a5).  The fused kernel reaches exactly this result; fusion only
 * removes the memory round trips between the steps.
 *
 *  k, v          bf16 [num_tokens rows, row_stride elems], C = Hkv*D used
 *  cu_seqlens    int32 [num_seqs+1], cu[0] = 0, non-decreasing,
 *                cu[num_seqs] = num_tokens
 *  conv_w_k/v    bf16 [W, C]
 *  gamma_k/v     fp32 [D]
 *  conv_state    bf16 [state_pool_size, W-1, 2C] (in/out)
 *  state_indices int32 [num_seqs] or NULL (identity)
 *  slot_mapping  int64 [num_tokens], negative = skip
 *  k/v_cache     bf16, element offsets as in the file header
 *  z_k, z_v      optional double [num_tokens, C]: normalised values before
 *                rounding (rows of skipped slots are filled too)
 * Duplicate non-negative slots are refused (the result would depend on the
 * write order).  Returns ORACLE_OK or a negative ORACLE_ERR_*.
 */
int oracle_prefill_varlen_opts(
    const uint16_t* k, const uint16_t* v, int64_t row_stride,
    int64_t num_tokens, const int32_t* cu_seqlens, int num_seqs,
    const uint16_t* conv_w_k, const uint16_t* conv_w_v, const float* gamma_k,
    const float* gamma_v, int64_t gamma_head_stride, double eps, int W,
    int num_heads, int D, uint16_t* conv_state, const int32_t* state_indices,
    const int64_t* state_positions, int64_t state_pool_size,
    const int64_t* slot_mapping, uint16_t* k_cache,
    uint16_t* v_cache, int64_t num_pages, int64_t page_size,
    int64_t stride_page, int64_t stride_slot, int64_t stride_head,
    double* z_k, double* z_v) {
  if (W < 1 || num_heads < 1 || D < 1 || num_seqs < 0 || num_tokens < 0)
    return ORACLE_ERR_ARG;
  if (gamma_head_stride != 0 && gamma_head_stride != D) return ORACLE_ERR_ARG;
  if (state_positions)
    for (int i = 0; i < num_seqs; ++i)
      if (state_positions[i] < 0) return ORACLE_ERR_ARG;
  const int C = num_heads * D;
  const int64_t num_slots = num_pages * page_size;
  if (row_stride < C) return ORACLE_ERR_ARG;

  /* cu_seqlens must describe a partition of [0, num_tokens) */
  if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != num_tokens)
    return ORACLE_ERR_CU_SEQLENS;
  for (int i = 0; i < num_seqs; ++i)
    if (cu_seqlens[i + 1] < cu_seqlens[i]) return ORACLE_ERR_CU_SEQLENS;

  /* slots: in range and unique */
  if (num_slots > 0) {
    unsigned char* seen = (unsigned char*)calloc((size_t)num_slots, 1);
    if (!seen) return ORACLE_ERR_NOMEM;
    for (int64_t t = 0; t < num_tokens; ++t) {
      int64_t sl = slot_mapping[t];
      if (sl < 0) continue;
      if (sl >= num_slots) {
        free(seen);
        return ORACLE_ERR_SLOT_RANGE;
      }
      if (seen[sl]) {
        free(seen);
        return ORACLE_ERR_SLOT_DUP;
      }
      seen[sl] = 1;
    }
    free(seen);
  } else {
    for (int64_t t = 0; t < num_tokens; ++t)
      if (slot_mapping[t] >= 0) return ORACLE_ERR_SLOT_RANGE;
  }
  for (int i = 0; i < num_seqs; ++i) {
    int64_t si = state_indices ? state_indices[i] : i;
    if (si < 0 || si >= state_pool_size) return ORACLE_ERR_STATE_INDEX;
  }

  const int64_t state_row_stride = 2 * (int64_t)C;
  const int64_t state_seq_stride = (int64_t)(W - 1) * state_row_stride;
  int64_t max_len = 0;
  for (int i = 0; i < num_seqs; ++i) {
    int64_t L = cu_seqlens[i + 1] - cu_seqlens[i];
    if (L > max_len) max_len = L;
  }
  double* y = (double*)malloc(sizeof(double) * (size_t)(max_len ? max_len : 1) *
                              (size_t)C);
  double* z = (double*)malloc(sizeof(double) * (size_t)(max_len ? max_len : 1) *
                              (size_t)C);
  if (!y || !z) {
    free(y);
    free(z);
    return ORACLE_ERR_NOMEM;
  }

  /* a ring state is read through a linear copy of the rows in front of the
     sequence (oldest first) */
  uint16_t* lin = NULL;
  if (state_positions && W > 1) {
    lin = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)state_seq_stride);
    if (!lin) {
      free(y);
      free(z);
      return ORACLE_ERR_NOMEM;
    }
  }

  int status = ORACLE_OK;
  for (int i = 0; i < num_seqs; ++i) {
    const int64_t t0 = cu_seqlens[i];
    const int64_t L = cu_seqlens[i + 1] - t0;
    const int64_t si = state_indices ? state_indices[i] : i;
    uint16_t* st = conv_state ? conv_state + si * state_seq_stride : NULL;
    const int64_t pos0 = state_positions ? state_positions[i] : 0;
    if (lin && st) ring_to_linear(st, state_row_stride, W, 2 * C, pos0, lin);
    for (int which = 0; which < 2; ++which) { /* 0 = K, 1 = V */
      const uint16_t* x = (which == 0 ? k : v) + t0 * row_stride;
      const uint16_t* w = (which == 0 ? conv_w_k : conv_w_v);
      const float* g = (which == 0 ? gamma_k : gamma_v);
      uint16_t* cache = (which == 0 ? k_cache : v_cache);
      uint16_t* s = st ? st + (which == 0 ? 0 : C) : NULL;
      const uint16_t* s_read = (lin && st) ? lin + (which == 0 ? 0 : C) : s;
      double* zout = (which == 0 ? z_k : z_v);

      oracle_conv(x, row_stride, L, s_read, state_row_stride, w, W, C, y);
      oracle_rmsnorm_strided(y, L, num_heads, D, g, gamma_head_stride, eps, z);
      int rc = oracle_scatter(z, L, num_heads, D, slot_mapping + t0,
                              num_slots, page_size, stride_page, stride_slot,
                              stride_head, cache);
      if (rc != ORACLE_OK) status = rc;
      if (s && lin) oracle_state_update_ring(x, row_stride, L, s, state_row_stride, C, W, pos0);
      else if (s) oracle_state_update(x, row_stride, L, s, state_row_stride, C, W);
      if (zout) memcpy(zout + t0 * C, z, sizeof(double) * (size_t)(L * C));
    }
  }
  free(lin);
  free(y);
  free(z);
  return status;
}

/* The step with gamma shared by all heads and a linear (oldest first) state. */
int oracle_prefill_varlen(
    const uint16_t* k, const uint16_t* v, int64_t row_stride,
    int64_t num_tokens, const int32_t* cu_seqlens, int num_seqs,
    const uint16_t* conv_w_k, const uint16_t* conv_w_v, const float* gamma_k,
    const float* gamma_v, double eps, int W, int num_heads, int D,
    uint16_t* conv_state, const int32_t* state_indices,
    int64_t state_pool_size, const int64_t* slot_mapping, uint16_t* k_cache,
    uint16_t* v_cache, int64_t num_pages, int64_t page_size,
    int64_t stride_page, int64_t stride_slot, int64_t stride_head,
    double* z_k, double* z_v) {
  return oracle_prefill_varlen_opts(k, v, row_stride, num_tokens, cu_seqlens, num_seqs,
                                    conv_w_k, conv_w_v, gamma_k, gamma_v, 0, eps, W,
                                    num_heads, D, conv_state, state_indices, NULL,
                                    state_pool_size, slot_mapping, k_cache, v_cache,
                                    num_pages, page_size, stride_page, stride_slot,
                                    stride_head, z_k, z_v);
}

/*
 * Decode: the same step with exactly one new token per sequence
 * (cu_seqlens = 0, 1, ..., batch).
 */
int oracle_decode_opts(const uint16_t* k, const uint16_t* v, int64_t row_stride,
                       int batch, const uint16_t* conv_w_k,
                       const uint16_t* conv_w_v, const float* gamma_k,
                       const float* gamma_v, int64_t gamma_head_stride, double eps, int W,
                       int num_heads, int D, uint16_t* conv_state,
                       const int32_t* state_indices, const int64_t* state_positions,
                       int64_t state_pool_size, const int64_t* slot_mapping,
                       uint16_t* k_cache, uint16_t* v_cache, int64_t num_pages,
                       int64_t page_size, int64_t stride_page, int64_t stride_slot,
                       int64_t stride_head, double* z_k, double* z_v) {
  if (batch < 0) return ORACLE_ERR_ARG;
  int32_t* cu = (int32_t*)malloc(sizeof(int32_t) * (size_t)(batch + 1));
  if (!cu) return ORACLE_ERR_NOMEM;
  for (int i = 0; i <= batch; ++i) cu[i] = i;
  int rc = oracle_prefill_varlen_opts(
      k, v, row_stride, batch, cu, batch, conv_w_k, conv_w_v, gamma_k,
      gamma_v, gamma_head_stride, eps, W, num_heads, D, conv_state, state_indices,
      state_positions, state_pool_size, slot_mapping, k_cache, v_cache, num_pages,
      page_size, stride_page, stride_slot, stride_head, z_k, z_v);
  free(cu);
  return rc;
}

int oracle_decode(const uint16_t* k, const uint16_t* v, int64_t row_stride,
                  int batch, const uint16_t* conv_w_k,
                  const uint16_t* conv_w_v, const float* gamma_k,
                  const float* gamma_v, double eps, int W, int num_heads,
                  int D, uint16_t* conv_state, const int32_t* state_indices,
                  int64_t state_pool_size, const int64_t* slot_mapping,
                  uint16_t* k_cache, uint16_t* v_cache, int64_t num_pages,
                  int64_t page_size, int64_t stride_page, int64_t stride_slot,
                  int64_t stride_head, double* z_k, double* z_v) {
  return oracle_decode_opts(k, v, row_stride, batch, conv_w_k, conv_w_v, gamma_k, gamma_v, 0,
                            eps, W, num_heads, D, conv_state, state_indices, NULL,
                            state_pool_size, slot_mapping, k_cache, v_cache, num_pages,
                            page_size, stride_page, stride_slot, stride_head, z_k, z_v);
}

/* Vector helper for the Python side: round n doubles to bf16 bit patterns
 * with oracle_double_to_bf16. */
void oracle_round_bf16_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_bf16(x[i]);
}

/* ==================================================================== */
/* MXFP8 (block-scaled) cache store.                                    */
/*                                                                      */
/* Source: "Inkling-Small" SGLang cookbook, section 3.6 (Long Context):  */
/* KV entries can be stored as block-scaled MXFP8 instead of BF16,      */
/* about doubling the tokens a pool holds.  The pages give no block     */
/* size or scale format; MXFP8 is read as the OCP Microscaling format:  */
/* blocks of 32 consecutive elements (here: 32 channels of one head)    */
/* share one power-of-two scale X = 2^s stored as an E8M0 byte (s+127), */
/* and each element is stored as FP8 E4M3 of v/X.  The shared exponent  */
/* is s = floor(log2(max|v|)) - 8 (8 = exponent of E4M3's largest       */
/* normal, 448 = 1.75 * 2^8), clamped to [-127, 127]; elements are      */
/* rounded to nearest even and saturated to +-448.  The quantisation    */
/* decisions are taken on the normalised value rounded to binary32 (the */
/* kernel's precision), so both sides decide from the same kind of      */
/* number.                                                              */
/* ==================================================================== */

/* FP8 E4M3 (sign, 4-bit exponent with bias 7, 3-bit mantissa; largest
 * finite 448, no infinities, subnormals M * 2^-9) of a double: nearest
 * even on the E4M3 grid, magnitudes at or above 448 saturate to 448. */
uint8_t oracle_double_to_e4m3(double x) {
  if (isnan(x)) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1): floor(log2 a) = e-1 */
  int q = (e - 1) - 3;     /* grid spacing 2^q for normals */
  if (q < -9) q = -9;      /* subnormal spacing 2^-9 */
  double r = ldexp(rint(ldexp(a, -q)), q);
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return sign;
  frexp(r, &e);
  int E = (e - 1) + 7;
  if (E <= 0) return (uint8_t)(sign | (uint8_t)ldexp(r, 9)); /* M * 2^-9 */
  int M = (int)(ldexp(r, -(e - 1)) * 8.0) - 8;
  return (uint8_t)(sign | (uint8_t)(E << 3) | (uint8_t)M);
}

double oracle_e4m3_to_double(uint8_t c) {
  const double sign = (c & 0x80) ? -1.0 : 1.0;
  const int E = (c >> 3) & 0xF, M = c & 0x7;
  if (E == 0xF && M == 0x7) return NAN;
  if (E == 0) return sign * ldexp((double)M, -9);
  return sign * ldexp(1.0 + M / 8.0, E - 7);
}

/* Quantise one block of n binary32 values: shared exponent -> *scale
 * (E8M0 code), element codes -> codes[0..n). */
void oracle_mx_block(const float* v, int n, uint8_t* codes, uint8_t* scale) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i)
    if (fabs((double)v[i]) > amax) amax = fabs((double)v[i]);
  int s;
  if (amax < ldexp(1.0, -126)) {
    s = -127; /* zero or subnormal block: the smallest scale */
  } else {
    int e;
    frexp(amax, &e);
    s = (e - 1) - 8;
    if (s < -127) s = -127;
    if (s > 127) s = 127;
  }
  *scale = (uint8_t)(s + 127);
  for (int i = 0; i < n; ++i) codes[i] = oracle_double_to_e4m3(ldexp((double)v[i], -s));
}

/* The whole step with the MXFP8 store (steps a1-a3 and a5 as in
 * oracle_prefill_varlen; a4 writes E4M3 codes and E8M0 block scales).
 * Data caches: uint8, element (slot, h, d) at the usual element offset;
 * scale caches: uint8, block (slot, h, b) at (page*stride_page +
 * off*stride_slot + h*stride_head)/32 + b (all strides multiples of 32).
 * z_k / z_v (optional) receive the unrounded double values. */
int oracle_prefill_varlen_mxfp8_opts(
    const uint16_t* k, const uint16_t* v, int64_t row_stride,
    int64_t num_tokens, const int32_t* cu_seqlens, int num_seqs,
    const uint16_t* conv_w_k, const uint16_t* conv_w_v, const float* gamma_k,
    const float* gamma_v, int64_t gamma_head_stride, double eps, int W, int num_heads,
    int D, uint16_t* conv_state, const int32_t* state_indices,
    const int64_t* state_positions, int64_t state_pool_size,
    const int64_t* slot_mapping, uint8_t* k_data,
    uint8_t* k_scale, uint8_t* v_data, uint8_t* v_scale, int64_t num_pages,
    int64_t page_size, int64_t stride_page, int64_t stride_slot,
    int64_t stride_head, double* z_k, double* z_v) {
  if (D % 32 || stride_page % 32 || stride_slot % 32 || stride_head % 32)
    return ORACLE_ERR_ARG;
  const int C = num_heads * D;
  /* run the bf16 oracle for z and the state (its bf16 caches are scratch) */
  const int64_t num_slots = num_pages * page_size;
  uint16_t* scratch_k = (uint16_t*)calloc((size_t)(num_slots > 0 ? num_slots : 1) * (size_t)C, 2);
  uint16_t* scratch_v = (uint16_t*)calloc((size_t)(num_slots > 0 ? num_slots : 1) * (size_t)C, 2);
  double* zk = z_k ? z_k : (double*)malloc(sizeof(double) * (size_t)(num_tokens ? num_tokens : 1) * (size_t)C);
  double* zv = z_v ? z_v : (double*)malloc(sizeof(double) * (size_t)(num_tokens ? num_tokens : 1) * (size_t)C);
  if (!scratch_k || !scratch_v || !zk || !zv) {
    free(scratch_k); free(scratch_v);
    if (!z_k) free(zk);
    if (!z_v) free(zv);
    return ORACLE_ERR_NOMEM;
  }
  int rc = oracle_prefill_varlen_opts(
      k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v,
      gamma_k, gamma_v, gamma_head_stride, eps, W, num_heads, D, conv_state, state_indices,
      state_positions, state_pool_size, slot_mapping, scratch_k, scratch_v, num_slots, 1,
      C, C, D, zk, zv);
  free(scratch_k);
  free(scratch_v);
  if (rc == ORACLE_OK) {
    float block[32];
    for (int64_t t = 0; t < num_tokens; ++t) {
      const int64_t slot = slot_mapping[t];
      if (slot < 0 || slot >= num_slots) continue;
      const int64_t page = slot / page_size, off = slot % page_size;
      for (int which = 0; which < 2; ++which) {
        const double* z = (which == 0 ? zk : zv) + t * C;
        uint8_t* data = which == 0 ? k_data : v_data;
        uint8_t* scl = which == 0 ? k_scale : v_scale;
        for (int h = 0; h < num_heads; ++h) {
          const int64_t base = page * stride_page + off * stride_slot + h * stride_head;
          for (int b = 0; b < D / 32; ++b) {
            for (int i = 0; i < 32; ++i) block[i] = (float)z[h * D + b * 32 + i];
            oracle_mx_block(block, 32, data + base + b * 32, scl + base / 32 + b);
          }
        }
      }
    }
  }
  if (!z_k) free(zk);
  if (!z_v) free(zv);
  return rc;
}

int oracle_prefill_varlen_mxfp8(
    const uint16_t* k, const uint16_t* v, int64_t row_stride,
    int64_t num_tokens, const int32_t* cu_seqlens, int num_seqs,
    const uint16_t* conv_w_k, const uint16_t* conv_w_v, const float* gamma_k,
    const float* gamma_v, double eps, int W, int num_heads, int D,
    uint16_t* conv_state, const int32_t* state_indices,
    int64_t state_pool_size, const int64_t* slot_mapping, uint8_t* k_data,
    uint8_t* k_scale, uint8_t* v_data, uint8_t* v_scale, int64_t num_pages,
    int64_t page_size, int64_t stride_page, int64_t stride_slot,
    int64_t stride_head, double* z_k, double* z_v) {
  return oracle_prefill_varlen_mxfp8_opts(
      k, v, row_stride, num_tokens, cu_seqlens, num_seqs, conv_w_k, conv_w_v, gamma_k,
      gamma_v, 0, eps, W, num_heads, D, conv_state, state_indices, NULL, state_pool_size,
      slot_mapping, k_data, k_scale, v_data, v_scale, num_pages, page_size, stride_page,
      stride_slot, stride_head, z_k, z_v);
}

/* Vector helper for the Python side: E4M3 codes of n doubles. */
void oracle_e4m3_array(const double* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_e4m3(x[i]);
}
