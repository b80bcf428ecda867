// Fused ShortConv K/V step over a packed varlen batch, streaming version
// (sm_100a).
//
// Work split.  The packed token axis [0, T) is cut into `ctas` contiguous
// ranges of near-equal cost (a token costs 1, a sequence start a fixed
// number of tokens; one sequence is cut evenly), one per persistent CTA
// (x), and the channel groups into slices of at most 256 groups of 8
// channels (y).  A cut that
// would fall on positions 1..W-2 of a sequence is moved to position W-1 (or
// to the sequence's end), so the CTA holding position 0 of a sequence also
// holds every position whose window reaches into the old conv_state: that
// CTA is the only reader of the old state and the only writer of the new
// one, and no inter-CTA synchronisation is needed.  A cut moves forward by
// at most W-2 rows, so each CTA requests the full chunks of its unmoved
// range before it has read cu_seqlens.
//
// Pipeline.  The rows of the CTA's range (the W-1 rows in front of a range
// that starts inside a sequence are read directly) stream through a ring of
// `stages` shared-memory stages of R token rows each, filled by bulk
// asynchronous copies (for packed rows, one per chunk for K and one for V;
// otherwise one per row part), completion counted in bytes on the stage's
// "full" barrier.  Every warp waits on "full", copies
// the stage's rows into registers and arrives on the stage's "empty"
// barrier.  Thread 0 is also the producer: it fills the whole ring up front,
// and in iteration c it refills the stage of chunk c-1 (once every warp has
// released it) with chunk c-1+stages.  Loads in flight therefore do not
// occupy registers: each CTA keeps up to a ring's worth of rows requested
// while it computes.  (No separate producer warp: a 256-thread CTA may use
// up to 255 registers per thread, which the W <= 8 carried partials need.)
//
// Consumers.  Consumer thread g owns 8 channels (16 bytes of a row) and walks
// the rows in token order, carrying the causal depthwise conv in fp32
// registers as W-1 partial sums (transposed form, conv_step).  Per token:
// conv (packed-fp32 FMAs), per-head sum of squares (in-thread, then xor
// shuffles over D/8 lanes, a few tokens at once in the fast path), rsqrt,
// gamma, round to bf16 (or the MXFP8 block encoding), one streaming store
// into the cache slot.  At a sequence start the partials are built from the
// sequence's conv_state and the new state (the sequence's last W-1 raw rows)
// is written by the same thread over the rows it has just read.
#pragma once
#include "common.cuh"
#include "tma.cuh"

namespace sconv {

// Compile-time tuning (defaults chosen by measurement on B200).
#ifndef SCONV_PREFILL_ROWS
#define SCONV_PREFILL_ROWS 8
#endif
#ifndef SCONV_PREFILL_RING_KB
#define SCONV_PREFILL_RING_KB 96  // per CTA when two CTAs share an SM
#endif
#ifndef SCONV_PREFILL_SMALL_W_PER_SM
#define SCONV_PREFILL_SMALL_W_PER_SM 2  // CTAs per SM for W <= 4
#endif
#ifndef SCONV_PREFILL_BF16_THREADS
#define SCONV_PREFILL_BF16_THREADS 256  // threads per CTA of the bf16 store for W <= 4
#endif
#ifndef SCONV_PREFILL_BF16_UNROLL
#define SCONV_PREFILL_BF16_UNROLL 4  // fast-path unroll of the bf16 store for W <= 4
#endif
// Fast-path tokens per batched head reduction (head_rsqrt_batch).  Measured
// on B200 against batches of 4 (bf16, W <= 4 and MXFP8) and 8 (W > 4), one
// box, back to back: 65,536 tokens at W=8 101.1 -> 98.6 us, MXFP8 chunk
// 80.7 -> 80.1 us, MXFP8 varlen 178.4 -> 176.4 us, bf16 chunk 93.1 ->
// 92.3 us, bf16 varlen 206.5 -> 203.8 us (the shorter dependent shuffle
// chain hides better); the bf16 8192-token launch is the opposite case
// (15.6 against 16.1 us) and has its own instance (SCONV_PREFILL_SHORT_*).
#ifndef SCONV_PREFILL_NORM_BATCH
#define SCONV_PREFILL_NORM_BATCH 2
#endif
#ifndef SCONV_PREFILL_MX_NORM_BATCH
#define SCONV_PREFILL_MX_NORM_BATCH 2  // the same for the MXFP8 store, W <= 4
#endif
// Short launches (at most SCONV_PREFILL_SHORT_CHUNKS chunks per CTA) of the
// bf16 W <= 4 store: every CTA's chunks land at about the same time and the
// launch ends in a compute-bound tail, where fewer instructions per token
// count more than the reduction's latency: that instance reduces 4 tokens
// at a time.
#ifndef SCONV_PREFILL_SHORT_CHUNKS
#define SCONV_PREFILL_SHORT_CHUNKS 8
#endif
#ifndef SCONV_PREFILL_SHORT_NORM_BATCH
#define SCONV_PREFILL_SHORT_NORM_BATCH 4
#endif
#ifndef SCONV_PREFILL_MX_UNROLL
#define SCONV_PREFILL_MX_UNROLL 8  // fast-path unroll of the MXFP8 store for W <= 4
#endif
// The MXFP8 store for W <= 4: threads per CTA (= channel groups per slice)
// and CTAs per SM.  Measured on B200, with an 8-token unroll and gammas in
// registers: three 128-thread CTAs per SM (166 registers, 12 warps)
// against one 256-thread CTA (211 registers, 8 warps): 65,536-token launch
// 92.2 -> 85.3 us, varlen batch 198.2 -> 184.6 us, 8192-token launch
// 18.0 -> 17.7 us; one 256-thread CTA in turn beat two with a 2-token
// unroll (102.1 -> 92.2 us).  The MX store's per-token chain is longer
// than the bf16 store's: the launch is issue-latency-bound, and both the
// wider unroll and the extra warps hide it.
#ifndef SCONV_PREFILL_MX_THREADS
#define SCONV_PREFILL_MX_THREADS 128
#endif
#ifndef SCONV_PREFILL_MX_PER_SM
#define SCONV_PREFILL_MX_PER_SM 3
#endif
#ifndef SCONV_PREFILL_FIRST_FILL
// Chunks requested before the first one has landed (0 = the whole ring);
// the rest of the ring is requested once chunk 0 has landed.
#define SCONV_PREFILL_FIRST_FILL 0
#endif
#ifndef SCONV_PREFILL_BLOCK_LAYOUT
// Stage layout: 1 = [K rows][V rows] (one bulk copy per part when rows are
// packed), 0 = row by row (one copy per row part), 2 = per instance as
// block_layout<W, MX>() says.
#define SCONV_PREFILL_BLOCK_LAYOUT 2
#endif

constexpr int kTmaMaxGroups = 256;   // channel groups per CTA slice
#ifndef SCONV_PREFILL_ROWS_SMALL_W
#define SCONV_PREFILL_ROWS_SMALL_W SCONV_PREFILL_ROWS  // token rows per stage for W <= 4
#endif
// Token rows per stage (a chunk), by conv width.
template <int W>
__host__ __device__ constexpr int prefill_rows() {
  return W <= 4 ? SCONV_PREFILL_ROWS_SMALL_W : SCONV_PREFILL_ROWS;
}
inline int prefill_rows(int W) { return W <= 4 ? SCONV_PREFILL_ROWS_SMALL_W : SCONV_PREFILL_ROWS; }

// Measured on B200: with W <= 4 (two CTAs per SM, 128 registers) the fast
// path is unrolled by 4 and gamma is read from shared memory per token,
// which frees the registers the unrolled tokens need; wider windows run one
// CTA per SM with room for an 8-token unroll and gamma in registers.
template <int W, bool MX>
__host__ __device__ constexpr int prefill_ctas_per_sm() {
  return W <= 4 ? (MX ? SCONV_PREFILL_MX_PER_SM : SCONV_PREFILL_SMALL_W_PER_SM) : 1;
}
// Threads per CTA, one per channel group of the CTA's slice.
template <int W, bool MX>
__host__ __device__ constexpr int prefill_threads() {
  return W <= 4 ? (MX ? SCONV_PREFILL_MX_THREADS : SCONV_PREFILL_BF16_THREADS) : kTmaMaxGroups;
}
inline int prefill_threads(int W, bool mx) {
  return W <= 4 ? (mx ? SCONV_PREFILL_MX_THREADS : SCONV_PREFILL_BF16_THREADS) : kTmaMaxGroups;
}
// gammas read from shared memory per token: when an SM holds 512 threads
// or more (at most 128 registers each) there is no room to hold them
template <int W, bool MX>
__host__ __device__ constexpr bool gamma_in_smem() {
  return prefill_threads<W, MX>() * prefill_ctas_per_sm<W, MX>() >= 512;
}
// (the W=3 and W=4 bf16 layout-variant instances carry two more live
// values at their 128-register cap: there only a 2-token unroll and batch
// stay free of spills for every head size)
template <int W, bool MX, bool LV = false>
__host__ __device__ constexpr int fast_unroll() {
  return (W >= 3 && W <= 4 && !MX && LV) ? 2
         : W <= 4 ? (MX ? SCONV_PREFILL_MX_UNROLL : SCONV_PREFILL_BF16_UNROLL) : 8;
}
// tokens whose head reductions run together in the fast path (a divisor
// of the unroll)
// NBX > 0: an instance's own batch (the short-launch instances)
template <int W, bool MX, bool LV, int NBX = 0>
__host__ __device__ constexpr int norm_batch() {
  return NBX > 0 ? NBX
         : (W <= 4 && MX) ? SCONV_PREFILL_MX_NORM_BATCH
         : (W >= 3 && W <= 4 && !MX && LV) ? 2
         : SCONV_PREFILL_NORM_BATCH < fast_unroll<W, MX>() ? SCONV_PREFILL_NORM_BATCH
                                                           : fast_unroll<W, MX>();
}
// Measured on B200: the block layout (2 bulk copies per chunk instead of
// 2 per row) speeds up the wide-window and MXFP8 instances by 14-25 %; in
// the W=4 bf16 instance its extra per-thread register spills at the
// 128-register cap and costs 5 %, so that one keeps the row layout.
template <int W, bool MX>
__host__ __device__ constexpr bool block_layout() {
  return SCONV_PREFILL_BLOCK_LAYOUT == 1 ||
         (SCONV_PREFILL_BLOCK_LAYOUT == 2 && !(W == 4 && !MX));
}
constexpr int kTmaRingBytes2 = SCONV_PREFILL_RING_KB * 1024;
constexpr int kTmaCuSmemMax = 2048;  // cu_seqlens entries staged in shared memory
// per-warp slot tables: the cache row offset of each row of a 32-row window
// in units of 8 elements (kNoRow: not written), 4 bytes per row; the host
// refuses caches whose row offsets do not fit
constexpr uint32_t kNoRow = 0xFFFFFFFFu;
constexpr int kTmaOffTableBytes = (kTmaMaxGroups / 32) * 32 * 4;
// Every stage is laid out for a full slice: R rows of (threads per CTA) *
// 16 bytes (the row layout keeps that fixed pitch between rows, so a
// thread's per-token shared-memory loads take immediate offsets).
template <int W, bool MX>
__host__ __device__ constexpr int prefill_row_pitch() { return prefill_threads<W, MX>() * 16; }
template <int W, bool MX>
__host__ __device__ constexpr int prefill_stage_bytes() {
  return prefill_rows<W>() * prefill_row_pitch<W, MX>();
}
inline int prefill_stage_bytes(int W, bool mx) { return prefill_rows(W) * prefill_threads(W, mx) * 16; }
// per-thread gammas in shared memory (8 floats per thread), when used
template <int W, bool MX>
__host__ __device__ constexpr int prefill_gamma_bytes() {
  return gamma_in_smem<W, MX>() ? prefill_threads<W, MX>() * 32 : 0;
}
inline int prefill_gamma_bytes(int W, bool mx) {
  const int per_sm = W <= 4 ? (mx ? SCONV_PREFILL_MX_PER_SM : SCONV_PREFILL_SMALL_W_PER_SM) : 1;
  return prefill_threads(W, mx) * per_sm >= 512 ? prefill_threads(W, mx) * 32 : 0;
}

struct TmaGeom {
  int slice;      // channel groups per full slice (min(NG, threads per CTA))
  int stages;     // ring depth
  int ctas;       // persistent CTAs along the token axis
  int withhold_first;  // testing: chunk 0 is never requested (its wait runs out)
  int seq_cost;   // weight of a sequence start, in tokens (cut by cost)
  int cut_q;      // num_tokens / ctas
  int cut_r;      // num_tokens % ctas (the first cut_r ranges take one more token)
  int cu_smem;    // cu_seqlens copied to shared memory (num_seqs < kTmaCuSmemMax)
  int smem_ring;  // bytes of the stage ring
  int state_wait_only;  // only conv_state reads wait for the previous kernel
  unsigned long long timeout_ns;
};

// Per-token work of one thread: the conv of its 8 channels, in transposed
// form.  part[k-1] holds P_k, the part of the output k tokens ahead that the
// rows seen so far contribute: P_k = w_0 x_{t+k-W+1} + ... + w_{W-1-k} x_t,
// summed in tap order.  A new row x_t completes y_t = w_{W-1} x_t + P_1 and
// extends every other partial by one tap, P_k <- w_{W-1-k} x_t + P_{k+1}
// (P_{W-1} <- w_0 x_t).  Each output is thus the same chain of fused
// multiply-adds, in the same tap order, as the direct sum over the window
// w_0 x_{t-W+1} + ... + w_{W-1} x_t, and bitwise equal to it; the carried
// values are produced in place, so no window rows are shifted between
// tokens.  Returns the conv output in acc.
template <int W>
__device__ __forceinline__ void conv_step(const float2 (&tw)[W][4], float2 (&part)[W > 1 ? W - 1 : 1][4],
                                          const uint4& xr, float2 (&acc)[4]) {
  float2 xf[4];
  unpack8(xr, xf);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if constexpr (W == 1) {
      acc[e] = fmul2(tw[0][e], xf[e]);
    } else {
      acc[e] = ffma2(tw[W - 1][e], xf[e], part[0][e]);
#pragma unroll
      for (int k = 1; k < W - 1; ++k) part[k - 1][e] = ffma2(tw[W - 1 - k][e], xf[e], part[k][e]);
      part[W - 2][e] = fmul2(tw[0][e], xf[e]);
    }
  }
}

// The partials P_1 .. P_{W-1} of the window's W-1 rows in front of a token
// (h[0] oldest), built tap by tap in the order conv_step extends them.
template <int W>
__device__ __forceinline__ void conv_prime(const float2 (&tw)[W][4], const uint4 (&hb)[W > 1 ? W - 1 : 1],
                                           float2 (&part)[W > 1 ? W - 1 : 1][4]) {
  if constexpr (W > 1) {
    float2 h[W - 1][4];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) unpack8(hb[j], h[j]);
#pragma unroll
    for (int k = 1; k < W; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 p = fmul2(tw[0][e], h[k - 1][e]);
#pragma unroll
        for (int j = 1; j < W - k; ++j) p = ffma2(tw[j][e], h[k + j - 1][e], p);
        part[k - 1][e] = p;
      }
  }
}

// Sum of squares of this lane's 8 conv outputs (even and odd lanes of the
// packed pairs summed separately, then added).
__device__ __forceinline__ float sum_sq8(const float2 (&acc)[4]) {
  float2 s2 = fmul2(acc[0], acc[0]);
  s2 = ffma2(acc[1], acc[1], s2);
  s2 = ffma2(acc[2], acc[2], s2);
  s2 = ffma2(acc[3], acc[3], s2);
  return s2.x + s2.y;
}

// 1/rms of NB tokens at once: v[t] holds this lane's sum of squares of
// token t; r[t] receives rsqrt(total over the lane's group of G lanes *
// inv_d + eps) on every lane.  The first log2(min(NB, G)) butterfly levels
// halve the values a lane carries: of each pair of tokens it keeps the one
// its lane bit at that level selects and adds the partner lane's partial of
// that token; the remaining levels are plain.  Every addition joins the same
// two lane sets as group_sum's butterfly (own partial + partner's), so each
// total is bitwise the one group_sum gives.  One rsqrt per lane, then each
// token's value is fetched from a lane that holds it (shfl.idx whose
// segment mask keeps the lane's own bits outside the selecting ones).
template <int G, int NB>
__device__ __forceinline__ void head_rsqrt_batch(float (&v)[NB], float inv_d, float eps, float (&r)[NB]) {
  constexpr int LG = G >= 32 ? 5 : G >= 16 ? 4 : G >= 8 ? 3 : G >= 4 ? 2 : G >= 2 ? 1 : 0;
  constexpr int LN = NB >= 8 ? 3 : NB >= 4 ? 2 : NB >= 2 ? 1 : 0;
  static_assert((1 << LG) == G && (1 << LN) == NB, "powers of two");
  constexpr int H = LN < LG ? LN : LG;  // halving levels
  constexpr int NL = NB >> H;           // values left per lane
#pragma unroll
  for (int i = 0; i < H; ++i) {
    const int m = G >> (i + 1);
    const bool hi = (threadIdx.x & m) != 0;
    const int half = NB >> (i + 1);
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float a = v[k], b = v[k + half];
      const float keep = hi ? b : a;
      const float send = hi ? a : b;
      v[k] = keep + __shfl_xor_sync(kFullMask, send, m);
    }
  }
  float own[NL];
#pragma unroll
  for (int k = 0; k < NL; ++k) {
    float x = v[k];
#pragma unroll
    for (int m = G >> (H + 1); m >= 1; m >>= 1) x += __shfl_xor_sync(kFullMask, x, m);
    own[k] = rsqrt_approx(fmaf(x, inv_d, eps));
  }
  // token t = k + sum_i b_i * (NB >> (i+1)), b_i the lane bit at position
  // LG-1-i: its holders have those bits, any others
  constexpr int kSel = ((1 << LG) - 1) & ~((1 << (LG - H)) - 1);
  constexpr unsigned kC = ((0x1fu & ~static_cast<unsigned>(kSel)) << 8) | 0x1fu;
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    int bits = 0;
#pragma unroll
    for (int i = 0; i < H; ++i)
      if ((t / (NB >> (i + 1))) & 1) bits |= 1 << (LG - 1 - i);
    if constexpr (H == 0) {
      r[t] = own[t];
    } else {
      float y;
      asm volatile("shfl.sync.idx.b32 %0, %1, %2, %3, 0xffffffff;"
                   : "=f"(y) : "f"(own[t % NL]), "r"(bits), "n"(kC));
      r[t] = y;
    }
  }
}

// 8 gammas from shared memory, read at the point of use (kept out of
// registers: the loads are volatile, so they are not hoisted).
__device__ __forceinline__ void lds_gamma(const float* g, float2 (&gm)[4]) {
  float4 a, b;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(a.x), "=f"(a.y), "=f"(a.z), "=f"(a.w)
               : "r"(smem_u32(g)));
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(b.x), "=f"(b.y), "=f"(b.z), "=f"(b.w)
               : "r"(smem_u32(g + 4)));
  gm[0] = make_float2(a.x, a.y);
  gm[1] = make_float2(a.z, a.w);
  gm[2] = make_float2(b.x, b.y);
  gm[3] = make_float2(b.z, b.w);
}

// NB consecutive entries of a slot table (16-byte aligned for NB >= 4,
// NB * 4 bytes aligned below that) in as few shared-memory loads as fit.
template <int NB>
__device__ __forceinline__ void load_offsets(const uint32_t* p, uint32_t (&o)[NB]) {
  if constexpr (NB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NB; i += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(p + i);
      o[i] = v.x; o[i + 1] = v.y; o[i + 2] = v.z; o[i + 3] = v.w;
    }
  } else if constexpr (NB == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    o[0] = v.x; o[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < NB; ++i) o[i] = p[i];
  }
}

// Gamma and the head's 1/rms applied, then either bf16 rounding and a
// 16-byte store into the bf16 cache (MX = false), or the MXFP8 block store
// (8 E4M3 bytes + the block's E8M0 scale), at cache row offset off8 (units
// of 8 elements; kNoRow: not written).
template <bool MX>
__device__ __forceinline__ void scale_store(const float2 (&acc)[4], const float2 (&gm)[4], float rn,
                                            uint32_t off8, uint16_t* cache, uint8_t* mx_data,
                                            uint8_t* mx_scale, int scale_lane) {
  const float2 rr = make_float2(rn, rn);
  if constexpr (MX) {
    const float2 t[4] = {fmul2(acc[0], gm[0]), fmul2(acc[1], gm[1]), fmul2(acc[2], gm[2]),
                         fmul2(acc[3], gm[3])};
    uint32_t w0, w1, sb;
    mx_encode8(t, rn, w0, w1, sb);
    st_row_mx(off8, mx_data, mx_scale, scale_lane, w0, w1, sb);
  } else {
    uint4 o;
    o.x = pack_bf16x2(fmul2(fmul2(acc[0], rr), gm[0]));
    o.y = pack_bf16x2(fmul2(fmul2(acc[1], rr), gm[1]));
    o.z = pack_bf16x2(fmul2(fmul2(acc[2], rr), gm[2]));
    o.w = pack_bf16x2(fmul2(fmul2(acc[3], rr), gm[3]));
    st_row_bf16(off8, cache, o);
  }
}

template <int W, int D, bool MX, bool LV, int NBX>
__device__ __forceinline__ void prefill_body(const StepParams& P, const TmaGeom& Gm) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int R = prefill_rows<W>();
  constexpr int kTmaStageBytes = prefill_stage_bytes<W, MX>();
  constexpr int kTmaRowPitch = prefill_row_pitch<W, MX>();
  constexpr int kTmaGammaBytes = prefill_gamma_bytes<W, MX>();
  // layout variants (per-head gamma stride, ring-buffer state) only in the
  // LV instances: elsewhere these fold to the defaults at compile time, so
  // the default path carries no extra live values
  const int64_t gamma_hs = LV ? P.gamma_hs : 0;
  const int64_t* const state_pos = LV ? P.state_pos : nullptr;
  const int S = P.num_seqs;
  const int T = static_cast<int>(P.num_tokens);
  const int NS = Gm.stages;
  const int first_fill = SCONV_PREFILL_FIRST_FILL > 0 ? min(NS, SCONV_PREFILL_FIRST_FILL) : NS;

  // ---- channel slice of this CTA
  const int half = P.NG >> 1;
  const int g0 = blockIdx.y * Gm.slice;
  const int cs = min(Gm.slice, P.NG - g0);
  const int ncw = (cs + 31) >> 5;  // warps (all consume; thread 0 also produces)
  const int kn = max(0, min(g0 + cs, half) - g0);           // K groups in slice
  const int vg0 = max(g0, half);
  const int vn = max(0, g0 + cs - vg0);                     // V groups in slice
  const int row_bytes = cs * 16;

  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Gm.smem_ring);
  uint64_t* empty = full + NS;
  volatile int* abort = reinterpret_cast<volatile int*>(empty + NS);
  // after the barriers: abort flag (16 bytes), one int per warp (32 bytes),
  // then cu_seqlens when staged in shared memory
  int* s_cu = const_cast<int*>(reinterpret_cast<volatile int*>(empty + NS) + 12);
  // per-warp table of the cache row offsets of the current 32-row window
  // (host reserves 8 warps x 32 x 8 bytes right below the barriers)
  uint32_t* warp_off =
      reinterpret_cast<uint32_t*>(smem + Gm.smem_ring - kTmaOffTableBytes) + (threadIdx.x >> 5) * 32;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Even split of the token axis: range b starts at cut_even(b).  The final
  // cut (below, once cu_seqlens is read) only moves a start forward, by at
  // most W-2 rows, so the chunks of [cut_even(b), cut_even(b+1)) can be
  // requested before cu_seqlens arrives.  Chunk c covers rows
  // first_row + c*R ... whatever the final start is; rows in front of the
  // final start are skipped by the consumers.
  auto cut_even = [&](int b) -> int { return min(b * Gm.cut_q + min(b, Gm.cut_r), T); };
  int first_row = cut_even(blockIdx.x);  // (final value set below)
  int tb = cut_even(blockIdx.x + 1);      // end of the range (final value set below)

  // =================================================================== producer
  // Issue chunk c into stage `st` (= c % NS, tracked by the caller).
  // Block layout: a stage holds its R rows' K parts (kn*16 bytes each) back
  // to back, then their V parts.  When a part is a whole row of a packed
  // tensor (row_stride == C), the chunk's rows of that part are one
  // contiguous range in global memory and take a single bulk copy.  Row
  // layout: row r of the stage is its K part then its V part.
  constexpr bool kBlock = block_layout<W, MX>();
  const bool k_packed = kn == half && P.row_stride == P.C;
  const bool v_packed = vn == half && P.row_stride == P.C;
  auto issue = [&](int c, int st) {
    if (c == 0 && Gm.withhold_first) return;  // nothing will complete this stage
    const int r0 = first_row + c * R;
    const int rows = min(R, tb - r0);
    mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(rows * row_bytes));
    unsigned char* sdst = ring + static_cast<size_t>(st) * kTmaStageBytes;
    const uint16_t* ksrc = P.k + static_cast<int64_t>(r0) * P.row_stride + g0 * 8;
    const uint16_t* vsrc = P.v + static_cast<int64_t>(r0) * P.row_stride + (vg0 - half) * 8;
    if constexpr (kBlock) {
      unsigned char* vdst = sdst + R * kn * 16;
      if (kn) {
        if (k_packed) {
          bulk_g2s(sdst, ksrc, rows * kn * 16, &full[st]);
        } else {
          for (int r = 0; r < rows; ++r)
            bulk_g2s(sdst + r * kn * 16, ksrc + static_cast<int64_t>(r) * P.row_stride, kn * 16,
                     &full[st]);
        }
      }
      if (vn) {
        if (v_packed) {
          bulk_g2s(vdst, vsrc, rows * vn * 16, &full[st]);
        } else {
          for (int r = 0; r < rows; ++r)
            bulk_g2s(vdst + r * vn * 16, vsrc + static_cast<int64_t>(r) * P.row_stride, vn * 16,
                     &full[st]);
        }
      }
    } else {
      for (int r = 0; r < rows; ++r) {
        const int64_t o = static_cast<int64_t>(r) * P.row_stride;
        if (kn) bulk_g2s(sdst, ksrc + o, kn * 16, &full[st]);
        if (vn) bulk_g2s(sdst + kn * 16, vsrc + o, vn * 16, &full[st]);
        sdst += kTmaRowPitch;
      }
    }
  };
  int issued = 0;  // chunks issued so far (thread 0 only)

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], ncw);
    }
    *abort = 0;
    mbar_init_fence();
  }
  // inputs may come from the previous kernel in the stream; with the
  // state-only dependency only the reads of conv_state rows wait for it
  if (!Gm.state_wait_only) grid_dependency_wait();
  // This grid lets the next one launch (griddepcontrol.launch_dependents)
  // once its copies are all issued; a CTA that has not waited for the
  // previous grid yet does so first, so that the next grid never runs
  // ahead of this grid's own predecessor.
  auto trigger = [&]() {
    if (Gm.state_wait_only) grid_dependency_wait();
    allow_dependent_launch();
  };
  if (kBlock && threadIdx.x == 0) {
    // full chunks that lie inside the even range: requested at once (block
    // layout only; in the W=4 bf16 instance the extra live values spill at
    // its 128-register cap, so it requests after the cut)
    const int spec = S == 1 ? min(first_fill, (tb - first_row) / R) : 0;
    for (; issued < spec; ++issued) issue(issued, issued);
  }
  if (Gm.cu_smem)
    for (int i = threadIdx.x; i <= S; i += blockDim.x) s_cu[i] = P.cu_seqlens[i];
  __syncthreads();

  auto cu = [&](int i) -> int { return Gm.cu_smem ? s_cu[i] : __ldg(P.cu_seqlens + i); };
  // largest i in [0, S-1] with cu[i] <= t
  auto seq_of = [&](int t) -> int {
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cu(mid) <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  // start of range b: even cut, moved off positions 1..W-2 of a sequence
  // Cut by cost: a token weighs 1 and a sequence start Gm.seq_cost tokens
  // (its state read and write are latency the CTA cannot hide), so CTAs
  // full of short sequences get fewer tokens.  Sequence i's start sits at
  // weight cu[i] + cost*i; target weight X falls in the last sequence whose
  // start is at or below it.  A single sequence keeps the even split.
  auto base_cut = [&](int b) -> int {
    if (S <= 1 || Gm.seq_cost == 0) return cut_even(b);
    const long long cost = Gm.seq_cost;
    const long long X = static_cast<long long>(b) * (T + cost * S) / Gm.ctas;
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cu(mid) + cost * mid <= X) lo = mid; else hi = mid - 1;
    }
    long long t = cu(lo) + max(0ll, X - (cu(lo) + cost * lo) - cost);
    t = min(t, static_cast<long long>(cu(lo + 1)));
    return static_cast<int>(min(max(t, 0ll), static_cast<long long>(T)));
  };
  static_assert(R > W - 2, "a moved cut must stay inside the first chunk");
  auto cut = [&](int b) -> int {
    const int s0 = base_cut(b);
    if (s0 >= T) return T;
    int s = s0;
    if (W > 1) {
      const int i = seq_of(s);
      const int a = cu(i), e = cu(i + 1);
      const int p = s - a;
      if (p > 0 && p < W - 1) s = a + min(W - 1, e - a);
      // never backwards nor by W-1 or more rows, even for a malformed
      // cu_seqlens (which is flagged below)
      s = min(max(s, s0), min(s0 + W - 2, T));
    }
    return s;
  };
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    // cu_seqlens must start at 0, end at T and never decrease (the block's
    // threads check the entries in parallel)
    bool ok = threadIdx.x != 0 || (cu(0) == 0 && cu(S) == T);
    for (int i = threadIdx.x; i < S && ok; i += blockDim.x) ok = cu(i) <= cu(i + 1);
    if (!ok) raise_flag(P.err, kFlagCuSeqlens);
  }
  first_row = base_cut(blockIdx.x);  // equals the even cut for a single sequence
  const int ta = cut(blockIdx.x);
  // rows of chunk 0 in front of ta, one copy per warp in shared memory (read
  // once per 32-row window: a register here spills in the W=4 bf16 instance)
  volatile int* s_skip = abort + 4 + warp;
  if (lane == 0) *s_skip = ta - first_row;
  __syncwarp();
  tb = max(ta, cut(blockIdx.x + 1));
  if (ta >= tb) return;
  // The CTA walks rows from first_row.  Rows first_row .. ta-1 (at most W-2,
  // all in chunk 0) belong to the previous range: they only feed the conv's
  // partials, and their stores are masked through the slot table.  A moved
  // cut puts ta at position W-1 of its sequence (the partials then cover
  // rows 0 .. W-2 of it) or at a sequence start (whose partials are built
  // from its state).  An empty range has requested nothing: its even range
  // is shorter than W-1 < R rows.
  const int seq0 = seq_of(first_row);
  // a walk that starts inside a sequence needs the W-1 rows in front of
  // first_row (its halo); they are read directly below, so the ring holds
  // exactly the walked rows and every full chunk can take the fast path
  const bool mid_sequence = (W > 1 && first_row > cu(seq0));
  const int nrows = tb - first_row;
  const int nchunks = (nrows + R - 1) / R;

  // After giving up, let the copies already issued land before the CTA's
  // shared memory can be released (bounded as well).
  auto drain = [&]() {
    for (int d = max(0, issued - NS); d < issued; ++d) {
      if (d == 0 && Gm.withhold_first) continue;  // never requested
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(&full[d % NS], (d / NS) & 1) && global_ns() - t0 < kDrainTimeoutNs) {
      }
    }
  };
  if (threadIdx.x == 0) {
    for (; issued < min(first_fill, nchunks); ++issued) issue(issued, issued);
    if (issued == nchunks) trigger();
  }

  // =================================================================== consumers
  const int lg = threadIdx.x;  // local channel group
  const bool active = lg < cs;
  const int g = g0 + (active ? lg : 0);
  const bool isv = g >= half;
  const int c0 = (isv ? g - half : g) * 8;
  const int d0 = c0 % D;
  const uint16_t* xbase = (isv ? P.v : P.k) + c0;
  uint16_t* cache = MX ? nullptr : (isv ? P.v_cache : P.k_cache) + (c0 / D) * P.stride_head + d0;
  // MXFP8 store: element offsets as for bf16 (bytes), scale offset / 32
  const int64_t head_off = (c0 / D) * P.stride_head + d0;
  uint8_t* mxdata = MX ? (isv ? P.v_data : P.k_data) + head_off : nullptr;
  uint8_t* mxscale = MX ? (isv ? P.v_scale : P.k_scale) + (head_off >> 5) : nullptr;
  const int64_t srow = 2 * static_cast<int64_t>(P.C);
  const int st_chan = (isv ? P.C : 0) + c0;

  float2 tw[W][4];
  {
    const uint16_t* w = (isv ? P.w_v : P.w_k) + c0;
#pragma unroll
    for (int j = 0; j < W; ++j) unpack8(ld_ro(w + static_cast<int64_t>(j) * P.C), tw[j]);
  }
  // gamma: this thread's 8 values, either staged in its own 32 bytes of
  // shared memory (read per token) or held in registers
  float* my_gamma = reinterpret_cast<float*>(smem + Gm.smem_ring - kTmaOffTableBytes -
                                             kTmaGammaBytes) + threadIdx.x * 8;
  float2 gm[4];
  {
    const float* gam = (isv ? P.gamma_v : P.gamma_k) + (c0 / D) * gamma_hs + d0;
    const float4 a = __ldg(reinterpret_cast<const float4*>(gam));
    const float4 b = __ldg(reinterpret_cast<const float4*>(gam) + 1);
    if constexpr (gamma_in_smem<W, MX>()) {
      reinterpret_cast<float4*>(my_gamma)[0] = a;
      reinterpret_cast<float4*>(my_gamma)[1] = b;
    } else {
      gm[0] = make_float2(a.x, a.y);
      gm[1] = make_float2(a.z, a.w);
      gm[2] = make_float2(b.x, b.y);
      gm[3] = make_float2(b.z, b.w);
    }
  }
  // the conv's carried partials (conv_step), set at each sequence start
  constexpr int NH = W > 1 ? W - 1 : 1;
  float2 part[NH][4];
#pragma unroll
  for (int j = 0; j < NH; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) part[j][e] = make_float2(0.f, 0.f);

  int seq = seq0;
  int next = (seq + 1 <= S) ? cu(seq + 1) : T;
  bool skip = false;  // current sequence is not processed (bad state index / cu)
  const bool report = blockIdx.y == 0 && threadIdx.x == 0;
  const bool report_slots = blockIdx.y == 0 && warp == 0;  // lane r checks row r's slot

  // Is sequence i processed?  (cu_seqlens entry sane, state index in the
  // pool.)  A sequence that fails is skipped by every CTA that touches it.
  auto check_sequence = [&](int i, int64_t& si) -> bool {
    const int a = cu(i), e = cu(i + 1);
    if (!(a >= 0 && a <= e && e <= T)) {
      if (report) raise_flag(P.err, kFlagCuSeqlens);
      return false;
    }
    si = i;
    if constexpr (W > 1) {
      si = P.state_indices ? static_cast<int64_t>(P.state_indices[i]) : i;
      if (si < 0 || si >= P.pool || (state_pos && state_pos[i] < 0)) {
        if (report) raise_flag(P.err, kFlagStateIndex);
        return false;
      }
    }
    return true;
  };

  // Enter sequence `i` at its first token: validate, build the conv's
  // partials from the old state, write the new state.
  auto start_sequence = [&](int i) {
    int64_t si;
    skip = !check_sequence(i, si);
    if (skip) return;
    if constexpr (W > 1) {
      // the previous kernel in the stream may have written this state row
      if (Gm.state_wait_only) grid_dependency_wait();
      const int a = cu(i), e = cu(i + 1);
      uint16_t* st = P.state + si * (W - 1) * srow + st_chan;
      // ring state: position p in row p mod (W-1); the window's oldest row
      // (position pos0-(W-1)) sits in row pos0 mod (W-1)
      const int rot = state_pos ? static_cast<int>(state_pos[i] % (W - 1)) : 0;
      uint4 hb[W - 1];
#pragma unroll
      for (int j = 0; j < W - 1; ++j) {
        const int row = rot + j < W - 1 ? rot + j : rot + j - (W - 1);
        hb[j] = active ? *reinterpret_cast<const uint4*>(st + row * srow) : make_uint4(0, 0, 0, 0);
      }
      if (active) {
        const int L = e - a;
        const uint16_t* xs = xbase + static_cast<int64_t>(a) * P.row_stride;
        if (state_pos) {
          // ring: only the rows of the last min(L, W-1) positions change
#pragma unroll
          for (int j = 0; j < W - 1; ++j) {
            const int q = L - (W - 1) + j;
            if (q >= 0)
              *reinterpret_cast<uint4*>(st + ((rot + q) % (W - 1)) * srow) =
                  ld_ro(xs + static_cast<int64_t>(q) * P.row_stride);
          }
        } else {
#pragma unroll
          for (int j = 0; j < W - 1; ++j) {
            const int q = L - (W - 1) + j;  // row of (old state ++ sequence)
            uint4 r;
            if (q >= 0) {
              r = ld_ro(xs + static_cast<int64_t>(q) * P.row_stride);
            } else {
              r = hb[0];
#pragma unroll
              for (int m = 1; m < W - 1; ++m)
                if (m == W - 1 + q) r = hb[m];
            }
            *reinterpret_cast<uint4*>(st + j * srow) = r;
          }
        }
      }
      conv_prime<W>(tw, hb, part);
    }
  };

  if (!mid_sequence) {
    start_sequence(seq);
  } else {
    int64_t si;
    skip = !check_sequence(seq, si);
    if constexpr (W > 1) {
      // halo: rows first_row-(W-1) .. first_row-1.  When first_row == ta
      // (the cut did not move) they lie in ta's sequence at positions >= 0,
      // never in the state; otherwise they only feed the masked rows.
      uint4 hb[W - 1];
#pragma unroll
      for (int j = 0; j < W - 1; ++j) {
        const int64_t q = static_cast<int64_t>(first_row) - (W - 1) + j;
        hb[j] = (active && q >= 0) ? ld_ro(xbase + q * P.row_stride) : make_uint4(0, 0, 0, 0);
      }
      conv_prime<W>(tw, hb, part);
    }
  }

  const float eps = P.eps, inv_d = P.inv_d;
  // A row's cache offset is kept in units of 8 elements (bf16: 16 bytes;
  // MXFP8: 8 code bytes, and a quarter of a scale byte), kNoRow if the row
  // is not written; lanes outside the slice force every offset to kNoRow.
  // (vector loads of a batch's offsets only where registers are plentiful:
  // at the 128-register cap of the bf16 W <= 4 instances they spill)
  constexpr bool kVecOffsets = !gamma_in_smem<W, MX>();
  const int scale_lane = (threadIdx.x & 3) == 0;  // MXFP8: writes its block's scale
#define SCALE_STORE(a, rn, gs, off)                                                 \
  scale_store<MX>(a, gs, rn, off, cache, mxdata, mxscale, scale_lane)
  // one token (sequence starts, partial chunks): its head's 1/rms, the store
#define NORM_STORE(off)                                                             \
  do {                                                                              \
    float2 gs[4];                                                                   \
    if constexpr (gamma_in_smem<W, MX>()) lds_gamma(my_gamma, gs);                  \
    const float ss_ = group_sum<D / 8>(sum_sq8(acc));                               \
    SCALE_STORE(acc, rsqrt_approx(fmaf(ss_, inv_d, eps)),                           \
                (gamma_in_smem<W, MX>() ? gs : gm), off);                           \
  } while (0)
  // NB tokens from row `rb` of the stage: conv, their 1/rms together
  // (head_rsqrt_batch), then scale and store each; the batch's NB row
  // offsets are one vector load (rb is a multiple of NB)
#define FAST_BATCH(rb)                                                              \
  do {                                                                              \
    float2 acc[NB][4];                                                              \
    float ss[NB], rn[NB];                                                           \
    _Pragma("unroll") for (int u = 0; u < NB; ++u) {                                \
      const uint4 xr = *reinterpret_cast<const uint4*>(stage + ((rb) + u) * my_rs); \
      conv_step<W>(tw, part, xr, acc[u]);                                           \
      ss[u] = sum_sq8(acc[u]);                                                      \
    }                                                                               \
    head_rsqrt_batch<D / 8, NB>(ss, inv_d, eps, rn);                                \
    uint32_t offs[NB];                                                              \
    if constexpr (kVecOffsets) load_offsets<NB>(warp_off + sbase + (rb), offs);     \
    _Pragma("unroll") for (int u = 0; u < NB; ++u) {                                \
      if constexpr (!kVecOffsets) offs[u] = warp_off[sbase + (rb) + u];             \
      float2 gs[4];                                                                 \
      if constexpr (gamma_in_smem<W, MX>()) lds_gamma(my_gamma, gs);                \
      SCALE_STORE(acc[u], rn[u], (gamma_in_smem<W, MX>() ? gs : gm), active ? offs[u] : kNoRow); \
    }                                                                               \
  } while (0)
  // inactive lanes read column 0 (and never store): no predicated loads
  const unsigned char* my_ring =
      !kBlock ? ring + (active ? lg : 0) * 16
              : ring + (!active ? 0 : lg < kn ? lg * 16 : R * kn * 16 + (lg - kn) * 16);
  // bytes between consecutive rows of this thread's part of a stage
  const int my_rs = !kBlock ? kTmaRowPitch : (active && lg >= kn) ? vn * 16 : kn * 16;
  // slot_mapping is read one 32-row window ahead of use, lane l holding row
  // (window start + l), so its load latency hides behind four chunks.
  constexpr int SW = (32 / R) * R;
  auto load_slot = [&](int w) -> long long {
    const int r = first_row + w * SW + lane;
    return r < tb ? P.slots[r] : -1;
  };
  long long next_slot = load_slot(0);
  // stage and phase parity of chunk c (kept without divisions)
  int s = 0;
  uint32_t ph = 0;
  for (int c = 0; c < nchunks; ++c) {
    // a wait that gives up ends the whole warp at once (lanes may disagree,
    // and no lane may be left waiting at a warp-synchronous step for one
    // that has left); thread 0 first lets its issued copies land
    if (!__all_sync(kFullMask, mbar_wait(&full[s], ph, abort, Gm.timeout_ns))) {
      if (lane == 0) raise_flag(P.err, kFlagTimeout);
      if (threadIdx.x == 0) drain();
      return;
    }
    if (SCONV_PREFILL_FIRST_FILL > 0 && c == 0 && threadIdx.x == 0 && issued < min(NS, nchunks)) {
      // chunk 0 has landed: the rest of the ring
      for (; issued < min(NS, nchunks); ++issued) issue(issued, issued);
      if (issued == nchunks) trigger();
    }
    const int r0 = first_row + c * R;
    const int rows = min(R, tb - r0);
    if (c % (SW / R) == 0) {
      // rows [r0, r0 + SW): lane l writes row r0 + l's cache row offset
      // (-1, masked, for the rows of chunk 0 in front of ta)
      __syncwarp();
      // (rows past the range's end have slot -1: their stores are masked
      // here, so the fast path needs no row bound)
      const int64_t ro = (c == 0 && lane < *s_skip) ? -1 : slot_row_offset(P, next_slot, report_slots);
      warp_off[lane] = ro < 0 ? kNoRow : static_cast<uint32_t>(ro >> 3);
      __syncwarp();
      next_slot = load_slot(c / (SW / R) + 1);
    }
    const int sbase = (c % (SW / R)) * R;  // this chunk's first lane
    const unsigned char* stage = my_ring + static_cast<size_t>(s) * kTmaStageBytes;
    if (next >= r0 + rows && !skip) {
      // fast path: up to R tokens of one sequence, no branches (rows past
      // the end of the range compute on stale data and are not stored).
      // Where the unroll is shorter than a chunk, the tokens go in groups of
      // UF and a range's last, partial chunk skips the groups wholly past
      // its end (a short launch's ranges end in such a chunk).
      constexpr int UF = fast_unroll<W, MX, LV>();
      constexpr int NB = norm_batch<W, MX, LV, NBX>();
      static_assert(UF % NB == 0, "an unrolled group is a whole number of batches");
      if constexpr (UF < R) {
        static_assert(R % UF == 0, "a chunk is a whole number of groups");
        for (int rb = 0; rb < rows; rb += UF) {
#pragma unroll
          for (int u0 = 0; u0 < UF; u0 += NB) FAST_BATCH(rb + u0);
        }
      } else {
#pragma unroll
        for (int u0 = 0; u0 < R; u0 += NB) FAST_BATCH(u0);
      }
    } else {
      for (int r = 0; r < rows; ++r) {
        const int t = r0 + r;
        if (t >= next) {
          // a new sequence starts at t (skip empty ones)
          while (seq + 1 < S && cu(seq + 1) <= t) ++seq;
          next = (seq + 1 <= S) ? cu(seq + 1) : T;
          start_sequence(seq);
        }
        const uint4 xr = *reinterpret_cast<const uint4*>(stage + r * my_rs);
        float2 acc[4];
        conv_step<W>(tw, part, xr, acc);
        NORM_STORE(active && !skip ? warp_off[sbase + r] : kNoRow);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // stage fully consumed
    bool gave_up = false;
    if (threadIdx.x == 0 && c >= 1 && issued < nchunks) {
      // refill the stage of chunk c-1 (issued == c-1+NS lands there) once
      // every warp has released it
      const int sp = s == 0 ? NS - 1 : s - 1;
      const uint32_t pp = s == 0 ? ph ^ 1u : ph;
      if (mbar_wait(&empty[sp], pp, abort, Gm.timeout_ns)) {
        issue(issued++, sp);
        if (issued == nchunks) trigger();
      } else {
        gave_up = true;
      }
    }
    if (__any_sync(kFullMask, gave_up)) {  // warp 0 leaves together
      if (lane == 0) raise_flag(P.err, kFlagTimeout);
      if (threadIdx.x == 0) drain();
      return;
    }
    if (++s == NS) {
      s = 0;
      ph ^= 1;
    }
  }
#undef NORM_STORE
#undef SCALE_STORE
#undef FAST_BATCH
}

template <int W, int D, int MINB, bool MX, bool LV, int NBX = 0>
__global__ void __launch_bounds__(prefill_threads<W, MX>(), MINB)
    prefill_tma_kernel(const StepParams P, const TmaGeom Gm) {
  prefill_body<W, D, MX, LV, NBX>(P, Gm);
  // With the state-only dependency a CTA that never touched a state row has
  // not waited for the previous grid yet: it does before it exits, so this
  // grid's completion still implies its predecessor's.
  if (Gm.state_wait_only && threadIdx.x == 0) grid_dependency_wait();
}

}  // namespace sconv
