// The ShortConv K/V step as separate passes over HBM (sm_100a): causal conv,
// per-head RMSNorm, paged cache scatter and conv_state update, each its own
// kernel with its intermediate stored in bf16.  This is the unfused chain
// that the fused kernels replace ("SGLang and Miles announce day-0 Inkling
// support", aib.vote English news item, paragraph 2); each stage is also
// usable on its own.
//
// Every kernel is a plain grid-stride loop in which one thread handles one
// group of 8 channels (16 bytes) of one token row.  Each waits for the
// previous kernel in the stream before touching global memory (the chain
// is launched with programmatic dependent launch).
#pragma once
#include "common.cuh"
#include "tma.cuh"

namespace sconv {

// Arguments of the stage kernels (passed by value).
struct StageParams {
  const uint16_t* k;  // bf16 [T, C] rows, row_stride apart
  const uint16_t* v;
  int64_t row_stride;
  int64_t num_tokens;
  const int32_t* cu_seqlens;
  int num_seqs;
  const uint16_t* w_k;  // bf16 [W, C]
  const uint16_t* w_v;
  const float* gamma_k;  // fp32 [D]
  const float* gamma_v;
  float eps;
  float inv_d;
  int C;   // channels of K (= of V)
  int D;   // head_dim
  int NG;  // groups of 8 channels over K and V (2C / 8)
  int W;   // conv width
  uint16_t* state;  // bf16 [pool, W-1, 2C]
  const int32_t* state_indices;
  int64_t pool;
  uint16_t* y;  // bf16 [T, 2C] conv output (K channels, then V)
  uint16_t* z;  // bf16 [T, 2C] normalised values
  const int64_t* slots;
  uint16_t* k_cache;
  uint16_t* v_cache;
  int64_t num_slots;
  int64_t page_size;
  int64_t stride_page;
  int64_t stride_slot;
  int64_t stride_head;
  int* err;
};

// Sequence of packed token t: largest i in [0, S-1] with cu[i] <= t.
__device__ __forceinline__ int stage_seq_of(const int32_t* cu, int S, int64_t t) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// State row of sequence i (or -1 after flagging a bad index).
__device__ __forceinline__ int64_t stage_state_index(const StageParams& P, int i) {
  const int64_t si = P.state_indices ? static_cast<int64_t>(__ldg(P.state_indices + i)) : i;
  if (si < 0 || si >= P.pool) {
    raise_flag(P.err, kFlagStateIndex);
    return -1;
  }
  return si;
}

// Pass 1: y[t] = sum_j w[j] * x[t - W + 1 + j] (rows before the sequence
// from its old state), rounded to bf16.  The state is only read here.
template <int W>
__global__ void __launch_bounds__(256) stage_conv_kernel(const StageParams P) {
  grid_dependency_wait();
  const int64_t total = P.num_tokens * P.NG;
  const int half = P.NG >> 1;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / P.NG;
    const int g = static_cast<int>(idx - t * P.NG);
    const bool isv = g >= half;
    const int c0 = (isv ? g - half : g) * 8;
    const int i = stage_seq_of(P.cu_seqlens, P.num_seqs, t);
    const int64_t a = __ldg(P.cu_seqlens + i);
    if (!(a >= 0 && a <= t && t < __ldg(P.cu_seqlens + i + 1))) {  // malformed cu_seqlens
      raise_flag(P.err, kFlagCuSeqlens);
      continue;
    }
    const int64_t p = t - a;  // position in the sequence
    int64_t si = 0;
    if (W > 1 && p < W - 1) {
      si = stage_state_index(P, i);
      if (si < 0) continue;
    }
    const uint16_t* x = (isv ? P.v : P.k) + c0;
    const uint16_t* w = (isv ? P.w_v : P.w_k) + c0;
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                     make_float2(0.f, 0.f)};
#pragma unroll
    for (int j = 0; j < W; ++j) {
      const int64_t q = p - (W - 1) + j;
      uint4 r;
      if (q >= 0) {
        r = ld_ro(x + (a + q) * P.row_stride);
      } else {
        r = *reinterpret_cast<const uint4*>(P.state + (si * (W - 1) + (W - 1 + q)) * 2 * P.C +
                                            (isv ? P.C : 0) + c0);
      }
      float2 xf[4], wf[4];
      unpack8(r, xf);
      unpack8(ld_ro(w + static_cast<int64_t>(j) * P.C), wf);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = ffma2(wf[e], xf[e], acc[e]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0]);
    o.y = pack_bf16x2(acc[1]);
    o.z = pack_bf16x2(acc[2]);
    o.w = pack_bf16x2(acc[3]);
    st_stream(P.y + t * 2 * P.C + static_cast<int64_t>(g) * 8, o);
  }
}

// Pass 2: z = y / sqrt(mean_d y^2 + eps) * gamma per head, rounded to bf16.
// A head's D channels are D/8 consecutive lanes; every lane of a warp takes
// part in the shuffles (the thread count per row, 2C/8, is a multiple of
// D/8, and idx runs in whole warps).
template <int D>
__global__ void __launch_bounds__(256) stage_rmsnorm_kernel(const StageParams P) {
  grid_dependency_wait();
  const int64_t total = P.num_tokens * P.NG;
  const int half = P.NG >> 1;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t start = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  // iterate in whole warps so the shuffles see full groups
  const int64_t warp_total = ((total + 31) / 32) * 32;
  for (int64_t idx = start; idx < warp_total; idx += stride) {
    const bool valid = idx < total;
    const int64_t t = valid ? idx / P.NG : 0;
    const int g = valid ? static_cast<int>(idx - t * P.NG) : 0;
    const bool isv = g >= half;
    const int c0 = (isv ? g - half : g) * 8;
    const int d0 = c0 % D;
    float2 yf[4];
    unpack8(valid ? *reinterpret_cast<const uint4*>(P.y + t * 2 * P.C + static_cast<int64_t>(g) * 8)
                  : make_uint4(0, 0, 0, 0),
            yf);
    float2 s2 = fmul2(yf[0], yf[0]);
    s2 = ffma2(yf[1], yf[1], s2);
    s2 = ffma2(yf[2], yf[2], s2);
    s2 = ffma2(yf[3], yf[3], s2);
    const float ss = group_sum<D / 8>(s2.x + s2.y);
    const float rn = rsqrt_approx(fmaf(ss, P.inv_d, P.eps));
    if (!valid) continue;
    const float* gam = (isv ? P.gamma_v : P.gamma_k) + d0;
    const float4 ga = __ldg(reinterpret_cast<const float4*>(gam));
    const float4 gb = __ldg(reinterpret_cast<const float4*>(gam) + 1);
    const float2 rr = make_float2(rn, rn);
    uint4 o;
    o.x = pack_bf16x2(fmul2(fmul2(yf[0], rr), make_float2(ga.x, ga.y)));
    o.y = pack_bf16x2(fmul2(fmul2(yf[1], rr), make_float2(ga.z, ga.w)));
    o.z = pack_bf16x2(fmul2(fmul2(yf[2], rr), make_float2(gb.x, gb.y)));
    o.w = pack_bf16x2(fmul2(fmul2(yf[3], rr), make_float2(gb.z, gb.w)));
    st_stream(P.z + t * 2 * P.C + static_cast<int64_t>(g) * 8, o);
  }
}

// Pass 3: cache[slot_mapping[t]] = z[t] (K half into k_cache, V half into
// v_cache); slot < 0 skips the token, slot >= num_slots is flagged.  When
// cu_seqlens is given, the tokens of a sequence that the fused step would
// skip (malformed cu_seqlens entry; for W > 1 a state index outside the
// pool) are not written either, so the chain leaves the same cache slots
// untouched as the fused kernels (the conv and state passes raise the
// flags).
__global__ void __launch_bounds__(256) stage_scatter_kernel(const StageParams P) {
  grid_dependency_wait();
  const int64_t total = P.num_tokens * P.NG;
  const int half = P.NG >> 1;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / P.NG;
    const int g = static_cast<int>(idx - t * P.NG);
    const int64_t slot = __ldg(P.slots + t);
    if (slot < 0) continue;
    if (P.cu_seqlens) {
      const int i = stage_seq_of(P.cu_seqlens, P.num_seqs, t);
      const int64_t a = __ldg(P.cu_seqlens + i), e = __ldg(P.cu_seqlens + i + 1);
      if (!(a >= 0 && a <= t && t < e && e <= P.num_tokens)) continue;
      if (P.W > 1) {
        const int64_t si =
            P.state_indices ? static_cast<int64_t>(__ldg(P.state_indices + i)) : i;
        if (si < 0 || si >= P.pool) continue;
      }
    }
    if (slot >= P.num_slots) {
      if (g == 0) raise_flag(P.err, kFlagSlotRange);
      continue;
    }
    const bool isv = g >= half;
    const int c0 = (isv ? g - half : g) * 8;
    const int64_t page = slot / P.page_size;
    const int64_t off = page * P.stride_page + (slot - page * P.page_size) * P.stride_slot +
                        (c0 / P.D) * P.stride_head + c0 % P.D;
    const uint4 zv =
        *reinterpret_cast<const uint4*>(P.z + t * 2 * P.C + static_cast<int64_t>(g) * 8);
    st_stream((isv ? P.v_cache : P.k_cache) + off, zv);
  }
}

// Pass 4: each sequence's new state = the last W-1 raw rows of (old state ++
// its rows).  One thread owns one 8-channel column of one sequence and reads
// every source row before writing, so the in-place update never reads a
// row it has already overwritten.
template <int W>
__global__ void __launch_bounds__(256) stage_state_kernel(const StageParams P) {
  grid_dependency_wait();
  const int64_t total = static_cast<int64_t>(P.num_seqs) * P.NG;
  const int half = P.NG >> 1;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx / P.NG);
    const int g = static_cast<int>(idx - static_cast<int64_t>(i) * P.NG);
    const int64_t a = __ldg(P.cu_seqlens + i), e = __ldg(P.cu_seqlens + i + 1);
    if (!(a >= 0 && a <= e && e <= P.num_tokens)) {  // malformed cu_seqlens
      raise_flag(P.err, kFlagCuSeqlens);
      continue;
    }
    const int64_t L = e - a;
    if (L == 0) continue;  // no rows: the state is unchanged
    const int64_t si = stage_state_index(P, i);
    if (si < 0) continue;
    const bool isv = g >= half;
    const int c0 = (isv ? g - half : g) * 8;
    uint16_t* st = P.state + si * (W - 1) * 2 * P.C + (isv ? P.C : 0) + c0;
    const uint16_t* x = (isv ? P.v : P.k) + c0;
    uint4 old[W - 1], nw[W - 1];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) old[j] = *reinterpret_cast<const uint4*>(st + j * 2 * P.C);
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
      const int64_t q = L - (W - 1) + j;  // row of (old state ++ sequence)
      if (q >= 0) {
        nw[j] = ld_ro(x + (a + q) * P.row_stride);
      } else {
        nw[j] = old[0];
#pragma unroll
        for (int m = 1; m < W - 1; ++m)
          if (m == W - 1 + q) nw[j] = old[m];
      }
    }
#pragma unroll
    for (int j = 0; j < W - 1; ++j) *reinterpret_cast<uint4*>(st + j * 2 * P.C) = nw[j];
  }
}

}  // namespace sconv
