// Fused ShortConv K/V decode step: one new token per sequence (sm_100a).
//
// One CTA = one sequence x a span of 8-channel groups.  Thread g loads the
// W-1 state rows and the new row of its 8 channels (all independent 16-byte
// loads, issued together), convolves, reduces the head's sum of squares by
// xor shuffles over D/8 lanes, writes the normalised bf16 row to the cache
// slot and rewrites its state rows shifted by one (oldest dropped, new row
// appended).  The state rows it overwrites are exactly the ones it read, so
// the in-place update needs no synchronisation.
#pragma once
#include "common.cuh"

namespace sconv {

template <int W, int D>
__global__ void __launch_bounds__(256) decode_kernel(const StepParams P) {
  constexpr int G = D / 8;
  const int64_t bseq = blockIdx.x;
  const int g_raw = blockIdx.y * blockDim.x + threadIdx.x;
  const bool active = g_raw < P.NG;
  const int g = active ? g_raw : 0;
  const int half = P.NG >> 1;
  const bool isv = g >= half;
  const int c0 = (isv ? g - half : g) * 8;
  const int d0 = c0 % D;

  uint16_t* st = nullptr;
  const int64_t srow = 2 * static_cast<int64_t>(P.C);
  if constexpr (W > 1) {
    const int64_t si = P.state_indices ? static_cast<int64_t>(P.state_indices[bseq]) : bseq;
    if (si < 0 || si >= P.pool) {
      if (blockIdx.y == 0 && threadIdx.x == 0) raise_flag(P.err, kFlagStateIndex);
      return;
    }
    st = P.state + si * (W - 1) * srow + (isv ? P.C : 0) + c0;
  }
  const int64_t off =
      slot_row_offset(P, P.slots[bseq], blockIdx.y == 0 && threadIdx.x == 0);

  // independent loads first: state rows, new row, taps, gamma
  constexpr int NH = W > 1 ? W - 1 : 1;
  uint4 hb[NH];
  uint4 xr = make_uint4(0, 0, 0, 0);
  if (active) {
    if constexpr (W > 1) {
#pragma unroll
      for (int j = 0; j < W - 1; ++j) hb[j] = *reinterpret_cast<const uint4*>(st + j * srow);
    }
    xr = ld_ro((isv ? P.v : P.k) + bseq * P.row_stride + c0);
  } else {
#pragma unroll
    for (int j = 0; j < NH; ++j) hb[j] = make_uint4(0, 0, 0, 0);
  }
  const uint16_t* w = (isv ? P.w_v : P.w_k) + c0;
  float2 tw[W][4];
#pragma unroll
  for (int j = 0; j < W; ++j) unpack8(ld_ro(w + static_cast<int64_t>(j) * P.C), tw[j]);
  const float* gam = (isv ? P.gamma_v : P.gamma_k) + d0;
  const float4 g0 = __ldg(reinterpret_cast<const float4*>(gam));
  const float4 g1 = __ldg(reinterpret_cast<const float4*>(gam) + 1);

  // conv: y = sum_j w[j] * row[j], rows oldest first, new row last
  float2 xf[4];
  unpack8(xr, xf);
  float2 acc[4];
  if constexpr (W == 1) {
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = fmul2(tw[0][e], xf[e]);
  } else {
    float2 hf[4];
    unpack8(hb[0], hf);
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = fmul2(tw[0][e], hf[e]);
#pragma unroll
    for (int j = 1; j < W - 1; ++j) {
      unpack8(hb[j], hf);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = ffma2(tw[j][e], hf[e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = ffma2(tw[W - 1][e], xf[e], acc[e]);
  }

  // RMSNorm over the head
  float2 s2 = fmul2(acc[0], acc[0]);
  s2 = ffma2(acc[1], acc[1], s2);
  s2 = ffma2(acc[2], acc[2], s2);
  s2 = ffma2(acc[3], acc[3], s2);
  const float ss = group_sum<G>(s2.x + s2.y);
  const float r = rsqrtf(fmaf(ss, P.inv_d, P.eps));
  if (!active) return;

  if (off >= 0) {
    const float2 rr = make_float2(r, r);
    uint4 o;
    o.x = pack_bf16x2(fmul2(fmul2(acc[0], rr), make_float2(g0.x, g0.y)));
    o.y = pack_bf16x2(fmul2(fmul2(acc[1], rr), make_float2(g0.z, g0.w)));
    o.z = pack_bf16x2(fmul2(fmul2(acc[2], rr), make_float2(g1.x, g1.y)));
    o.w = pack_bf16x2(fmul2(fmul2(acc[3], rr), make_float2(g1.z, g1.w)));
    uint16_t* cache = (isv ? P.v_cache : P.k_cache) + off + (c0 / D) * P.stride_head + d0;
    st_stream(cache, o);
  }
  if constexpr (W > 1) {
#pragma unroll
    for (int j = 0; j < W - 2; ++j) *reinterpret_cast<uint4*>(st + j * srow) = hb[j + 1];
    *reinterpret_cast<uint4*>(st + (W - 2) * srow) = xr;
  }
}

}  // namespace sconv
