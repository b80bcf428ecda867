// Fused ShortConv K/V step over a packed varlen batch (sm_100a).
//
// One CTA = one tile of `tile` consecutive tokens of ONE sequence x a span of
// 8-channel groups (256 groups = all 2*C channels of K and V when C = 1024).
// Thread g owns channels [8g', 8g'+8) of K (g < NG/2) or of V and walks the
// tile's tokens in order, keeping the last W-1 rows of its 8 channels in
// registers (fp32), so every input row is read from memory once by the tile
// and the W-1-row halo in front of the tile once more (an L2 hit: the
// neighbouring tile reads the same rows at about the same time).
//
// Per token: conv (W packed-fp32 FMAs per channel pair), sum of squares over
// the head (8 channels in-thread, then D/8 lanes by xor shuffles), one
// rsqrt, scale by gamma, round to bf16, one 16-byte store to the cache slot.
//
// Tiles never cross sequences.  Sequence i owns the virtual tiles
// [floor(cu[i]/tile) + i, floor(cu[i+1]/tile) + i + 1); that range is at
// least ceil(L_i/tile) long, so the grid is floor(T/tile) + S CTAs and at
// most one CTA per sequence finds no work.  The CTA holding positions
// [0, tile) of a sequence (tile >= W-1) is the only reader of the
// sequence's old conv_state, and it is also the one that writes the new
// state (re-reading the last W-1 rows of the sequence), so no other CTA can
// observe a half-updated state and no inter-CTA synchronisation is needed.
#pragma once
#include "common.cuh"

namespace sconv {

constexpr int kCuSmemMax = 2048;  // cu_seqlens entries staged in shared memory
constexpr int kChunk = 8;         // rows loaded per batch by each thread

__device__ __forceinline__ int64_t first_vtile(int cu_i, int i, int tile) {
  return static_cast<int64_t>(cu_i / tile) + i;
}

// Largest i in [0, S-1] with first_vtile(cu[i], i) <= vt.
template <typename Load>
__device__ __forceinline__ int find_seq(Load cu, int S, int tile, int64_t vt) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (first_vtile(cu(mid), mid, tile) <= vt)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

template <int W, int D>
__global__ void __launch_bounds__(256, (W <= 4 ? 2 : 1))
    prefill_kernel(const StepParams P) {
  __shared__ int s_cu[kCuSmemMax + 1];
  __shared__ int s_seq;
  constexpr int G = D / 8;  // lanes per head
  const int S = P.num_seqs;
  const int tile = P.tile;
  const int64_t vt = blockIdx.x;

  // ---- which sequence / tile is this CTA?
  int seq, a, b;
  if (S <= kCuSmemMax) {
    for (int i = threadIdx.x; i <= S; i += blockDim.x) s_cu[i] = P.cu_seqlens[i];
    __syncthreads();
    seq = find_seq([&](int i) { return s_cu[i]; }, S, tile, vt);
    a = s_cu[seq];
    b = s_cu[seq + 1];
  } else {
    if (threadIdx.x == 0)
      s_seq = find_seq([&](int i) { return P.cu_seqlens[i]; }, S, tile, vt);
    __syncthreads();
    seq = s_seq;
    a = P.cu_seqlens[seq];
    b = P.cu_seqlens[seq + 1];
  }
  if (vt == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    const int c_first = (S <= kCuSmemMax) ? s_cu[0] : P.cu_seqlens[0];
    const int c_last = (S <= kCuSmemMax) ? s_cu[S] : P.cu_seqlens[S];
    if (c_first != 0 || c_last != P.num_tokens) raise_flag(P.err, kFlagCuSeqlens);
  }
  if (a < 0 || b < a || b > P.num_tokens) {
    if (blockIdx.y == 0 && threadIdx.x == 0) raise_flag(P.err, kFlagCuSeqlens);
    return;
  }
  const int64_t L = b - a;
  const int64_t tl = vt - first_vtile(a, seq, tile);
  const int64_t p0 = tl * tile;  // first position of the tile in the sequence
  if (tl < 0 || p0 >= L) return;
  const int n = static_cast<int>(min(static_cast<int64_t>(tile), L - p0));

  // ---- this thread's 8 channels
  const int g_raw = blockIdx.y * blockDim.x + threadIdx.x;
  const bool active = g_raw < P.NG;
  const int g = active ? g_raw : 0;
  const int half = P.NG >> 1;
  const bool isv = g >= half;
  const int c0 = (isv ? g - half : g) * 8;
  const int d0 = c0 % D;
  const uint16_t* xs = (isv ? P.v : P.k) + c0 + static_cast<int64_t>(a) * P.row_stride;
  const uint16_t* w = (isv ? P.w_v : P.w_k) + c0;
  const float* gam = (isv ? P.gamma_v : P.gamma_k) + d0;
  uint16_t* cache = (isv ? P.v_cache : P.k_cache) + (c0 / D) * P.stride_head + d0;
  const int lane = threadIdx.x & 31;

  // ---- conv_state of the sequence (validated before any access)
  uint16_t* st = nullptr;
  if constexpr (W > 1) {
    const int64_t si = P.state_indices ? static_cast<int64_t>(P.state_indices[seq]) : seq;
    if (si < 0 || si >= P.pool) {
      if (tl == 0 && blockIdx.y == 0 && threadIdx.x == 0) raise_flag(P.err, kFlagStateIndex);
      return;
    }
    st = P.state + si * (W - 1) * 2 * static_cast<int64_t>(P.C) + (isv ? P.C : 0) + c0;
  }

  // ---- taps and gamma
  float2 tw[W][4];
#pragma unroll
  for (int j = 0; j < W; ++j) unpack8(ld_ro(w + static_cast<int64_t>(j) * P.C), tw[j]);
  float2 gm[4];
  {
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(gam));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(gam) + 1);
    gm[0] = make_float2(g0.x, g0.y);
    gm[1] = make_float2(g0.z, g0.w);
    gm[2] = make_float2(g1.x, g1.y);
    gm[3] = make_float2(g1.z, g1.w);
  }

  // ---- halo: the W-1 rows before the tile (old state rows when p < 0)
  constexpr int NH = W > 1 ? W - 1 : 1;
  float2 win[NH][4];
  if constexpr (W > 1) {
    const int64_t srow = 2 * static_cast<int64_t>(P.C);
    uint4 hb[W - 1];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
      const int64_t q = p0 - (W - 1) + j;
      if (!active)
        hb[j] = make_uint4(0, 0, 0, 0);
      else if (q >= 0)
        hb[j] = ld_ro(xs + q * P.row_stride);
      else
        hb[j] = *reinterpret_cast<const uint4*>(st + (W - 1 + q) * srow);
    }
    if (p0 == 0 && active) {
      // New state row j = row L-(W-1)+j of (old state ++ sequence).  The old
      // rows this CTA needs are already in registers, so the overwrite is
      // safe (same thread, same addresses, program order).
#pragma unroll
      for (int j = 0; j < W - 1; ++j) {
        const int64_t q = L - (W - 1) + j;
        uint4 r;
        if (q >= 0) {
          r = ld_ro(xs + q * P.row_stride);
        } else {
          r = hb[0];
#pragma unroll
          for (int m = 1; m < W - 1; ++m)
            if (m == W - 1 + q) r = hb[m];
        }
        *reinterpret_cast<uint4*>(st + j * srow) = r;
      }
    }
#pragma unroll
    for (int j = 0; j < W - 1; ++j) unpack8(hb[j], win[j]);
  }

  // ---- walk the tile
  const float eps = P.eps;
  const float inv_d = P.inv_d;
  const uint16_t* xp = xs + p0 * P.row_stride;
  const int64_t* sl = P.slots + a + p0;
  const bool report = blockIdx.y == 0 && threadIdx.x < 32;
  for (int t0 = 0; t0 < n; t0 += 32) {
    const int cnt = min(32, n - t0);
    long long my_off = -1;
    if (lane < cnt) my_off = slot_row_offset(P, sl[t0 + lane], report);
    for (int u0 = 0; u0 < cnt; u0 += kChunk) {
      uint4 xr[kChunk];
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        if (active && u0 + u < cnt)
          xr[u] = ld_ro(xp + static_cast<int64_t>(t0 + u0 + u) * P.row_stride);
        else
          xr[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        float2 xf[4];
        unpack8(xr[u], xf);
        float2 acc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (W == 1) {
            acc[e] = fmul2(tw[0][e], xf[e]);
          } else {
            acc[e] = fmul2(tw[0][e], win[0][e]);
#pragma unroll
            for (int j = 1; j < W - 1; ++j) acc[e] = ffma2(tw[j][e], win[j][e], acc[e]);
            acc[e] = ffma2(tw[W - 1][e], xf[e], acc[e]);
          }
        }
        if constexpr (W > 1) {
#pragma unroll
          for (int j = 0; j < W - 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) win[j][e] = win[j + 1][e];
#pragma unroll
          for (int e = 0; e < 4; ++e) win[W - 2][e] = xf[e];
        }
        float2 s2 = fmul2(acc[0], acc[0]);
        s2 = ffma2(acc[1], acc[1], s2);
        s2 = ffma2(acc[2], acc[2], s2);
        s2 = ffma2(acc[3], acc[3], s2);
        const float ss = group_sum<G>(s2.x + s2.y);
        const float r = rsqrtf(fmaf(ss, inv_d, eps));
        const long long off = __shfl_sync(kFullMask, my_off, u0 + u);
        if (active && off >= 0 && u0 + u < cnt) {
          const float2 rr = make_float2(r, r);
          uint4 o;
          o.x = pack_bf16x2(fmul2(fmul2(acc[0], rr), gm[0]));
          o.y = pack_bf16x2(fmul2(fmul2(acc[1], rr), gm[1]));
          o.z = pack_bf16x2(fmul2(fmul2(acc[2], rr), gm[2]));
          o.w = pack_bf16x2(fmul2(fmul2(acc[3], rr), gm[3]));
          st_stream(cache + off, o);
        }
      }
    }
  }
}

}  // namespace sconv
