// Device helpers shared by the fused ShortConv K/V kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sconv {

constexpr unsigned kFullMask = 0xffffffffu;

// Arguments of one launch, passed by value (lives in the constant bank).
struct StepParams {
  const uint16_t* k;  // bf16 rows, row_stride apart
  const uint16_t* v;
  int64_t row_stride;  // elements
  int64_t num_tokens;
  const int32_t* cu_seqlens;  // prefill only
  int num_seqs;               // prefill: sequences; decode: batch
  const uint16_t* w_k;        // bf16 [W, C]
  const uint16_t* w_v;
  const float* gamma_k;  // fp32 [D]
  const float* gamma_v;
  float eps;
  float inv_d;      // 1 / head_dim
  int C;            // Hkv * D (channels of K, equally of V)
  int NG;           // groups of 8 channels over K and V = 2C / 8
  uint16_t* state;  // bf16 [pool, W-1, 2C]
  const int32_t* state_indices;
  int64_t pool;
  const int64_t* slots;
  uint16_t* k_cache;
  uint16_t* v_cache;
  int64_t num_slots;
  int64_t page_size;
  int64_t stride_page;
  int64_t stride_slot;
  int64_t stride_head;
  int slot_linear;  // stride_page == page_size * stride_slot
  int* err;
  int tile;  // unused
  // MXFP8 store (block-scaled): E4M3 data caches (uint8, same element
  // offsets as the bf16 caches) and E8M0 scale caches (one byte per 32
  // channels: element offset / 32)
  uint8_t* k_data;
  uint8_t* v_data;
  uint8_t* k_scale;
  uint8_t* v_scale;
  // layout variants: elements between heads' gammas (0 = one gamma [D]
  // shared by all heads), and the ring-buffer state's positions (nullptr =
  // linear state, oldest row first; else the raw row of position p of
  // sequence i lives in state row p mod (W-1), and state_pos[i] is the
  // number of tokens the sequence has seen before this call)
  int64_t gamma_hs;
  const int64_t* state_pos;
};

// Flag bits (same values as the public SCONV_KV_FLAG_*).
constexpr int kFlagSlotRange = 1;
constexpr int kFlagStateIndex = 2;
constexpr int kFlagCuSeqlens = 4;
constexpr int kFlagTimeout = 8;

__device__ __forceinline__ void raise_flag(int* err, int bit) {
  if (err) atomicOr(err, bit);
}

// bf16 pair (low element first in memory) -> two fp32.  Widening bf16 is a
// 16-bit shift of the bit pattern.
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

__device__ __forceinline__ void unpack8(const uint4& u, float2 (&f)[4]) {
  f[0] = unpack_bf16x2(u.x);
  f[1] = unpack_bf16x2(u.y);
  f[2] = unpack_bf16x2(u.z);
  f[3] = unpack_bf16x2(u.w);
}

// Two fp32 -> bf16 pair, round to nearest even (low element = f.x).
__device__ __forceinline__ uint32_t pack_bf16x2(float2 f) {
  __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Read-only streaming load of 16 bytes (k / v rows, taps): non-coherent path.
__device__ __forceinline__ uint4 ld_ro(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Streaming 16-byte store of a cache row segment (not re-read by this kernel).
__device__ __forceinline__ void st_stream(uint16_t* p, const uint4& v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}

// The same store under a predicate, as one predicated instruction (no
// branch around it).
__device__ __forceinline__ void st_stream_if(bool pred, uint16_t* p, const uint4& v) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %0, 0;\n\t"
      "@q st.global.cs.v4.u32 [%1], {%2, %3, %4, %5};\n\t}" ::"r"(static_cast<int>(pred)),
      "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
      : "memory");
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  return __ffma2_rn(a, b, c);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  return __fmul2_rn(a, b);
}

// Element offset of the start of cache row `slot` (head 0, dim 0), or -1
// when the token is not written.  Sets the slot-range flag when asked.
__device__ __forceinline__ int64_t slot_row_offset(const StepParams& P,
                                                   int64_t slot,
                                                   bool report) {
  if (slot < 0) return -1;
  if (slot >= P.num_slots) {
    if (report) raise_flag(P.err, kFlagSlotRange);
    return -1;
  }
  if (P.slot_linear) return slot * P.stride_slot;
  const int64_t page = slot / P.page_size;
  return page * P.stride_page + (slot - page * P.page_size) * P.stride_slot;
}

// ---- MXFP8 (OCP Microscaling) block store: 32 channels = 4 lanes x 8.

// E8M0 scale byte (s + 127) of a block whose largest magnitude is
// `amax` (binary32, >= 0): the shared exponent s is floor(log2(amax)) - 8,
// the 8 being the exponent of E4M3's largest normal (448 = 1.75 * 2^8),
// and blocks whose amax is zero or subnormal take -127.  With e the biased
// exponent of amax (its sign bit is clear), floor(log2(amax)) = e - 127
// for a normal amax, so s + 127 = max(e - 8, 0) covers every case.
__device__ __forceinline__ uint32_t mx_scale_byte(float amax) {
  return static_cast<uint32_t>(max(static_cast<int>(__float_as_uint(amax) >> 23) - 8, 0));
}
// 2^-s from the scale byte s + 127: biased exponent 254 - (s + 127).
__device__ __forceinline__ float mx_inv_scale(uint32_t scale_byte) {
  return __uint_as_float((254u - scale_byte) << 23);
}
// max(|a|, |b|, |c|) in one instruction (sm_100: three-input max with the
// absolute-value modifier).
__device__ __forceinline__ float max_abs3(float a, float b, float c) {
  float r;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Two binary32 -> two E4M3 codes (nearest even, saturating), low element
// in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  unsigned short h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
  return h;
}

// Quantise this lane's 8 normalised values z = t * r (t = conv output times
// gamma, r = the head's 1/rms; channels d0..d0+7 of a head) as part of their
// 32-channel block: the 8 E4M3 codes (w0: channels 0-3, w1: 4-7, low
// element in the low byte) and the block's E8M0 scale byte sb.  z is formed
// first and then scaled by the exact power of two 2^-s (<= 2^127, and
// |z| * 2^-s < 512, so nothing overflows; folding 2^-s into r instead would
// overflow for all-zero blocks).  All 32 lanes of the warp must call it
// (shuffles over each block's 4 lanes).
__device__ __forceinline__ void mx_encode8(const float2 (&t)[4], float r, uint32_t& w0,
                                           uint32_t& w1, uint32_t& sb) {
  const float2 rr = make_float2(r, r);
  const float2 z[4] = {__fmul2_rn(t[0], rr), __fmul2_rn(t[1], rr), __fmul2_rn(t[2], rr),
                       __fmul2_rn(t[3], rr)};
  const float m0 = max_abs3(z[0].x, z[0].y, z[1].x);
  const float m1 = max_abs3(z[1].y, z[2].x, z[2].y);
  float amax = fmaxf(m1, max_abs3(z[3].x, z[3].y, m0));
  amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 2));
  sb = mx_scale_byte(amax);
  const float m = mx_inv_scale(sb);  // 2^-s, exact
  const float2 mm = make_float2(m, m);
  const float2 a = __fmul2_rn(z[0], mm), b = __fmul2_rn(z[1], mm);
  const float2 c = __fmul2_rn(z[2], mm), d = __fmul2_rn(z[3], mm);
  w0 = e4m3x2(a.x, a.y) | (e4m3x2(b.x, b.y) << 16);
  w1 = e4m3x2(c.x, c.y) | (e4m3x2(d.x, d.y) << 16);
}

// mx_encode8, then the store: 8 code bytes at `data`, and (lane % 4 == 0
// of the block's 4 lanes) the scale byte at `scale`; `write` masks both.
__device__ __forceinline__ void mx_store8(const float2 (&t)[4], float r, bool write,
                                          uint8_t* data, uint8_t* scale) {
  uint32_t w0, w1, sb;
  mx_encode8(t, r, w0, w1, sb);
  const bool scale_writer = write && ((threadIdx.x & 3) == 0);
  asm volatile(
      "{\n\t.reg .pred q, r;\n\t"
      "setp.ne.b32 q, %0, 0;\n\t"
      "setp.ne.b32 r, %1, 0;\n\t"
      "@q st.global.cs.v2.u32 [%2], {%3, %4};\n\t"
      "@r st.global.cs.u8 [%5], %6;\n\t}" ::"r"(static_cast<int>(write)),
      "r"(static_cast<int>(scale_writer)), "l"(data), "r"(w0), "r"(w1), "l"(scale), "r"(sb)
      : "memory");
}

// Row stores addressed by a cache row offset in units of 8 elements
// (`off8`; 0xFFFFFFFF: the row is not written, and the store is skipped).
// bf16: the 16 bytes at base + off8 * 16.
__device__ __forceinline__ void st_row_bf16(uint32_t off8, uint16_t* base, const uint4& v) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t.reg .u64 a;\n\t"
      "setp.ne.u32 q, %0, -1;\n\t"
      "mad.wide.u32 a, %0, 16, %1;\n\t"
      "@q st.global.cs.v4.u32 [a], {%2, %3, %4, %5};\n\t}" ::"r"(off8),
      "l"(base), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
      : "memory");
}
// MXFP8: the 8 code bytes at data + off8 * 8 and, where scale_lane is
// nonzero, the scale byte at scale + off8 / 4.
__device__ __forceinline__ void st_row_mx(uint32_t off8, uint8_t* data, uint8_t* scale,
                                          int scale_lane, uint32_t w0, uint32_t w1, uint32_t sb) {
  asm volatile(
      "{\n\t.reg .pred q, r;\n\t.reg .u32 o;\n\t.reg .u64 a, b;\n\t"
      "setp.ne.u32 q, %0, -1;\n\t"
      "setp.ne.and.b32 r, %1, 0, q;\n\t"
      "mad.wide.u32 a, %0, 8, %2;\n\t"
      "shr.u32 o, %0, 2;\n\t"
      "mad.wide.u32 b, o, 1, %3;\n\t"
      "@q st.global.cs.v2.u32 [a], {%4, %5};\n\t"
      "@r st.global.cs.u8 [b], %6;\n\t}" ::"r"(off8),
      "r"(scale_lane), "l"(data), "l"(scale), "r"(w0), "r"(w1), "r"(sb)
      : "memory");
}

// Hardware reciprocal square root (PTX rsqrt.approx.ftz.f32, one MUFU op;
// relative error about 2^-22).  Callers pass x >= eps > 0, so the
// flush-to-zero and special-value behaviour never matters.
__device__ __forceinline__ float rsqrt_approx(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Sum of `v` over aligned groups of G lanes (G = D/8 lanes own one head).
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int m = G / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(kFullMask, v, m);
  return v;
}

}  // namespace sconv
