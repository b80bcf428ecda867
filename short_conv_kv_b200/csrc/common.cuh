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
  int tile;  // tokens per CTA tile (prefill)
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
