// Kernel instances of the fused step, picked by (W, head_dim) at run time.
// Each pick_* function is defined in its own translation unit (inst_*.cu),
// which instantiates the kernel templates for W in 1..8 and head_dim in
// {64, 128, 256}; the library's host code (sconv_kv.cu) only includes the
// templates' geometry types and never instantiates a kernel itself.
#pragma once
#include "common.cuh"
#include "decode_tma.cuh"
#include "prefill_tma.cuh"

namespace sconv {

using TmaFn = void (*)(StepParams, TmaGeom);
using DecFn = void (*)(StepParams, DecGeom);

// Persistent prefill CTAs per SM (prefill_ctas_per_sm<W, MX>() in
// prefill_tma.cuh): W <= 4 fits 128 registers, two CTAs per SM (twice the
// warps to hide latency); wider windows need more registers and run one CTA
// per SM.
inline int prefill_ctas_per_sm(int W, bool mx) {
  return W <= 4 ? (mx ? SCONV_PREFILL_MX_PER_SM : SCONV_PREFILL_SMALL_W_PER_SM) : 1;
}

// nullptr for an unsupported (W, D).
TmaFn pick_prefill_bf16(int W, int D);
TmaFn pick_prefill_mx(int W, int D);
TmaFn pick_prefill_bf16_lv(int W, int D);
// bf16 store, W <= 4, for short launches (SCONV_PREFILL_SHORT_CHUNKS in
// prefill_tma.cuh); nullptr for W > 4
TmaFn pick_prefill_bf16_short(int W, int D);
TmaFn pick_prefill_mx_lv(int W, int D);
DecFn pick_decode(int W, int D, bool mx, bool lv);

// Body of a pick function: the instance of KERNEL_FOR<W, D> for the run-time
// (W, D), or nullptr.
#define SCONV_PICK_BY_W_D(KERNEL_FOR)                                   \
  switch (D) {                                                         \
    case 64: return SCONV_PICK_W(KERNEL_FOR, 64);                      \
    case 128: return SCONV_PICK_W(KERNEL_FOR, 128);                    \
    case 256: return SCONV_PICK_W(KERNEL_FOR, 256);                    \
    default: return nullptr;                                           \
  }
#define SCONV_PICK_W(KERNEL_FOR, DD)                                           \
  (W == 1 ? KERNEL_FOR(1, DD) : W == 2 ? KERNEL_FOR(2, DD) : W == 3 ? KERNEL_FOR(3, DD) \
   : W == 4 ? KERNEL_FOR(4, DD) : W == 5 ? KERNEL_FOR(5, DD) : W == 6 ? KERNEL_FOR(6, DD) \
   : W == 7 ? KERNEL_FOR(7, DD) : W == 8 ? KERNEL_FOR(8, DD) : nullptr)

}  // namespace sconv
