// Prefill kernel instances for short launches: bf16 cache store, W <= 4,
// head reductions batched SCONV_PREFILL_SHORT_NORM_BATCH tokens at a time.
#include "instances.h"

namespace sconv {

#define SCONV_PREFILL_SHORT_FOR(WW, DD)                                                   \
  ((WW) <= 4 ? &prefill_tma_kernel<((WW) <= 4 ? (WW) : 4), DD,                            \
                                   prefill_ctas_per_sm<((WW) <= 4 ? (WW) : 4), false>(),  \
                                   false, false, SCONV_PREFILL_SHORT_NORM_BATCH>          \
             : nullptr)

TmaFn pick_prefill_bf16_short(int W, int D) { SCONV_PICK_BY_W_D(SCONV_PREFILL_SHORT_FOR) }

}  // namespace sconv
