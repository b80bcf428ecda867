// Prefill kernel instances: bf16 cache store, with the layout variants.
#include "instances.h"

namespace sconv {

#define SCONV_PREFILL_FOR(WW, DD) (&prefill_tma_kernel<WW, DD, prefill_ctas_per_sm<WW, false>(), false, true>)

TmaFn pick_prefill_bf16_lv(int W, int D) { SCONV_PICK_BY_W_D(SCONV_PREFILL_FOR) }

}  // namespace sconv
