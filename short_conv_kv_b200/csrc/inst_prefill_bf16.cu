// Prefill kernel instances: bf16 cache store, without the layout variants.
#include "instances.h"

namespace sconv {

#define SCONV_PREFILL_FOR(WW, DD) (&prefill_tma_kernel<WW, DD, prefill_ctas_per_sm<WW, false>(), false, false>)

TmaFn pick_prefill_bf16(int W, int D) { SCONV_PICK_BY_W_D(SCONV_PREFILL_FOR) }

}  // namespace sconv
