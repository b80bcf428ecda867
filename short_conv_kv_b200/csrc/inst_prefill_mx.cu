// Prefill kernel instances: MXFP8 cache store, without the layout variants.
#include "instances.h"

namespace sconv {

#define SCONV_PREFILL_FOR(WW, DD) (&prefill_tma_kernel<WW, DD, prefill_ctas_per_sm<WW, true>(), true, false>)

TmaFn pick_prefill_mx(int W, int D) { SCONV_PICK_BY_W_D(SCONV_PREFILL_FOR) }

}  // namespace sconv
