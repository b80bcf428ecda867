// Decode kernel instances: bf16 or MXFP8 cache store, without or with the
// layout variants.
#include "instances.h"

namespace sconv {

#define SCONV_DECODE_FOR(WW, DD) (&decode_tma_kernel<WW, DD, MX, LV>)

template <bool MX, bool LV>
DecFn pick_decode_t(int W, int D) { SCONV_PICK_BY_W_D(SCONV_DECODE_FOR) }

DecFn pick_decode(int W, int D, bool mx, bool lv) {
  if (mx) return lv ? pick_decode_t<true, true>(W, D) : pick_decode_t<true, false>(W, D);
  return lv ? pick_decode_t<false, true>(W, D) : pick_decode_t<false, false>(W, D);
}

}  // namespace sconv
