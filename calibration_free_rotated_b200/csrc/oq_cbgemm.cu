// Kernel 2 placeholder: the codebook GEMM is added in its own change.
#include "oq_internal.h"

namespace oq {
int launch_cbgemm(int, oq_codebook_t, oq_codebook_t, const uint8_t*, const float*, int, const uint8_t*,
                  const uint16_t*, int, const uint16_t*, int, float*, uint16_t*, void*) {
  return fail(OQ_ERR_UNSUPPORTED, "codebook GEMM not built yet");
}
}  // namespace oq
