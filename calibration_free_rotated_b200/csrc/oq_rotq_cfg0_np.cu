// Instantiations of the rotate+quantize kernel for configuration 0
// (P*d <= 6144: 24 KB pair buffers, byte gather addresses), Block-RHT / Full RHT (no permutation).
#include "oq_rotq.cuh"

namespace oq {
namespace rotq {
OQ_ROTQ_DEFINE_PICK(pick_cfg0_np, 0, false)
}  // namespace rotq
}  // namespace oq
