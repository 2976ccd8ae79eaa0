// Instantiations of the rotate+quantize kernel for configuration 1
// (6144 < d <= 12288: 48 KB pair buffers, byte gather addresses), Block-RHT / Full RHT (no permutation).
#include "oq_rotq.cuh"

namespace oq {
namespace rotq {
OQ_ROTQ_DEFINE_PICK(pick_cfg1_np, 1, false)
}  // namespace rotq
}  // namespace oq
