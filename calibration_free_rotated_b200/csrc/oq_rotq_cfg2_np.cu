// Instantiations of the rotate+quantize kernel for configuration 2
// (12288 < d <= 16384: 64 KB pair buffers, word gather addresses), Block-RHT / Full RHT (no permutation).
#include "oq_rotq.cuh"

namespace oq {
namespace rotq {
OQ_ROTQ_DEFINE_PICK(pick_cfg2_np, 2, false)
}  // namespace rotq
}  // namespace oq
