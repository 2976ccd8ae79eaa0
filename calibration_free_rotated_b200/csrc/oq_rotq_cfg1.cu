// Instantiations of the rotate+quantize kernel for configuration 1
// (6144 < d <= 12288: 48 KB pair buffers, byte gather addresses), RPBH (with the permutation).
#include "oq_rotq.cuh"

namespace oq {
namespace rotq {
OQ_ROTQ_DEFINE_PICK(pick_cfg1, 1, true)
}  // namespace rotq
}  // namespace oq
