// Instantiations of the rotate+quantize kernel for configuration 0
// (P*d <= 6144: 24 KB pair buffers, byte gather addresses), RPBH (with the permutation).
#include "oq_rotq.cuh"

namespace oq {
namespace rotq {
OQ_ROTQ_DEFINE_PICK(pick_cfg0, 0, true)
}  // namespace rotq
}  // namespace oq
