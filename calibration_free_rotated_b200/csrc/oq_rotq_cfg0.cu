// Instantiations of the rotate+quantize kernel for configuration 0
// (P*d <= 6144: 24 KB pair buffers, byte gather addresses).
#include "oq_rotq.cuh"

namespace oq {
namespace rotq {
OQ_ROTQ_DEFINE_PICK(0)
}  // namespace rotq
}  // namespace oq
