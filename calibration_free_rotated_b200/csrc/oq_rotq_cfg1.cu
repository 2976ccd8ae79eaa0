// Instantiations of the rotate+quantize kernel for configuration 1
// (6144 < d <= 12288: 48 KB pair buffers, byte gather addresses).
#include "oq_rotq.cuh"

namespace oq {
namespace rotq {
OQ_ROTQ_DEFINE_PICK(1)
}  // namespace rotq
}  // namespace oq
