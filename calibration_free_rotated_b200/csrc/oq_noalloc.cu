// oq_linear_noalloc: the full layer (oq_linear) for callers that cannot
// allocate device memory, with its scratch in a fixed static device array.
//
// Who needs it: host code that runs where it may not allocate device memory
// and has no spare buffer of its own to lend as a workspace -- for example an
// execute callback of an inference engine that owns every device allocation,
// or a latency-critical loop where the implicit synchronisation of cudaMalloc
// is not acceptable.  The OrbitQuant pages have no counterpart for this; it
// is plumbing only.
//
// The scratch is one file-scope __device__ array of OQ_NOALLOC_SCRATCH_BYTES,
// which every GPU that loads the library holds until the process exits.  In
// host code the array's name is only a host-side stand-in, so the device
// address is fetched with cudaGetSymbolAddress once per device (with that
// device current) and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "oq_internal.h"

static __device__ __align__(256) unsigned char g_oq_noalloc_scratch[OQ_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[OQ_MAX_DEVICES] = {};

int scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_oq_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return oq::fail(OQ_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return OQ_OK;
}
}  // namespace

extern "C" int oq_linear_noalloc(oq_rpbh_t r, oq_codebook_t cb_a, oq_codebook_t cb_w, const void* X, int M,
                                 const uint8_t* w_codes, const void* w_norm, int N, const void* bias, int epilogue,
                                 float* Y_f32, void* Y_bf16, void* stream) {
  oq::clear_error();
  if (!r || !cb_a) return oq::fail(OQ_ERR_ARG, "NULL handle");
  if (M < 0) return oq::fail(OQ_ERR_ARG, "M must be >= 0 (got %d)", M);
  const size_t need = oq_linear_workspace_bytes(M, r->d, cb_a->bits);
  if (need > (size_t)OQ_NOALLOC_SCRATCH_BYTES)
    return oq::fail(OQ_ERR_UNSUPPORTED,
                    "M=%d rows of d=%d at %d bits need %zu bytes of scratch; the static scratch holds %zu "
                    "(use oq_linear with a workspace, or split M)",
                    M, r->d, cb_a->bits, need, (size_t)OQ_NOALLOC_SCRATCH_BYTES);
  int dev;
  if (int rc = oq::current_device(&dev)) return rc;
  // Everything the launch needs must already exist on this device, so that
  // nothing on this path allocates: the rotation's tables (uploaded when the
  // handle was created with this device current) and the status word (made
  // by the first kernel launch of any other entry point, or by
  // oq_get_device_status).
  if (oq::rpbh_tables_if_present(r, dev) != OQ_OK)
    return oq::fail(OQ_ERR_ARG, "the RPBH handle has no tables on device %d: create it with that device current",
                    dev);
  if (oq::codebook_qtable_if_present(cb_a, dev) != OQ_OK)
    return oq::fail(OQ_ERR_ARG,
                    "the activation codebook has no tables on device %d: build it with that device current", dev);
  int* status = nullptr;
  if (oq::device_status_word_if_present(&status) != OQ_OK)
    return oq::fail(OQ_ERR_ARG,
                    "device %d has no status word yet: call oq_get_device_status() (or any other launching entry "
                    "point) once on it first",
                    dev);
  void* scratch;
  if (int rc = scratch_address(dev, &scratch)) return rc;
  return oq_linear(r, cb_a, cb_w, X, M, w_codes, w_norm, N, bias, epilogue, Y_f32, Y_bf16, scratch,
                   (size_t)OQ_NOALLOC_SCRATCH_BYTES, stream);
}
