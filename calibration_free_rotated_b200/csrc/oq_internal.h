// Internal declarations shared by the library's translation units only.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/orbitquant.h"

#define OQ_MAX_DEVICES 64
#define OQ_VERSION 100

struct oq_rpbh_s {
  uint64_t seed = 0;
  int d = 0, h = 0;
  int kind = OQ_ROT_RPBH;  // OQ_ROT_*; only OQ_ROT_RPBH permutes
  std::vector<int32_t> perm;        // pi, (P x)_j = x_{pi(j)}
  std::vector<uint32_t> sign_bits;  // bit j%32 of word j/32 set <=> sign_j = -1
  // Composed rotation Pi_rounds ... Pi_1: rounds 2.. (round 1 is perm / sign_bits)
  int rounds = 1;
  std::vector<int32_t> perm_more;       // [rounds - 1][d]
  std::vector<uint32_t> sign_bits_more;  // [rounds - 1][ceil(d/32)]
  std::mutex mu;
  uint16_t* dev_perm[OQ_MAX_DEVICES] = {};   // pi as uint16 [d]
  uint32_t* dev_signs[OQ_MAX_DEVICES] = {};  // sign words [d/32]
  // composed kernel, per register order (0: coordinate order, 1: the
  // block-transposed layout's): gather slots uint16[rounds][d], store slots
  // uint16[rounds][d], sign words uint32[rounds][d/32], in one allocation
  unsigned char* dev_ctab[2][OQ_MAX_DEVICES] = {};
};

struct oq_codebook_s {
  int d = 0, bits = 0;
  std::vector<double> centroids;  // 2^b ascending, exactly antisymmetric
  std::vector<double> bounds;     // 2^b - 1 midpoints
  std::vector<uint16_t> lut;      // fp16 bits of RNE(sqrt(d) c_k)
  int iterations = 0;
  double distortion = 0.0;
  // Bucket table for the branchless centroid search (see build_qtable).
  float qt_alpha = 0.0f;  // y = t * qt_alpha + 1/2 maps the boundaries into (0, 1)
  int qt_nb = 0;          // buckets; the table has qt_nb + 1 entries
  std::vector<uint32_t> qtable;
  std::mutex mu;
  uint32_t* dev_qtable[OQ_MAX_DEVICES] = {};
};

namespace oq {

// Error reporting: store a message for oq_last_error() and return `code`.
int fail(int code, const char* fmt, ...);
void clear_error();

// Host planning (oq_host.cpp).
uint64_t splitmix64_next(uint64_t& state);
void lloyd_max(int d, int bits, std::vector<double>& centroids, std::vector<double>& bounds, int& iterations,
               double& distortion);
uint16_t double_to_fp16_rne(double v);

// Device-side state (oq_host.cpp).
int current_device(int* dev);
int rpbh_device_tables(oq_rpbh_t r, const uint16_t** perm, const uint32_t** signs);
// Tables of the composed kernel: coordinate order, or (xch) the register order
// of the block-transposed FWHT (OQ_ERR_UNSUPPORTED when the block has none):
// gather slots, store slots (rounds before the last) and sign words.
int rpbh_composed_tables(oq_rpbh_t r, const uint16_t** slots, const uint16_t** store, const uint32_t** signs,
                         bool xch = false);
int codebook_device_qtable(oq_codebook_t cb, const uint32_t** qtable);
void build_qtable(oq_codebook_t cb);
int device_status_word(int** status);
int device_status_word_if_present(int** status);  // never allocates
// OQ_OK when the handle's tables exist on device `dev`, else OQ_ERR_ARG (no
// message); they take the handle's lock and never allocate.
int rpbh_tables_if_present(oq_rpbh_t r, int dev);
int codebook_qtable_if_present(oq_codebook_t cb, int dev);
int sm_count(int* n);
bool aligned16(const void* p);
// Test hook (oq_test_stall_next): 1 exactly once, for the next launch of `kernel`.
int take_test_stall(int kernel);

// Launch preparation cached per device (oq_host.cpp).  On the first use of a
// kernel on a device its dynamic shared-memory limit is raised to the device's
// opt-in maximum; `occupancy` then returns the kernel's resident CTAs per SM
// (cluster == 0) or its resident clusters of `cluster` CTAs per device, queried
// once per (kernel, dynamic shared memory, block size, cluster) and device.
// Steady-state launches therefore make no attribute or occupancy calls.
int occupancy(const void* kernel, int smem, int threads, int cluster, int* value);

// Programmatic dependent launch (oq_host.cpp): whether launches carry the
// programmatic-serialisation attribute (on unless OQ_NO_PDL=1 is set).  A
// kernel so launched may start while the previous kernel in the stream
// finishes; it runs `griddepcontrol.wait` before it touches memory that an
// earlier kernel may write or read, and `griddepcontrol.launch_dependents`
// at its start.  Every grid of this library is persistent and fully resident,
// so the overlap cannot deadlock.
bool pdl_enabled();

// Encoded 2-D tensor maps cached by everything that defines them (base
// address, sizes, strides, box, element type, swizzle, promotion); a launch on
// the same buffers reuses the encoding instead of re-encoding.  `encode`
// fills the map on a miss and returns OQ_OK or an error code.
struct TmapKey {
  const void* base;
  unsigned long long dim0, dim1, stride1;
  unsigned box0, box1;
  int type, swizzle, promo;
  bool operator==(const TmapKey& o) const {
    return base == o.base && dim0 == o.dim0 && dim1 == o.dim1 && stride1 == o.stride1 && box0 == o.box0 &&
           box1 == o.box1 && type == o.type && swizzle == o.swizzle && promo == o.promo;
  }
};
int cached_tensor_map(const TmapKey& key, void* map128, int (*encode)(const TmapKey&, void*));

// Kernel launchers.
int launch_rotq(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, uint8_t* codes, float* norm_f32,
                uint16_t* norm_bf16, void* stream);
int launch_rotq_composed(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, uint8_t* codes, float* norm_f32,
                         uint16_t* norm_bf16, void* stream);
int launch_flatness(const void* X, int M, int d, float* rho3, float* rhoinf, float* batch_max, void* stream);
int launch_cbgemm(int d, oq_codebook_t cb_a, oq_codebook_t cb_w, const uint8_t* a_codes, const float* a_norm, int M,
                  const uint8_t* w_codes, const uint16_t* w_norm, int N, const uint16_t* bias, int epilogue,
                  float* Y_f32, uint16_t* Y_bf16, void* stream);

}  // namespace oq
