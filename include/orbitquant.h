/*
 * orbitquant.h -- C ABI of the B200 (sm_100a) OrbitQuant hot path.
 *
 * OrbitQuant quantizes both operands of a linear layer in one shared rotated,
 * normalised basis: activations are rotated online by the randomized
 * permuted block-Hadamard (RPBH) transform, split into norm and direction,
 * and the direction is coded against a data-free Lloyd-Max codebook; weights
 * went through the same steps offline; the layer multiplies the codes and
 * rescales by both norms.  Sources are cited by page title and section:
 *
 *   [OQ]  "OrbitQuant: Data-Agnostic Quantization for Image and Video
 *          Diffusion Transformers" -- the method.
 *   [TQ]  "TurboQuant: Online Vector Quantization with Near-optimal
 *          Distortion Rate" (slide deck) -- f_d and Lloyd-Max origins.
 *
 * Conventions for every entry point
 *   - Return value: OQ_OK (0) or one of the OQ_ERR_* codes below.  Argument
 *     errors are detected on the host before anything is launched, and
 *     oq_last_error() then returns a message (thread-local).
 *   - Device buffers are plain device pointers owned by the caller; they must
 *     be 16-byte aligned (OQ_ERR_ALIGN otherwise).  No entry point frees or
 *     keeps a caller buffer.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Kernel launches are asynchronous on that stream.
 *   - Handles (oq_rpbh_t, oq_codebook_t) are created on the host and own
 *     small device tables.  Tables are uploaded to the current device when
 *     the handle is created (if a device is present) and lazily, once, to any
 *     other device the handle is used on; that lazy first use allocates and
 *     copies synchronously, so make it outside any stream capture.
 *   - Device-side failures (a bounded wait in a kernel that gave up) are
 *     recorded in a per-device status word; read and clear it with
 *     oq_get_device_status().
 *   - Layouts: bf16 tensors are row-major uint16 bit patterns.  Packed codes
 *     of a row form a little-endian bit stream, code i in bits [i*b, (i+1)*b)
 *     (4 bits: element 2j in the low nibble of byte j; 6 bits: four codes in
 *     three bytes); each row is d*b/8 bytes.
 */
#ifndef ORBITQUANT_H
#define ORBITQUANT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define OQ_API __attribute__((visibility("default")))
#else
#define OQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  OQ_OK = 0,
  OQ_ERR_ARG = 1,          /* null handle/pointer, bad size, mismatched handles */
  OQ_ERR_UNSUPPORTED = 2,  /* valid for the method but not for these kernels */
  OQ_ERR_ALIGN = 3,        /* a device pointer is not 16-byte aligned */
  OQ_ERR_CUDA = 4,         /* a CUDA runtime call failed (message has the name) */
  OQ_ERR_TIMEOUT = 5,      /* a kernel's bounded wait gave up (device status) */
  OQ_ERR_NOMEM = 6         /* host or device allocation of a handle table failed */
};

enum { OQ_EPI_NONE = 0, OQ_EPI_GELU = 1 };

typedef struct oq_rpbh_s* oq_rpbh_t;
typedef struct oq_codebook_s* oq_codebook_t;

/* Version of this ABI (major*100 + minor). */
OQ_API int oq_version(void);

/* Number of device allocations (cudaMalloc) the library has made in this
 * process, on every device: the status words and the handles' device tables,
 * which are the only device memory it allocates.  A diagnostic: a call that
 * leaves it unchanged allocated nothing.  Never fails. */
OQ_API long long oq_device_allocations(void);

/* Message for the last error returned on this host thread ("" if none). */
OQ_API const char* oq_last_error(void);

/* Reads and clears the device status word of the current device after
 * synchronising `stream`.  Returns OQ_OK, OQ_ERR_TIMEOUT, or OQ_ERR_CUDA. */
OQ_API int oq_get_device_status(void* stream);

/* Synchronous checking, for debugging: when on, every launching entry point
 * waits for its stream and returns the device status word itself (so a kernel
 * that gave up is reported by the call that launched it, as OQ_ERR_TIMEOUT).
 * Off by default; the environment variable OQ_DEBUG=1 turns it on at first
 * use.  Not for use inside CUDA graph capture (it synchronises). */
OQ_API int oq_set_debug(int on);

/* Test hook for the failure path: the next launch of kernel 1 (rotate +
 * quantize, one-round rotations) or kernel 2 (codebook GEMM), on any stream,
 * issues none of its bulk / tensor copies.  Its bounded waits then run out
 * (about 1 s), it records OQ_ERR_TIMEOUT in the device status word and every
 * CTA leaves through its normal teardown, so the context stays usable; the
 * launch's outputs are undefined.  kernel 0 disarms.  One launch consumes it.
 * Errors: OQ_ERR_ARG for a kernel outside 0..2. */
OQ_API int oq_test_stall_next(int kernel);

/* Test hook (host only, no device needed): the composed-rotation kernel's
 * tables for handle r (rounds >= 2), as the library builds them, for the
 * coordinate register order (xch = 0) or the block-transposed one (xch = 1,
 * blocks of 64..256):
 *   gather : uint16 [rounds][d]   slot that register r of thread g reads in
 *                                 round k, at [k][32 g + r] (round 1: 4-byte
 *                                 bf16 pair words; later rounds: 8-byte slots);
 *   store  : uint16 [rounds][d]   slot it stores its output to in round k
 *                                 (rounds before the last; the last is 0);
 *   signs  : uint32 [rounds][d/32] bit r of word [k][g]: the sign of the
 *                                 coordinate register r of thread g gathers.
 * Buffers are caller-owned host arrays of those sizes.  Errors: OQ_ERR_ARG
 * (NULL, one-round handle), OQ_ERR_UNSUPPORTED (xch for another block). */
OQ_API int oq_test_composed_tables(oq_rpbh_t r, int xch, uint16_t* gather, uint16_t* store, uint32_t* signs);

/* ---------------------------------------------------------------------------
 * RPBH rotation  Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi
 * [OQ] Methodology, "Randomized Permuted Block-Hadamard (RPBH) Rotation".
 *
 * seed  : the fixed random draw ("drawn once per dimension").  SplitMix64
 *         with state = seed; pi by Fisher-Yates (i = d-1..1,
 *         j = next() mod (i+1), swap), then d signs: sign_j = -1 when the top
 *         bit of next() is set.
 * d     : dimension, >= 1.  The kernels need d % 32 == 0 and d <= 16384.
 * block : h, a power of two dividing d; 0 picks the page's rule (largest
 *         power of two dividing d).  The kernels support 32 <= h <= 1024.
 * H_h is the Sylvester-order Walsh-Hadamard matrix scaled by 1/sqrt(h), so
 * Pi_d is orthogonal; (P x)_j = x_{pi(j)}; the signs act before H.
 * Errors: OQ_ERR_ARG (d < 1, bad block, null out), OQ_ERR_NOMEM.
 * ------------------------------------------------------------------------- */
OQ_API int oq_make_rpbh(uint64_t seed, int d, int block, oq_rpbh_t* out);

/* ---------------------------------------------------------------------------
 * Rotation variants of the rotation ablation ([OQ] Experiments, "Rotation
 * Ablation (Table 3)"), as rotation handles that every entry point accepts:
 *   OQ_ROT_RPBH       blkdiag(H_h D_1..) P_pi, exactly oq_make_rpbh.
 *   OQ_ROT_BLOCK_RHT  "Block-RHT (no perm)": blkdiag(H_h D_1..), P = I.  The
 *                     signs are those RPBH draws for the same seed (the
 *                     generator still runs through the Fisher-Yates draws), so
 *                     the two differ only by the permutation.
 *   OQ_ROT_FULL_RHT   "Full RHT": one Hadamard block spanning the largest power
 *                     of two dividing d (all of d when d is a power of two),
 *                     P = I, the same signs.  `block` must be 0 or that size.
 * (The table's dense Haar rotation is a comparison system and is not built.)
 * Errors: as oq_make_rpbh; OQ_ERR_ARG for an unknown kind or a FULL_RHT block
 * other than 0 or d's largest power-of-two divisor.
 * ------------------------------------------------------------------------- */
enum { OQ_ROT_RPBH = 0, OQ_ROT_BLOCK_RHT = 1, OQ_ROT_FULL_RHT = 2 };
OQ_API int oq_make_rotation(uint64_t seed, int d, int block, int kind, oq_rpbh_t* out);
/* Kind (OQ_ROT_*) of a rotation handle. */
OQ_API int oq_rotation_kind(oq_rpbh_t r, int* kind);

/* ---------------------------------------------------------------------------
 * Composed RPBH rotation Pi^(k) = Pi_k ... Pi_1 of k = `rounds` rounds
 * ("Quantizing With Randomized Hadamard Transforms: Efficient Heuristic Now
 * Proven", Methodology: the composition of k randomized Hadamard transforms;
 * Key contributions 1 and 3: two rounds make every coordinate of ANY input
 * close to Gaussian, three also decorrelate the coordinates).  For a block
 * rotation each round is a full RPBH round, Pi_r = blkdiag(H_h D_r) P_r with
 * its own permutation and signs: the permutation is what lets a later round
 * mix coordinates that an earlier one kept inside a block.
 *   Round 1 is exactly oq_make_rpbh(seed, d, block); round r+1 continues the
 *   same SplitMix64 stream after round r's draws (Fisher-Yates, then d signs).
 * Every entry point accepts the handle (weights and activations rotated by the
 * same Pi^(k), so it still cancels in oq_linear).  rounds = 1 is oq_make_rpbh;
 * rounds 2 and 3 run a separate kernel that keeps the row pair in shared
 * memory between rounds (d <= 16384, 32 <= block <= 1024).
 * Errors: as oq_make_rpbh; OQ_ERR_ARG unless 1 <= rounds <= 3;
 * OQ_ERR_UNSUPPORTED for rounds >= 2 unless d % 32 == 0, d <= 16384 and
 * block >= 32 (the limits of the composed kernel, checked before any upload).
 * ------------------------------------------------------------------------- */
OQ_API int oq_make_composed_rpbh(uint64_t seed, int d, int block, int rounds, oq_rpbh_t* out);
/* Rounds of a rotation handle (1 for every handle but a composed one). */
OQ_API int oq_rotation_rounds(oq_rpbh_t r, int* rounds);
/* Copies round `round` (1-based) of a handle: pi (int32[d], host) and its sign
 * bits (uint32[ceil(d/32)], host), in oq_rpbh_export's layout.  Either output
 * may be NULL.  OQ_ERR_ARG for a round outside 1..rounds. */
OQ_API int oq_rpbh_export_round(oq_rpbh_t r, int round, int32_t* perm, uint32_t* sign_bits);

/* d and h of a handle.  Either output may be NULL. */
OQ_API int oq_rpbh_info(oq_rpbh_t r, int* d, int* block);

/* Copies pi (int32[d], host) and the sign bits (uint32[ceil(d/32)], host;
 * bit j%32 of word j/32 set <=> sign_j = -1).  Either output may be NULL. */
OQ_API int oq_rpbh_export(oq_rpbh_t r, int32_t* perm, uint32_t* sign_bits);

OQ_API void oq_free_rpbh(oq_rpbh_t r);

/* ---------------------------------------------------------------------------
 * Lloyd-Max codebook C^(d,b) for the sphere marginal
 *   f_d(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) (1 - t^2)^((d-3)/2)
 * [OQ] "Theoretical Basis" (f_d, codebook, q_hat) and "Data-Agnostic
 * Codebook"; [TQ] slides 14-16.  Built on the host with no data: Lloyd
 * iteration (midpoint boundaries, conditional-mean centroids) from
 * linspace(-a, a, 2^b), a = min(3/sqrt(d), 0.9), integrals by composite
 * Gauss-Legendre in theta = asin(t); stops when max|delta c| sqrt(d) < 1e-13
 * or after 200000 iterations; centroids then made exactly antisymmetric.
 * d >= 3, 1 <= bits <= 8 (kernels: bits <= 6).
 * ------------------------------------------------------------------------- */
OQ_API int oq_build_codebook(int d, int bits, oq_codebook_t* out);

/* d and bits of a handle.  Either output may be NULL. */
OQ_API int oq_codebook_info(oq_codebook_t cb, int* d, int* bits);

/* Copies (host) centroids double[2^b] ascending, bounds double[2^b-1]
 * (midpoints), the dequantisation table lut_fp16 uint16[2^b] = fp16 bits of
 * round-to-nearest-even(sqrt(d) * c_k), the Lloyd iteration count and the
 * per-coordinate distortion int (t - q(t))^2 f_d.  Any output may be NULL. */
OQ_API int oq_codebook_export(oq_codebook_t cb, double* centroids, double* bounds, uint16_t* lut_fp16,
                       int* iterations, double* distortion);

OQ_API void oq_free_codebook(oq_codebook_t cb);

/* ---------------------------------------------------------------------------
 * Online activation quantization  ([OQ] "Online Activation Quantization")
 *   x' = Pi_d x ;  s = ||x'||_2 ;  codes = q_hat(x' / (s + eps)),  eps = 1e-12
 * q_hat(t) = argmin_c |t - c| over C^(d,b); a t exactly on a boundary takes
 * the lower centroid.
 * X     : device bf16 [M][d] (row-major, rows contiguous).
 * codes : device uint8 [M][d*b/8], packed as described at the top.
 * norms : device float [M], s per row (the norm of x' equals that of x).
 * M >= 0 (M == 0 launches nothing).  d is the rotation's width; the codebook
 * is C^(d,b), or C^(h,b) for the rotation's block h (a reading of a
 * "codebook for d = h" on rows of width d; the rows are unit vectors either
 * way, so the codes are well defined).  Any other codebook: OQ_ERR_ARG.
 * ------------------------------------------------------------------------- */
OQ_API int oq_quantize_act(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, uint8_t* codes, float* norms,
                    void* stream);

/* ---------------------------------------------------------------------------
 * Offline weight quantization  ([OQ] "Offline Weight Quantization")
 *   w' = Pi_d w ;  r' = ||w'||_2 ;  codes = q_hat(w' / (r' + eps))
 * r' is stored in bf16 (round to nearest even), step 4 of that section.
 * W     : device bf16 [N][d]; codes: device uint8 [N][d*b/8];
 * norms_bf16 : device bf16 [N].
 * ------------------------------------------------------------------------- */
OQ_API int oq_quantize_weight(oq_rpbh_t r, oq_codebook_t cb, const void* W, int N, uint8_t* codes, void* norms_bf16,
                       void* stream);

/* ---------------------------------------------------------------------------
 * Flatness check of a batch of rows  ("Quantizing With Randomized Hadamard
 * Transforms: Efficient Heuristic Now Proven", Methodology, adaptive
 * verification, and Key contribution 4: an O(d) pass measuring the l3 norm
 * (scalar quantization) and the l_inf norm (vector quantization) of the unit
 * input, which tells whether one randomized Hadamard round suffices or the
 * input needs the two or three rounds of oq_make_composed_rpbh)
 *   rho3[m]   = sum_i |x_mi|^3 / (sum_i x_mi^2)^(3/2)
 *   rhoinf[m] = max_i |x_mi| / (sum_i x_mi^2)^(1/2)
 * Both are scale-free and lie in [d^-1/2, 1] (equal magnitudes .. one-hot);
 * a zero row gives 0 and 0.  rho3 is the Berry-Esseen ratio of one
 * randomized Hadamard coordinate of the row.  The page prints no thresholds:
 * the choice of the round count is the caller's.  One rotation serves a whole
 * layer, so the check reports the batch's maxima as well.
 * X         : device bf16 [M][d], 16-byte aligned, d % 8 == 0, finite values.
 * rho3, rhoinf : device float [M] each, or NULL (not written).
 * batch_max : device float [2] = {max_m rho3, max_m rhoinf}, or NULL; the call
 *             clears it on `stream` before the kernel runs (so it reads 0, 0
 *             for M == 0).
 * Outputs are fp32, from fp32 sums of exactly rescaled values (each row is
 * divided by the power of two at its maximum first), so no finite bf16 row
 * overflows or underflows.  One launch, HBM-bound (each row is read from
 * memory once).  Errors: OQ_ERR_ARG (M < 0, NULL X with M > 0, no output),
 * OQ_ERR_UNSUPPORTED (d), OQ_ERR_ALIGN.
 * ------------------------------------------------------------------------- */
OQ_API int oq_row_flatness(const void* X, int M, int d, float* rho3, float* rhoinf, float* batch_max, void* stream);

/* ---------------------------------------------------------------------------
 * Codebook linear on codes  ([OQ] "Online Activation Quantization", last
 * paragraph: W^' x^' ~= W Pi^T Pi x = W x, no inverse rotation)
 *   y[m][n] = s_m r'_n sum_k v_a[ca[m][k]] v_w[cw[n][k]]  (+ bias_n) (-> GELU)
 * with v = lut_fp16 / sqrt(d_cb) of each codebook (d_cb its dimension).
 * Accumulation is fp32 on the tensor cores (fp16 x fp16 products).
 * d           : common inner dimension.  cb_a and cb_w must have the same
 *               dimension d_cb, which divides d (d_cb = d, or the rotation's
 *               block when the codes were made with C^(h,b)); OQ_ERR_ARG
 *               otherwise.
 * a_codes     : device uint8 [M][d*ba/8];  a_norm : device float [M].
 * w_codes     : device uint8 [N][d*bw/8];  w_norm : device bf16 [N].
 * bias        : device bf16 [N] or NULL.
 * epilogue    : OQ_EPI_NONE or OQ_EPI_GELU (exact erf form).
 * Y_f32       : device float [M][N] or NULL; Y_bf16: device bf16 [M][N] or
 *               NULL (at least one).  Row stride N elements.
 * Needs d % 64 == 0, N % 16 == 0, bits in {2, 4, 6} for both operands, or
 * W3A3 (3 bits for both; [OQ] Experiments, Qualitative Results) with d % 128 == 0.
 * ------------------------------------------------------------------------- */
OQ_API int oq_linear_codes(int d, oq_codebook_t cb_a, oq_codebook_t cb_w, const uint8_t* a_codes, const float* a_norm,
                    int M, const uint8_t* w_codes, const void* w_norm, int N, const void* bias, int epilogue,
                    float* Y_f32, void* Y_bf16, void* stream);

/* Bytes of workspace oq_linear needs for M rows: the activation codes
 * (M*d*bits_a/8, rounded up to 256) plus the norms (4*M). */
OQ_API size_t oq_linear_workspace_bytes(int M, int d, int bits_a);

/* ---------------------------------------------------------------------------
 * Full layer: oq_quantize_act of X into `workspace`, then oq_linear_codes.
 * X : device bf16 [M][d].  workspace: device, >= oq_linear_workspace_bytes.
 * The rotation handle must be the one the weights were quantized with (the
 * shared rotation that cancels in the product).
 * ------------------------------------------------------------------------- */
OQ_API int oq_linear(oq_rpbh_t r, oq_codebook_t cb_a, oq_codebook_t cb_w, const void* X, int M, const uint8_t* w_codes,
              const void* w_norm, int N, const void* bias, int epilogue, float* Y_f32, void* Y_bf16,
              void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * oq_linear without a workspace, for callers that cannot allocate.
 * The OrbitQuant pages have no counterpart for this entry point.
 *
 * Some callers run where they may not allocate device memory and have no
 * buffer of their own to lend (an inference engine's execute callback that
 * owns every allocation, a latency-critical loop that cannot take the
 * implicit synchronisation of cudaMalloc).  This call does exactly what
 * oq_linear does, but keeps the activation codes and norms in a fixed static
 * device array of OQ_NOALLOC_SCRATCH_BYTES instead of a caller workspace.
 *   - It allocates nothing: no cudaMalloc/cudaFree, no allocating library
 *     routine.  The static array is held by every GPU that loads the library
 *     until the process exits.
 *   - Size limit: oq_linear_workspace_bytes(M, d, bits_a) must not exceed
 *     OQ_NOALLOC_SCRATCH_BYTES (32 MiB); larger calls return
 *     OQ_ERR_UNSUPPORTED before launching anything.
 *   - Preconditions (checked; OQ_ERR_ARG otherwise, never an allocation): the
 *     rotation handle was created with this device current, and the device
 *     already has the library's status word (any earlier launching call on
 *     the device, or oq_get_device_status(), creates it).
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current) and caches it.
 *   - All calls share the one array, which keeps the last call's contents;
 *     nothing in it has to start at zero (the quantize kernel rewrites the
 *     codes and norms of all M rows before the GEMM reads them).  Calls that
 *     overlap on the GPU (different streams, or several host threads) race on
 *     the array: serialise them.
 * Arguments, layouts and errors are otherwise those of oq_linear.
 * ------------------------------------------------------------------------- */
#define OQ_NOALLOC_SCRATCH_BYTES (32u << 20)

OQ_API int oq_linear_noalloc(oq_rpbh_t r, oq_codebook_t cb_a, oq_codebook_t cb_w, const void* X, int M,
                             const uint8_t* w_codes, const void* w_norm, int N, const void* bias, int epilogue,
                             float* Y_f32, void* Y_bf16, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ORBITQUANT_H */
