// Kernel 1: RPBH rotation + norm + Lloyd-Max nearest-centroid quantization
// + bit packing, for activation rows (fp32 norms) and weight rows (bf16 norms).
//
// "OrbitQuant: Data-Agnostic Quantization for Image and Video Diffusion
// Transformers", Methodology:
//   RPBH section:      x' = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi x
//   Online activation: s = ||x'||, codes = q_hat(x' / (s + eps))
//   Offline weight:    the same on rows of W, r' stored in BF16
// q_hat is the nearest centroid of the Lloyd-Max codebook ("Theoretical Basis").
//
// The kernel is bound by instruction issue and shared-memory wavefronts long
// before HBM, so every step is counted per element pair:
//   * Persistent CTAs of P row pairs (threads = P * d/32).  A 2-deep ring of
//     stage buffers is filled by 1-D bulk async copies (one per row, row 2p of
//     the stage to the slot's first half, row 2p+1 to its second half) with
//     mbarrier transaction counts, so HBM reads overlap compute.
//   * Interleave: each landed stage is rewritten into a pair buffer whose word
//     j of pair p holds (x[2p][j], x[2p+1][j]), so one 32-bit gather feeds both
//     rows.  Thread (p, g) rewrites its own 32 columns with 128-bit accesses in
//     a lane-rotated chunk order; odd 32-column segments swap their 16-byte
//     halves so the stores are free of bank conflicts too.
//   * The pair buffer is double-buffered and the loop is software-pipelined
//     (interleave of stage k+1, one barrier, quantize of stage k, gather of
//     stage k+1), so one CTA barrier per stage covers the buffer hand-off, the
//     ring-slot release and the row-norm partials.
//   * Gather: thread (p, g) owns output coordinates 32g..32g+31 of both rows.
//     Its 32 shared-memory gather addresses sit in 16 registers (two 16-bit
//     addresses each); the Rademacher signs sit in 8 registers as sign bytes
//     and are applied while splitting the gathered word into two floats
//     (one byte-permute, one shift-add, one logic op per pair).
//   * The two rows travel as f32x2 pairs: the sum of squares and the FWHT
//     stages are packed f32x2 instructions.  For blocks of h = 64, 128, 256
//     (L = h/32 lanes) every stage runs in-thread: the gather fills layout A,
//     where lane l's register group t holds coordinates 32 (t ^ l) + (32/L) l
//     + [0, 32/L), so A's stages cover the block bits above 5; one transpose
//     (register group t xor-shuffled with lane l ^ t, group 0 staying put)
//     then gives layout B, where group u holds 32 l + (32/L)(u ^ l) + [0,
//     32/L), for the stages over bits 0..4.  The XOR relabelling keeps every
//     register index a compile-time constant and turns the swapped roles of
//     the butterflies into a per-lane sign (one FMA per output); the packed
//     codes' groups are moved back from u to u ^ l before the store.  At
//     h = 128 this moves 24 pairs per thread through shuffles instead of 64.
//     Wider blocks, and code widths whose groups are not whole bytes, words or
//     three-word halves, keep log2(h/32) xor-shuffle butterfly stages.
//   * Row norms: lane-segment shuffle reductions, per-segment partials in
//     shared memory, summed in a fixed order (deterministic).
//   * Centroid search in the unit interval: y = sat(t * alpha + 1/2) (the row
//     scale is folded into the multiplier), bucket q = round(y * NB) read from
//     the low mantissa bits of fma(y, NB, 1.5 * 2^23).  Table entry q holds the
//     bucket's only boundary (in y) with the number of boundaries below the
//     bucket in its low b bits; code = entry + (y > boundary), the comparison
//     taken from the sign bit of (boundary - y), so ties take the lower
//     centroid.  (The host builds the table; see build_qtable.)
//   * Packing: each code is funnel-shifted in from the top of its output word
//     (b in {1, 2, 4}), so 32 codes fill exactly b words per row, stored with
//     vector stores.
//   * Every mbarrier wait is bounded (~1 s) and reports OQ_ERR_TIMEOUT; the
//     CTA agrees on a give-up through the barrier's OR-reduction and leaves
//     together.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "oq_rotq.cuh"

namespace oq {

namespace {

// Launch shape and shared-memory layout of one rotate+quantize launch.
struct RotqPlan {
  int cfg, loghb, P, threads, groups, stages, seg_log;
  uint32_t bar_off, part_off, qt_off, ring_off;
  size_t smem;
};

RotqPlan plan_rotq(int d, int h, int M, int qtable_len) {
  RotqPlan p;
  memset(&p, 0, sizeof(p));
  while ((32 << p.loghb) < h) ++p.loghb;
  p.cfg = d <= 6144 ? 0 : (d <= 12288 ? 1 : 2);
  p.P = p.cfg == 0 ? std::max(1, 6144 / d) : 1;
  const int spr = d / 32;
  p.threads = ((p.P * spr + 31) / 32) * 32;
  p.groups = M > 0 ? (M + 2 * p.P - 1) / (2 * p.P) : 0;
  p.stages = p.cfg == 2 ? 1 : 2;
  const int seg = std::min(32, spr & -spr);  // lanes per norm partial (never straddles a pair)
  while ((2 << p.seg_log) <= seg) ++p.seg_log;
  const uint32_t ibs = p.cfg == 0 ? 0x6000u : (p.cfg == 1 ? 0xC000u : 0x10000u);
  const uint32_t nparts = (uint32_t)p.threads >> p.seg_log;
  p.bar_off = 2u * ibs;
  p.part_off = p.bar_off + 64u;
  p.qt_off = p.part_off + ((2u * nparts * 8u + 127u) & ~127u);
  p.ring_off = (p.qt_off + 4u * (uint32_t)qtable_len + 1023u) & ~1023u;
  p.smem = (size_t)p.ring_off + (size_t)p.stages * ibs;
  return p;
}

}  // namespace

int launch_rotq(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, uint8_t* codes, float* norm_f32,
                uint16_t* norm_bf16, void* stream) {
  if (r->rounds > 1) return launch_rotq_composed(r, cb, X, M, codes, norm_f32, norm_bf16, stream);
  const int d = r->d, h = r->h, bits = cb->bits;
  const int qlen = (int)cb->qtable.size();
  if (qlen > 4097) return fail(OQ_ERR_UNSUPPORTED, "codebook d=%d bits=%d needs a %d-entry search table", cb->d, bits, qlen);
  const RotqPlan p = plan_rotq(d, h, M, qlen);
  rotq::KernelFn kern;
  if (r->kind == OQ_ROT_RPBH)
    kern = p.cfg == 0 ? rotq::pick_cfg0(bits, p.loghb)
                      : (p.cfg == 1 ? rotq::pick_cfg1(bits, p.loghb) : rotq::pick_cfg2(bits, p.loghb));
  else
    kern = p.cfg == 0 ? rotq::pick_cfg0_np(bits, p.loghb)
                      : (p.cfg == 1 ? rotq::pick_cfg1_np(bits, p.loghb) : rotq::pick_cfg2_np(bits, p.loghb));
  if (!kern) return fail(OQ_ERR_UNSUPPORTED, "no rotate+quantize kernel for bits=%d h=%d d=%d", bits, h, d);

  const uint16_t* perm;
  const uint32_t* signs;
  if (int rc = rpbh_device_tables(r, &perm, &signs)) return rc;
  const uint32_t* qtable;
  if (int rc = codebook_device_qtable(cb, &qtable)) return rc;
  int* status;
  if (int rc = device_status_word(&status)) return rc;
  int nsm;
  if (int rc = sm_count(&nsm)) return rc;

  rotq::Args a;
  memset(&a, 0, sizeof(a));
  a.X = static_cast<const uint16_t*>(X);
  a.codes = codes;
  a.norm_f32 = norm_f32;
  a.norm_bf16 = norm_bf16;
  a.perm2 = reinterpret_cast<const uint32_t*>(perm);
  a.signs = signs;
  a.qtable = qtable;
  a.status = status;
  a.M = M;
  a.d = d;
  a.P = p.P;
  a.groups = p.groups;
  a.qtable_len = qlen;
  a.seg_log = p.seg_log;
  a.bar_off = p.bar_off;
  a.part_off = p.part_off;
  a.qt_off = p.qt_off;
  a.ring_off = p.ring_off;
  a.alpha_h = (float)((double)cb->qt_alpha / std::sqrt((double)h));
  a.nb = (float)cb->qt_nb;
  a.stall = take_test_stall(1);

  int per_sm = 0;
  if (int rc = occupancy(reinterpret_cast<const void*>(kern), (int)p.smem, p.threads, 0, &per_sm)) return rc;
  if (per_sm < 1) return fail(OQ_ERR_UNSUPPORTED, "rotate+quantize kernel does not fit (d=%d)", d);
  if (a.groups == 0) return OQ_OK;
  const int grid = std::min(a.groups, nsm * per_sm);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3((unsigned)p.threads, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = (cudaStream_t)stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "rotate+quantize launch: %s", cudaGetErrorString(e));
  return OQ_OK;
}

}  // namespace oq
