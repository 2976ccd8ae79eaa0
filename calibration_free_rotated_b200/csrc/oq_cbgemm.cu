// Kernel 2: codebook GEMM on packed codes with the norm-rescale epilogue.
//
// "OrbitQuant: Data-Agnostic Quantization for Image and Video Diffusion
// Transformers", Methodology, "Online Activation Quantization" (last
// paragraph): the shared rotation cancels in the product, so the layer is
//   y[m][n] = s_m r'_n sum_k C_a[ca[m][k]] C_w[cw[n][k]]  (+ bias_n)
// computed here as  acc = sum_k LUT_a[ca] LUT_w[cw]  (fp16 operands,
// LUT = fp16(sqrt(d) c)), y = acc * s_m * r'_n / d + bias_n, optional GELU.
//
// sm_100a design (persistent; tiles of 256 x 256 shared by a CTA pair of a
// cluster with tcgen05 cta_group::2, or 128 x 256 on one CTA when M <= 128):
//   warp 20      TMA producer: 2-D tensor copies of the packed code tiles into a
//                4- or 8-deep packed ring (each CTA: 128 rows of A, its B rows;
//                3-bit codes travel two k-steps per copy).
//   warps 0..15  converters, four groups of four warps running out of phase,
//                group g expanding k-steps g, g+4, ...  Thread r of a group
//                expands activation row r through the fp16 LUT straight into
//                TMEM lane r with tcgen05.st, and its weight row(s) into the
//                canonical K-major 128-byte-swizzled UMMA layout in shared
//                memory.  (Register byte-permute tables for 2, 3 and 4 bits, a
//                128-byte shared table for 6 bits.)
//   warp 21      one elected lane of the leader CTA's warp issues tcgen05.mma (kind::f16,
//                A from TMEM, B from shared memory, M = 256 across the pair,
//                N = 256, K = 16, fp32 accumulate in TMEM); tcgen05.commit
//                (multicast to both CTAs) frees ring stages and publishes the
//                finished accumulator.
//   warps 16..19 epilogue: tcgen05.ld of the accumulator (each warp its 32-lane
//                quadrant), rescale, bias, GELU, fp32/bf16 stores.
//   (GELU tiles of short K with bf16 output: three converter groups, warps
//   0..11, and eight epilogue warps, 12..19, two per quadrant, that split the
//   tile's columns between them.)
// Keeping A in TMEM removes A's expanded stores and tensor-core reads from
// shared memory, whose bandwidth otherwise caps the kernel near 2/3 of the
// tensor rate.  TMEM: one 256-column fp32 accumulator plus 4 A stages of 32
// columns.  Every mbarrier wait is bounded (~1 s); a wait that gives up records
// OQ_ERR_TIMEOUT, raises an abort flag that makes every role skip its remaining
// work, and the CTA still reaches its teardown (TMEM is always released).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include <type_traits>

#include "oq_internal.h"

namespace oq {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;  // per-CTA A rows, tile N, K step
constexpr int GROUP_WARPS = 4;               // one warp per SM sub-partition and TMEM lane quarter
constexpr int TMA_WARP = 20;
constexpr int MMA_WARP = 21;
constexpr int NUM_THREADS = 22 * 32;
constexpr int TMEM_COLS = 512;
constexpr int A_COL0 = BN;                   // A stage s: TMEM columns A_COL0 + 32 s .. + 31

// Warp roles for NG converter groups (group g expands k-steps g, g + NG, ...):
// warps 0 .. 4 NG - 1 convert, the next 20 - 4 NG run the epilogue (four, one
// per TMEM lane quarter, for NG = 4; eight, two per quarter, for NG = 3), warp
// 20 is the TMA producer and warp 21 issues the MMAs.  NG = 3 is for GELU
// tiles with short K, where the epilogue's arithmetic, not the converters,
// paces the tiles.
template <int NG>
struct Roles {
  static_assert(NG == 3 || NG == 4, "converter groups");
  static constexpr int CONV_WARPS = NG * GROUP_WARPS;
  static constexpr int EPI_WARP0 = CONV_WARPS;
  static constexpr int NEPI = TMA_WARP - EPI_WARP0;
  static constexpr int ESTAGES = NG;                     // expanded ring: stage g belongs to group g
  static constexpr int SPARE_COL = A_COL0 + 32 * ESTAGES;  // 128 columns: epilogue spill area
  static_assert(SPARE_COL + BN / 2 <= TMEM_COLS, "TMEM plan");
};
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

struct GemmArgs {
  const float* a_norm;
  const uint16_t* w_norm;
  const uint16_t* bias;
  float* y32;
  uint16_t* y16;
  int* status;
  int M, N, K;
  int tiles_m, num_tiles;
  int epilogue;
  int stall;  // test hook: the producer issues no tensor copies (the waits run out)
  float inv_d;
  uint32_t lut_a[32];  // 64 fp16 entries, two per word (entry 2i in the low half)
  uint32_t lut_w[32];
};

template <int BITS>
struct PackedTile {
  static constexpr int kRowBytes = BK * BITS / 8;
};

// k-steps per packed ring stage (one TMA load of each operand): a tensor copy's
// box must be a multiple of 16 bytes wide, so 3-bit rows (24 bytes per k-step)
// travel two k-steps at a time; the two converter groups of those k-steps
// share the stage.
template <int BA, int BW>
struct PackedUnit {
  static constexpr int KP = (PackedTile<BA>::kRowBytes % 16 || PackedTile<BW>::kRowBytes % 16) ? 2 : 1;
  static constexpr int kRowA = KP * PackedTile<BA>::kRowBytes;  // bytes of an A row in a stage
  static constexpr int kRowB = KP * PackedTile<BW>::kRowBytes;
  static_assert(kRowA % 16 == 0 && kRowB % 16 == 0, "TMA box width");
};

// ---- shared memory plan (offsets from a 1024-aligned base) -------------------
// PAIR: two CTAs of a cluster share one 256 x 256 tile (cta_group::2); each holds
// 128 rows of A and 128 of the 256 B rows.  Otherwise one CTA owns 128 x 256.
template <int BA, int BW, bool PAIR, int NG = 4>
struct Smem {
  static constexpr int ESTAGES = Roles<NG>::ESTAGES;
  static constexpr int kBnCta = PAIR ? BN / 2 : BN;
  static constexpr int kExpBBytes = kBnCta * BK * 2;
  static constexpr int kPkA = BM * PackedUnit<BA, BW>::kRowA;
  static constexpr int kPkB = kBnCta * PackedUnit<BA, BW>::kRowB;
  static constexpr int kPkAStride = (kPkA + 127) / 128 * 128;
  static constexpr int kPkBStride = (kPkB + 127) / 128 * 128;
  // bytes that do not depend on the ring depth or the output staging
  static constexpr int kFixed = ESTAGES * kExpBBytes + 256 + 4 * 2 * BN * 4 + 512 + 16 + 1024;
  static constexpr int kBudget = 227 * 1024;
  // Packed ring: 8 stages (two per group) where they fit, else 4 (always 4 for
  // NG = 3, whose second epilogue half has two staging blocks of its own).
  // Output staging: 128 rows x 128-byte swizzled blocks of 16 KB (64 bf16 or
  // 32 fp32 columns).
  static constexpr int kXtraBlocks = NG == 3 ? 2 : 0;
  static constexpr int kPS =
      NG == 4 && kFixed + 8 * (kPkAStride + kPkBStride) + (PAIR ? 4 : 2) * 16384 <= kBudget ? 8 : 4;
  static constexpr int kRest = kBudget - kFixed - kPS * (kPkAStride + kPkBStride) - kXtraBlocks * 16384;
  static constexpr int kStageBlocks = (PAIR && kRest >= 4 * 16384) ? 4 : (kRest >= 2 * 16384 ? 2 : 1);
  static_assert(NG == 4 || (PAIR && kStageBlocks == 4), "the split epilogue needs four staging blocks");
  static constexpr int kExpB = 0;
  static constexpr int kStage = kExpB + ESTAGES * kExpBBytes;
  static constexpr int kPackA = kStage + (kStageBlocks + kXtraBlocks) * 16384;
  static constexpr int kPackB = kPackA + kPS * kPkAStride;
  static constexpr int kLut = kPackB + kPS * kPkBStride;
  static constexpr int kEpi = kLut + 256;                 // 4 warps x (r'[256], bias[256]) floats
  static constexpr int kBars = kEpi + 4 * 2 * BN * 4;
  // barriers: pk_full[P], pk_empty[P], ex_full[E], ex_empty[E], acc_full, acc_empty
  static constexpr int kNumBars = 2 * kPS + 2 * ESTAGES + 2;
  static constexpr int kMisc = kBars + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kTotal = kMisc + 16;
  // Room to align the base, and never less than half an SM's shared memory:
  // the kernel allocates all 512 TMEM columns, so a second resident CTA would
  // wait in tcgen05.alloc for the first one to finish.
  static constexpr int kMinAlloc = 120 * 1024;
  static constexpr int kAlloc = kTotal + 1024 > kMinAlloc ? kTotal + 1024 : kMinAlloc;
  static_assert(kNumBars * 8 <= 512, "barrier area");
  static_assert(kAlloc <= kBudget, "shared memory plan exceeds 227 KB");
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; on give-up records the status, raises the CTA abort flag.  The
// clock and the abort flag are read only every 64 polls.
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicExch(status, OQ_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait with cluster-scope acquire (barriers that the peer CTA arrives on).
__device__ bool wait_bounded_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicExch(status, OQ_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Arrive on the barrier at the same shared offset in CTA `rank` of the cluster.
// Callers order their shared-memory writes first (fence.proxy.async for data the
// tensor cores read, tcgen05.fence for TMEM reads); the arrive itself keeps the
// default semantics, which avoids a cluster-wide memory fence per call.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(bar), "r"(rank));
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused for this layout)
  d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset
  d |= (uint64_t)1 << 46;             // descriptor version for sm_100
  d |= (uint64_t)2 << 61;             // SWIZZLE_128B
  return d;
}

// Instruction descriptor: D f32, A/B f16, both K-major, N = 256, M = 128 (one CTA)
// or 256 (CTA pair).
template <int MMA_M>
__host__ __device__ constexpr uint32_t idesc_f16() {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(MMA_M >> 4) << 24);
}

template <bool PAIR>
__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t accumulate) {
  if constexpr (PAIR) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc_f16<256>()), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc_f16<128>()), "r"(accumulate)
        : "memory");
  }
}

// Arrives on `bar` (same offset) in every CTA of the pair, or locally, once all
// MMAs issued so far by this thread have completed.
template <bool PAIR>
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  if constexpr (PAIR) {
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"(mask)
        : "memory");
  } else {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
  }
}

// True in exactly one lane of the (fully converged) warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, e;\n\t}"
      : "=r"(p));
  return p != 0;
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// One packed row of a k-step into registers: BYTES = 16, 32 or 48 (16-byte
// aligned), or 24 for 3-bit codes (8-byte aligned).
template <int BYTES>
__device__ __forceinline__ void lds_row(uint32_t addr, uint32_t* w) {
  if constexpr (BYTES % 16 == 0) {
#pragma unroll
    for (int i = 0; i < BYTES / 16; ++i)
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[4 * i]), "=r"(w[4 * i + 1]), "=r"(w[4 * i + 2]), "=r"(w[4 * i + 3])
                   : "r"(addr + 16 * i));
  } else {
#pragma unroll
    for (int i = 0; i < BYTES / 8; ++i)
      asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[2 * i]), "=r"(w[2 * i + 1]) : "r"(addr + 8 * i));
  }
}

// Codes 8i .. 8i+7 of a packed row held in registers (little-endian bit stream).
template <int BITS>
__device__ __forceinline__ uint64_t row_chunk(const uint32_t* w, int i) {
  if constexpr (BITS == 4) {
    return w[i];
  } else if constexpr (BITS == 2) {
    return (w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
  } else if constexpr (BITS == 3) {  // 24 bits starting at byte 3 i
    const int byte = 3 * i, wi = byte >> 2, sh = 8 * (byte & 3);
    const uint64_t lo = w[wi], hi = (wi + 1 < 6) ? w[wi + 1] : 0u;
    return (((hi << 32) | lo) >> sh) & 0xFFFFFFull;
  } else {  // 6 bits: 48 bits starting at byte 6 i
    const int byte = 6 * i, wi = byte >> 2, sh = 8 * (byte & 3);
    const uint64_t lo = w[wi], hi = (wi + 1 < 12) ? w[wi + 1] : 0u;
    return (((hi << 32) | lo) >> sh) & 0xFFFFFFFFFFFFull;
  }
}

// ---- code -> fp16 expansion ---------------------------------------------------
// The codebooks are odd: entry 2^b-1-k is entry k with the sign bit flipped
// (the host checks this bit pattern before launch). A 4-bit code n is therefore
// the magnitude entry m = n (n < 8) or m = 15 - n (n >= 8) of the eight
// negative entries 0..7, negated when n >= 8. The magnitude tables are byte
// planes: lo0/hi0 hold the low/high bytes of entries 0..3, lo1/hi1 of 4..7.
struct Lut8 {
  uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ Lut8 make_lut8(const uint32_t* words) {
  Lut8 t;
  t.lo0 = prmt(words[0], words[1], 0x6420);
  t.hi0 = prmt(words[0], words[1], 0x7531);
  t.lo1 = prmt(words[2], words[3], 0x6420);
  t.hi1 = prmt(words[2], words[3], 0x7531);
  return t;
}

// x >> s for a constant s, on the IMAD pipe (which issues alongside the ALU pipe
// that byte-permutes and logic ops share): high word of x * 2^(32-s).
template <int S>
__device__ __forceinline__ uint32_t shr_imad(uint32_t x) {
  uint32_t r;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(1u << (32 - S)));
  return r;
}

__device__ __forceinline__ uint32_t mul_lo(uint32_t x, uint32_t y) {
  uint32_t r;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
  return r;
}

__device__ __forceinline__ uint32_t mul_hi(uint32_t x, uint32_t y) {
  uint32_t r;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(y));
  return r;
}

// Eight 4-bit codes (nibble i of x is code i) -> four fp16x2 words.
// ALU: 14 ops (byte permutes and logic); 3 multiplies go to the IMAD pipe.
__device__ __forceinline__ uint4 expand8_nib(uint32_t x, const Lut8& t) {
  const uint32_t xs = x & 0x88888888u;                           // bit 3 of every code
  const uint32_t sel = (x ^ mul_hi(xs, 0xE0000000u)) & 0x77777777u;  // m: n ^ 7 where bit 3 is set
  const uint32_t x4 = mul_lo(x, 16u);  // bit 3 of codes 0, 2, 4, 6 at bit 7 of a byte
  uint4 r;
  {
    const uint32_t lo = prmt(t.lo0, t.lo1, sel);
    const uint32_t sg = prmt(x4, x, 0xD9C8u);  // 0xFF in byte i where code i >= 8
    const uint32_t hi = prmt(t.hi0, t.hi1, sel) ^ (sg & 0x80808080u);
    r.x = prmt(lo, hi, 0x5140u);
    r.y = prmt(lo, hi, 0x7362u);
  }
  {
    const uint32_t s2 = shr_imad<16>(sel);
    const uint32_t lo = prmt(t.lo0, t.lo1, s2);
    const uint32_t sg = prmt(x4, x, 0xFBEAu);  // codes 4..7
    const uint32_t hi = prmt(t.hi0, t.hi1, s2) ^ (sg & 0x80808080u);
    r.z = prmt(lo, hi, 0x5140u);
    r.w = prmt(lo, hi, 0x7362u);
  }
  return r;
}

// Eight codes -> uint4 of eight fp16 (element 0 in the low half of .x).
template <int BITS>
__device__ __forceinline__ uint4 expand8(uint64_t packed, const Lut8& t8, uint32_t q0, uint32_t q1,
                                         uint32_t lut_smem) {
  uint4 r;
  if constexpr (BITS == 4) {
    r = expand8_nib((uint32_t)packed, t8);
  } else if constexpr (BITS == 2) {
    // q0 / q1 are the low / high byte planes of the 4-entry table.  The eight
    // 2-bit codes are spread to one code per nibble (three shift-mask steps,
    // shifts on the IMAD pipe); each nibble then selects its entry's bytes
    // from the planes, and the bytes interleave into fp16 pairs.
    uint32_t n = (uint32_t)packed & 0xFFFFu;
    n = (n | mul_lo(n, 1u << 8)) & 0x00FF00FFu;
    n = (n | mul_lo(n, 1u << 4)) & 0x0F0F0F0Fu;
    n = (n | mul_lo(n, 1u << 2)) & 0x33333333u;  // nibble i = code i
    const uint32_t n_hi = shr_imad<16>(n);
    uint32_t lo = prmt(q0, q0, n), hi = prmt(q1, q1, n);
    r.x = prmt(lo, hi, 0x5140u);
    r.y = prmt(lo, hi, 0x7362u);
    lo = prmt(q0, q0, n_hi);
    hi = prmt(q1, q1, n_hi);
    r.z = prmt(lo, hi, 0x5140u);
    r.w = prmt(lo, hi, 0x7362u);
  } else if constexpr (BITS == 3) {
    // t8 holds the byte planes of all eight entries (no sign folding).  The
    // eight 3-bit codes are spread to one code per nibble in three
    // shift-mask steps (shifts on the IMAD pipe): 12-bit halves to 16-bit
    // halves, 6-bit pairs to bytes, codes to nibbles.
    const uint32_t x = (uint32_t)packed;
    uint32_t n = (x & 0x00000FFFu) | (mul_lo(x, 1u << 4) & 0x0FFF0000u);
    n = (n & 0x003F003Fu) | (mul_lo(n, 1u << 2) & 0x3F003F00u);
    n = (n & 0x07070707u) | (mul_lo(n, 1u << 1) & 0x70707070u);  // nibble i = code i
    const uint32_t n_hi = shr_imad<16>(n);
    uint32_t lo = prmt(t8.lo0, t8.lo1, n), hi = prmt(t8.hi0, t8.hi1, n);
    r.x = prmt(lo, hi, 0x5140u);
    r.y = prmt(lo, hi, 0x7362u);
    lo = prmt(t8.lo0, t8.lo1, n_hi);
    hi = prmt(t8.hi0, t8.hi1, n_hi);
    r.z = prmt(lo, hi, 0x5140u);
    r.w = prmt(lo, hi, 0x7362u);
  } else {  // 6 bits: shared 64-entry table
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t c0 = (uint32_t)(packed >> (12 * i)) & 63u;
      const uint32_t c1 = (uint32_t)(packed >> (12 * i + 6)) & 63u;
      o[i] = lds_u16(lut_smem + 2 * c0) | (lds_u16(lut_smem + 2 * c1) << 16);
    }
    r = make_uint4(o[0], o[1], o[2], o[3]);
  }
  return r;
}

// Eight packed codes starting at shared address `addr` (8*BITS bits).

// Offset of (row, 16-byte chunk c) in a K-major 128-byte-swizzled tile of 64 fp16 per row.
__device__ __forceinline__ uint32_t sw128_offset(int row, int c) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4));
}

// ---- packed f32x2 arithmetic (two columns per instruction) -------------------
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU (exact erf form) of two values:  GELU(y) = y Phi(y),
// Phi(y) = (1 + erf(y / sqrt 2)) / 2, computed as
//   y Phi(y) = relu(y) - |y| (1 - erf(|y| / sqrt 2)) / 2
// (no sign restore, no cancellation in either tail).  1 - erf is the rational
// approximation of Abramowitz & Stegun, Handbook of Mathematical Functions,
// 7.1.26 (Hastings):
//   1 - erf(x) = t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-x^2),
//   t = 1 / (1 + p x),  x >= 0,  |error| <= 1.5e-7,
// with x = |y| / sqrt 2 folded into p and the exponent, and the factor -1/2
// folded into the a_i.  Branch-free, packed f32x2 except the two reciprocals,
// exponentials and maxima; large |y| gives exp -> 0.
__device__ __forceinline__ unsigned long long gelu2(unsigned long long y) {
  constexpr float kP = 0.3275911f * 0.70710678118654752f;  // p / sqrt 2
  constexpr float kA1 = -0.5f * 0.254829592f, kA2 = -0.5f * -0.284496736f, kA3 = -0.5f * 1.421413741f,
                  kA4 = -0.5f * -1.453152027f, kA5 = -0.5f * 1.061405429f;
  constexpr float kE = -0.72134752044448170f;  // -log2(e) / 2: exp(-y^2/2) = 2^(kE y^2)
  float y0, y1;
  f2_unpack(y, y0, y1);
  const unsigned long long ay = f2_pack(fabsf(y0), fabsf(y1));
  float d0, d1;
  f2_unpack(f2_fma(ay, f2_pack(kP, kP), f2_pack(1.0f, 1.0f)), d0, d1);
  const unsigned long long t = f2_pack(rcp_approx(d0), rcp_approx(d1));
  unsigned long long q = f2_fma(t, f2_pack(kA5, kA5), f2_pack(kA4, kA4));
  q = f2_fma(q, t, f2_pack(kA3, kA3));
  q = f2_fma(q, t, f2_pack(kA2, kA2));
  q = f2_fma(q, t, f2_pack(kA1, kA1));
  q = f2_mul(q, t);  // -(1 - erf(|y| / sqrt 2)) / 2 before the Gaussian factor
  float w0, w1;
  f2_unpack(f2_mul(y, f2_mul(y, f2_pack(kE, kE))), w0, w1);
  q = f2_mul(q, f2_pack(ex2_approx(w0), ex2_approx(w1)));
  return f2_fma(ay, q, f2_pack(fmaxf(y0, 0.0f), fmaxf(y1, 0.0f)));
}

__device__ __forceinline__ float bf16_to_f32(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// Two floats -> bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Epilogue arithmetic of 8 consecutive columns c .. c+7 of one row:
// y = acc * (s_m / d) * r'_n + bias_n, optional GELU, rounded to bf16.
__device__ __forceinline__ uint4 epi8_bf16(const uint32_t* v, const float* col_r, const float* col_b, int c,
                                           unsigned long long as2, bool gelu) {
  const ulonglong2 r01 = *reinterpret_cast<const ulonglong2*>(col_r + c);
  const ulonglong2 r23 = *reinterpret_cast<const ulonglong2*>(col_r + c + 4);
  const ulonglong2 b01 = *reinterpret_cast<const ulonglong2*>(col_b + c);
  const ulonglong2 b23 = *reinterpret_cast<const ulonglong2*>(col_b + c + 4);
  const unsigned long long rr[4] = {r01.x, r01.y, r23.x, r23.y};
  const unsigned long long bb[4] = {b01.x, b01.y, b23.x, b23.y};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    unsigned long long y2 = f2_fma(f2_mul(f2_pack(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])), as2),
                                   rr[j], bb[j]);
    if (gelu) y2 = gelu2(y2);
    float y0, y1;
    f2_unpack(y2, y0, y1);
    o[j] = bf16x2_rn(y0, y1);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Named barrier `id` over four epilogue warps (one epilogue group: ids 1, 2).
__device__ __forceinline__ void epi_bar(uint32_t id = 1) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// True in every thread of the epilogue group if `p` holds in any of them.
__device__ __forceinline__ bool epi_any(bool p, uint32_t id = 1) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred b, %2, 128, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id)
      : "memory");
  return r != 0;
}

// Bulk tensor store of one box from shared memory (clipped to the tensor).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Stores 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Loads 16 consecutive 32-bit TMEM columns of this thread's lane (complete
// after tcgen05.wait::ld).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

template <int BA, int BW, bool PAIR, int NG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    cbgemm_kernel(const __grid_constant__ GemmArgs args, const __grid_constant__ CUtensorMap map_a,
                  const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_y16,
                  const __grid_constant__ CUtensorMap map_y32) {
  using S = Smem<BA, BW, PAIR, NG>;
  using R = Roles<NG>;
  constexpr int ESTAGES = R::ESTAGES;
  constexpr int BN_CTA = S::kBnCta;
  constexpr int TILE_M = PAIR ? 2 * BM : BM;
  constexpr uint32_t NCTA = PAIR ? 2 : 1;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kMisc + 4);
  uint16_t* lut_a_s = reinterpret_cast<uint16_t*>(smem + S::kLut);
  uint16_t* lut_w_s = lut_a_s + 64;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the next kernel may launch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // 0 = leader (issues the MMAs)
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int nunits = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  constexpr int PSTAGES = S::kPS;
  const int PK_FULL = 0, PK_EMPTY = PSTAGES, EX_FULL = 2 * PSTAGES, EX_EMPTY = 2 * PSTAGES + ESTAGES,
            ACC_FULL = 2 * PSTAGES + 2 * ESTAGES, ACC_EMPTY = ACC_FULL + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(bar(PK_FULL + s), 1);
      mbar_init(bar(PK_EMPTY + s), GROUP_WARPS * PackedUnit<BA, BW>::KP);  // the groups that read it
    }
    for (int s = 0; s < ESTAGES; ++s) {
      mbar_init(bar(EX_FULL + s), GROUP_WARPS * NCTA);     // one group in each CTA
      mbar_init(bar(EX_EMPTY + s), 1);
    }
    mbar_init(bar(ACC_FULL), 1);
    mbar_init(bar(ACC_EMPTY), R::NEPI * NCTA);             // epilogue warps of both CTAs
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < 64) {
    lut_a_s[threadIdx.x] = (uint16_t)(args.lut_a[threadIdx.x >> 1] >> (16 * (threadIdx.x & 1)));
    lut_w_s[threadIdx.x] = (uint16_t)(args.lut_w[threadIdx.x >> 1] >> (16 * (threadIdx.x & 1)));
  }
  if (warp == MMA_WARP) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();   // barriers initialised in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // The set-up above overlaps the previous kernel in the stream (programmatic
  // dependent launch); the codes, norms and bias may be its outputs, and Y
  // may be its input: wait for it to complete before any global access.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int KB = args.K / BK;
  const int num_tiles = args.num_tiles;
  // k-steps this CTA runs over all its tiles (the converters' flat sequence)
  const uint32_t my_tiles = unit < num_tiles ? (uint32_t)((num_tiles - 1 - unit) / nunits + 1) : 0u;
  const uint32_t total_steps = my_tiles * (uint32_t)KB;

  if (warp == TMA_WARP) {
    if (lane == 0 && !args.stall) {
      constexpr uint32_t bytes = S::kPkA + S::kPkB;
      constexpr int KP = PackedUnit<BA, BW>::KP;
      uint32_t pc = 0;  // packed stages issued
      bool ok = true;
      for (int t = unit; t < num_tiles && ok; t += nunits) {
        const int m0 = (t % args.tiles_m) * TILE_M + (int)rank * BM;
        const int n0 = (t / args.tiles_m) * BN + (int)rank * BN_CTA;
        for (int kb = 0; kb < KB; kb += KP, ++pc) {
          const int s = pc % PSTAGES;
          const uint32_t ph = (pc / PSTAGES) & 1u;
          if (!wait_bounded(bar(PK_EMPTY + s), ph ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(PK_FULL + s), bytes);
          tma_load_2d(sbase + S::kPackA + s * S::kPkAStride, &map_a, kb * PackedTile<BA>::kRowBytes, m0,
                      bar(PK_FULL + s));
          tma_load_2d(sbase + S::kPackB + s * S::kPkBStride, &map_b, kb * PackedTile<BW>::kRowBytes, n0,
                      bar(PK_FULL + s));
        }
      }
    }
  } else if (warp < R::CONV_WARPS) {
    // ---- converters: group g = warp / 4 expands k-steps g, g+4, g+8, ... ----
    // Thread (quad q = warp % 4, lane) owns row r = 32 q + lane of both operands:
    // the activation row goes to TMEM lane r (32 columns of fp16 pairs, lower K
    // in the low half) and the weight row(s) to the swizzled shared stage. The
    // four groups run out of phase, so one group's waits overlap another's
    // arithmetic; each group expands before it waits for its ring slot.
    const int g = warp / GROUP_WARPS, q = warp % GROUP_WARPS;
    const int r = 32 * q + lane;
    Lut8 ta, tw;
    // 2-bit tables as byte planes (low bytes of the 4 entries, high bytes)
    const uint32_t qa0 = prmt(args.lut_a[0], args.lut_a[1], 0x6420), qa1 = prmt(args.lut_a[0], args.lut_a[1], 0x7531);
    const uint32_t qw0 = prmt(args.lut_w[0], args.lut_w[1], 0x6420), qw1 = prmt(args.lut_w[0], args.lut_w[1], 0x7531);
    if constexpr (BA == 4 || BA == 3) ta = make_lut8(args.lut_a);  // 4 bits: the negative half
    if constexpr (BW == 4 || BW == 3) tw = make_lut8(args.lut_w);
    constexpr int RB_A = PackedTile<BA>::kRowBytes, RB_B = PackedTile<BW>::kRowBytes;
    constexpr int NB_ROWS = BN_CTA / BM;  // weight rows per thread: 1 (pair) or 2
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(A_COL0 + 32 * g);
    constexpr int KP = PackedUnit<BA, BW>::KP;
    constexpr int ROW_A = PackedUnit<BA, BW>::kRowA, ROW_B = PackedUnit<BA, BW>::kRowB;
    for (uint32_t pc = (uint32_t)g, j = 0; pc < total_steps; pc += NG, ++j) {
      const uint32_t pu = pc / KP;  // packed stage that holds k-step pc
      const int ps = pu % PSTAGES;
      const uint32_t pph = (pu / PSTAGES) & 1u;
      const uint32_t sub = pc % KP;  // this k-step's part of the stage's rows
      bool got = wait_bounded(bar(PK_FULL + ps), pph, abort_flag, args.status);
      __syncwarp();
      if (__any_sync(0xFFFFFFFFu, !got)) break;
      uint32_t wa[RB_A / 4], wb[NB_ROWS][RB_B / 4];
      lds_row<RB_A>(sbase + S::kPackA + ps * S::kPkAStride + r * ROW_A + sub * RB_A, wa);
#pragma unroll
      for (int h = 0; h < NB_ROWS; ++h)
        lds_row<RB_B>(sbase + S::kPackB + ps * S::kPkBStride + (r + BM * h) * ROW_B + sub * RB_B, wb[h]);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(PK_EMPTY + ps));  // packed stage read by this warp
      uint32_t v[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 e = expand8<BA>(row_chunk<BA>(wa, i), ta, qa0, qa1, sbase + S::kLut);
        v[4 * i] = e.x; v[4 * i + 1] = e.y; v[4 * i + 2] = e.z; v[4 * i + 3] = e.w;
      }
      got = wait_bounded(bar(EX_EMPTY + g), (j & 1u) ^ 1u, abort_flag, args.status);
      __syncwarp();
      if (__any_sync(0xFFFFFFFFu, !got)) break;
      tc_fence_after();  // the MMAs that read this stage are complete
      tmem_st16(t_lane, v);
      tmem_st16(t_lane + 16u, v + 16);
      const uint32_t eb = sbase + S::kExpB + g * S::kExpBBytes;
#pragma unroll
      for (int h = 0; h < NB_ROWS; ++h) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          sts_v4(eb + sw128_offset(r + BM * h, i), expand8<BW>(row_chunk<BW>(wb[h], i), tw, qw0, qw1, sbase + S::kLut + 128));
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(bar(EX_FULL + g), 0);  // the leader's barrier
        else mbar_arrive(bar(EX_FULL + g));
      }
    }
  } else if (warp == MMA_WARP) {
    // The whole warp runs the loop, converged, so the stage addresses and
    // descriptors stay warp-uniform; one elected lane issues the MMAs and
    // commits.  (Issuing from a lone active lane cost about 1.4x more cycles
    // per k-step.)  The B descriptor of stage es, k-slice k is the stage-0
    // descriptor plus the byte offset / 16.
    if (rank == 0) {
      uint32_t ec = 0, lt = 0;
      bool ok = true;
      const uint64_t bdesc0 = umma_desc_sw128(sbase + S::kExpB);
      const uint32_t a_tmem0 = tmem_base + (uint32_t)A_COL0;
      for (int t = unit; t < num_tiles && ok; t += nunits, ++lt) {
        const uint32_t aph = lt & 1u;
        bool got = PAIR ? wait_bounded_cluster(bar(ACC_EMPTY), aph ^ 1u, abort_flag, args.status)
                        : wait_bounded(bar(ACC_EMPTY), aph ^ 1u, abort_flag, args.status);
        if (!__all_sync(0xFFFFFFFFu, got)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++ec) {
          const uint32_t es = ec % ESTAGES;
          const uint32_t eph = (ec / ESTAGES) & 1u;
          const bool full = PAIR ? wait_bounded_cluster(bar(EX_FULL + es), eph, abort_flag, args.status)
                                 : wait_bounded(bar(EX_FULL + es), eph, abort_flag, args.status);
          if (!__all_sync(0xFFFFFFFFu, full)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = a_tmem0 + 32u * es;
          const uint64_t bdesc = bdesc0 + (uint64_t)((es * (uint32_t)S::kExpBBytes) >> 4);
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_f16_ts<PAIR>(tmem_base, a_tmem + 8u * k, bdesc + 2u * k, (kb > 0 || k > 0) ? 1u : 0u);
            umma_commit<PAIR>(bar(EX_EMPTY + es));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) umma_commit<PAIR>(bar(ACC_FULL));
        __syncwarp();
      }
    }
  } else if (warp >= R::EPI_WARP0 && warp < R::EPI_WARP0 + R::NEPI) {
    // ---- epilogue: this CTA's 128 accumulator rows ----
    // TMEM -> registers -> scale, bias, GELU -> swizzled staging -> bulk tensor
    // stores. The accumulator is released right after its last TMEM read, so the
    // next tile's MMAs overlap the conversion and the stores. The four warps
    // take every decision together (named barrier 1), so none can wait on a
    // barrier that another has left.
    //
    // bf16-only output with the four-block staging (the usual case): the
    // accumulator is first evacuated without arithmetic -- columns 128..255 to
    // the spare TMEM columns, columns 0..127 as raw fp32 into the staging
    // buffer (exactly its 64 KB) -- and released; the arithmetic then runs
    // from those copies while the next tile's MMAs proceed.  The first half is
    // converted in place (each thread rewrites only its own row, and a raw
    // chunk is always read before a bf16 chunk lands on it).
    //
    // With NG = 3 the eight epilogue warps form two groups of four (named
    // barriers 1 and 2), one warp of each per TMEM lane quarter, and split
    // every tile (bf16-only output, which the launcher guarantees): group 0
    // evacuates columns 0..127 as raw fp32 into staging blocks 0..3 and
    // converts them in place (blocks 0, 1); group 1 evacuates columns
    // 128..255 into the spare TMEM columns and converts them into staging
    // blocks 4, 5.  Each group's leader issues and waits for its own stores.
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int rl = quad * 32 + lane;  // row within the CTA's 128
    const int sub = (warp - R::EPI_WARP0) >> 2;  // epilogue group (0 unless NG == 3)
    const uint32_t bid = 1u + (uint32_t)sub;     // its named barrier
    const bool leader = (warp == R::EPI_WARP0 + 4 * sub && lane == 0);
    const uint32_t stage = sbase + S::kStage;
    float* col_r = reinterpret_cast<float*>(smem + S::kEpi) + quad * 2 * BN;
    float* col_b = col_r + BN;
    const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16);
    constexpr int J0 = 0, JN = BN / 32;  // the 32-column chunks of the factors this warp loads
    const int j0 = NG == 3 ? 4 * sub : J0, jn = NG == 3 ? 4 * sub + 4 : JN;
    if constexpr (NG == 3) {
      if ((args.y16 == nullptr || args.y32 != nullptr) && leader && sub == 0) {
        atomicExch(args.status, OQ_ERR_UNSUPPORTED);  // never launched this way
        *abort_flag = 1;
      }
    }
    uint32_t lt = 0;
    for (int t = unit; t < num_tiles; t += nunits, ++lt) {
      const int m0 = (t % args.tiles_m) * TILE_M + (int)rank * BM, n0 = (t / args.tiles_m) * BN;
      const int row = m0 + rl;
      // this tile's factors, fetched while the MMAs run: a_row / d, r'_n and bias_n
      const float a_scale = row < args.M ? args.a_norm[row] * args.inv_d : 0.0f;
#pragma unroll
      for (int j = J0; j < JN; ++j) {
        if (j < j0 || j >= jn) continue;
        const int n = n0 + lane + 32 * j;
        const bool in = n < args.N;
        col_r[lane + 32 * j] = in ? bf16_to_f32(args.w_norm[n]) : 0.0f;
        col_b[lane + 32 * j] = (in && args.bias) ? bf16_to_f32(args.bias[n]) : 0.0f;
      }
      __syncwarp();
      const bool got = wait_bounded(bar(ACC_FULL), lt & 1u, abort_flag, args.status);
      if (epi_any(!got, bid)) break;
      tc_fence_after();
      if constexpr (NG == 3) {
        constexpr int H = BN / 2;
        const uint32_t rsw = (uint32_t)(rl & 7);  // the row's 128-byte swizzle
        const unsigned long long as2 = f2_pack(a_scale, a_scale);
        const bool gelu = args.epilogue == OQ_EPI_GELU;
        if (leader) bulk_wait_read();  // this group's previous stores have read its staging blocks
        epi_bar(bid);
        if (sub == 0) {
#pragma unroll 1
          for (int c = 0; c < H; c += 32) {  // columns 0.. -> staging block c / 32, raw fp32
            uint32_t v[32];
            __syncwarp();
            tmem_ld16(taddr + (uint32_t)c, v);
            tmem_ld16(taddr + (uint32_t)(c + 16), v + 16);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            const uint32_t rowb = stage + (uint32_t)(c / 32) * 16384u + (uint32_t)rl * 128u;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              sts_v4(rowb + (((uint32_t)j ^ rsw) << 4), make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
          }
        } else {
          const uint32_t spare = taddr + (uint32_t)R::SPARE_COL;
#pragma unroll 1
          for (int c = 0; c < H; c += 32) {  // columns H.. -> spare TMEM columns
            uint32_t v[32];
            __syncwarp();
            tmem_ld16(taddr + (uint32_t)(H + c), v);
            tmem_ld16(taddr + (uint32_t)(H + c + 16), v + 16);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            tmem_st16(spare + (uint32_t)c, v);
            tmem_st16(spare + (uint32_t)(c + 16), v + 16);
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(bar(ACC_EMPTY), 0);  // the leader's barrier
          else mbar_arrive(bar(ACC_EMPTY));
        }
        if (sub == 0) {
          // columns 0..127: raw fp32 (blocks 0..3) -> bf16 (blocks 0, 1), in place
#pragma unroll 1
          for (int c0 = 0; c0 < H; c0 += 16) {
            const uint32_t src = stage + (uint32_t)(c0 / 32) * 16384u + (uint32_t)rl * 128u;
            const uint32_t jr = (uint32_t)(c0 % 32) / 4;
            uint32_t v[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 w = lds_v4(src + (((jr + i) ^ rsw) << 4));
              v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
            }
            const uint32_t dst = stage + (uint32_t)(c0 / 64) * 16384u + (uint32_t)rl * 128u;
            const uint32_t jb = (uint32_t)(c0 % 64) / 8;
            sts_v4(dst + ((jb ^ rsw) << 4), epi8_bf16(v, col_r, col_b, c0, as2, gelu));
            sts_v4(dst + (((jb + 1) ^ rsw) << 4), epi8_bf16(v + 8, col_r, col_b, c0 + 8, as2, gelu));
          }
        } else {
          // columns 128..255: spare TMEM -> bf16 (blocks 4, 5); the next load is in flight during the arithmetic
          const uint32_t spare = taddr + (uint32_t)R::SPARE_COL;
          uint32_t va[16], vb[16];
          __syncwarp();
          tmem_ld16(spare, va);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll 1
          for (int c0 = 0; c0 < H; c0 += 32) {
            __syncwarp();
            tmem_ld16(spare + (uint32_t)(c0 + 16), vb);
            {
              const uint32_t dst = stage + (uint32_t)(4 + c0 / 64) * 16384u + (uint32_t)rl * 128u;
              const uint32_t jb = (uint32_t)(c0 % 64) / 8;
              sts_v4(dst + ((jb ^ rsw) << 4), epi8_bf16(va, col_r, col_b, H + c0, as2, gelu));
              sts_v4(dst + (((jb + 1) ^ rsw) << 4), epi8_bf16(va + 8, col_r, col_b, H + c0 + 8, as2, gelu));
            }
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            __syncwarp();
            if (c0 + 32 < H) tmem_ld16(spare + (uint32_t)(c0 + 32), va);
            {
              const uint32_t dst = stage + (uint32_t)(4 + (c0 + 16) / 64) * 16384u + (uint32_t)rl * 128u;
              const uint32_t jb = (uint32_t)((c0 + 16) % 64) / 8;
              sts_v4(dst + ((jb ^ rsw) << 4), epi8_bf16(vb, col_r, col_b, H + c0 + 16, as2, gelu));
              sts_v4(dst + (((jb + 1) ^ rsw) << 4), epi8_bf16(vb + 8, col_r, col_b, H + c0 + 24, as2, gelu));
            }
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        epi_bar(bid);
        if (leader) {
          const int b0 = sub == 0 ? 0 : 4, x0 = n0 + (sub == 0 ? 0 : H);
          for (int b = 0; b < 2; ++b)
            if (x0 + 64 * b < args.N && m0 < args.M)
              tma_store_2d(&map_y16, stage + (uint32_t)(b0 + b) * 16384u, x0 + 64 * b, m0);
          bulk_commit();
        }
        continue;
      }
      if (S::kStageBlocks == 4 && args.y16 != nullptr && args.y32 == nullptr) {
        constexpr int H = BN / 2;
        const uint32_t spare = taddr + (uint32_t)R::SPARE_COL;
        const uint32_t rsw = (uint32_t)(rl & 7);  // the row's 128-byte swizzle
        if (leader) bulk_wait_read();  // the previous tile's stores have read the staging buffer
        epi_bar();
#pragma unroll 1
        for (int c = 0; c < H; c += 32) {  // columns H.. -> spare TMEM columns
          uint32_t v[32];
          __syncwarp();
          tmem_ld16(taddr + (uint32_t)(H + c), v);
          tmem_ld16(taddr + (uint32_t)(H + c + 16), v + 16);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          tmem_st16(spare + (uint32_t)c, v);
          tmem_st16(spare + (uint32_t)(c + 16), v + 16);
        }
#pragma unroll 1
        for (int c = 0; c < H; c += 32) {  // columns 0.. -> staging block c / 32, raw fp32
          uint32_t v[32];
          __syncwarp();
          tmem_ld16(taddr + (uint32_t)c, v);
          tmem_ld16(taddr + (uint32_t)(c + 16), v + 16);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          const uint32_t rowb = stage + (uint32_t)(c / 32) * 16384u + (uint32_t)rl * 128u;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            sts_v4(rowb + (((uint32_t)j ^ rsw) << 4), make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(bar(ACC_EMPTY), 0);  // the leader's barrier
          else mbar_arrive(bar(ACC_EMPTY));
        }
        const unsigned long long as2 = f2_pack(a_scale, a_scale);
        const bool gelu = args.epilogue == OQ_EPI_GELU;
        // columns 0..127: raw fp32 (blocks 0..3) -> bf16 (blocks 0, 1)
#pragma unroll 1
        for (int c0 = 0; c0 < H; c0 += 16) {
          const uint32_t src = stage + (uint32_t)(c0 / 32) * 16384u + (uint32_t)rl * 128u;
          const uint32_t jr = (uint32_t)(c0 % 32) / 4;
          uint32_t v[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 w = lds_v4(src + (((jr + i) ^ rsw) << 4));
            v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
          }
          const uint32_t dst = stage + (uint32_t)(c0 / 64) * 16384u + (uint32_t)rl * 128u;
          const uint32_t jb = (uint32_t)(c0 % 64) / 8;
          sts_v4(dst + ((jb ^ rsw) << 4), epi8_bf16(v, col_r, col_b, c0, as2, gelu));
          sts_v4(dst + (((jb + 1) ^ rsw) << 4), epi8_bf16(v + 8, col_r, col_b, c0 + 8, as2, gelu));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        epi_bar();
        if (leader) {
          for (int b = 0; b < 2; ++b)
            if (n0 + 64 * b < args.N && m0 < args.M) tma_store_2d(&map_y16, stage + (uint32_t)b * 16384u, n0 + 64 * b, m0);
          bulk_commit();
        }
        // columns 128..255: spare TMEM -> bf16 (blocks 2, 3); the next load is in flight during the arithmetic
        {
          uint32_t va[16], vb[16];
          __syncwarp();
          tmem_ld16(spare, va);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll 1
          for (int c0 = 0; c0 < H; c0 += 32) {
            __syncwarp();
            tmem_ld16(spare + (uint32_t)(c0 + 16), vb);
            {
              const uint32_t dst = stage + (uint32_t)(2 + c0 / 64) * 16384u + (uint32_t)rl * 128u;
              const uint32_t jb = (uint32_t)(c0 % 64) / 8;
              sts_v4(dst + ((jb ^ rsw) << 4), epi8_bf16(va, col_r, col_b, H + c0, as2, gelu));
              sts_v4(dst + (((jb + 1) ^ rsw) << 4), epi8_bf16(va + 8, col_r, col_b, H + c0 + 8, as2, gelu));
            }
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            __syncwarp();
            if (c0 + 32 < H) tmem_ld16(spare + (uint32_t)(c0 + 32), va);
            {
              const uint32_t dst = stage + (uint32_t)(2 + (c0 + 16) / 64) * 16384u + (uint32_t)rl * 128u;
              const uint32_t jb = (uint32_t)((c0 + 16) % 64) / 8;
              sts_v4(dst + ((jb ^ rsw) << 4), epi8_bf16(vb, col_r, col_b, H + c0 + 16, as2, gelu));
              sts_v4(dst + (((jb + 1) ^ rsw) << 4), epi8_bf16(vb + 8, col_r, col_b, H + c0 + 24, as2, gelu));
            }
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        epi_bar();
        if (leader) {
          for (int b = 2; b < 4; ++b)
            if (n0 + 64 * b < args.N && m0 < args.M) tma_store_2d(&map_y16, stage + (uint32_t)b * 16384u, n0 + 64 * b, m0);
          bulk_commit();
        }
        continue;
      }
#pragma unroll 1
      for (int kind = 0; kind < 2; ++kind) {  // 0: bf16 output, 1: fp32 output
        const bool want = kind == 0 ? args.y16 != nullptr : args.y32 != nullptr;
        if (!want) continue;
        const bool last_kind = kind == 1 || args.y32 == nullptr;
        const int cpb = kind == 0 ? 64 : 32;  // columns per 128-byte block
        const int pass_cols = S::kStageBlocks * cpb;
#pragma unroll 1
        for (int p0 = 0; p0 < BN; p0 += pass_cols) {
          if (leader) bulk_wait_read();  // the previous stores have read the staging buffer
          epi_bar();
#pragma unroll 1
          for (int c0 = p0; c0 < p0 + pass_cols; c0 += 16) {
            uint32_t v[16];
            __syncwarp();
            tmem_ld16(taddr + (uint32_t)c0, v);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            if (last_kind && c0 + 16 == BN) {  // last read of this accumulator
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_cluster(bar(ACC_EMPTY), 0);  // the leader's barrier
                else mbar_arrive(bar(ACC_EMPTY));
              }
            }
            const int lc = c0 - p0;  // column within the pass
            const uint32_t blk = stage + (uint32_t)(lc / cpb) * 16384u + (uint32_t)rl * 128u;
            const int j0 = (lc % cpb) * (kind == 0 ? 2 : 4) / 16;  // first 16-byte chunk of the row
            const unsigned long long as2 = f2_pack(a_scale, a_scale);
#pragma unroll
            for (int q = 0; q < 2; ++q) {  // 8 columns at a time, as f32x2 pairs
              const ulonglong2 r01 = *reinterpret_cast<const ulonglong2*>(col_r + c0 + 8 * q);
              const ulonglong2 r23 = *reinterpret_cast<const ulonglong2*>(col_r + c0 + 8 * q + 4);
              const ulonglong2 b01 = *reinterpret_cast<const ulonglong2*>(col_b + c0 + 8 * q);
              const ulonglong2 b23 = *reinterpret_cast<const ulonglong2*>(col_b + c0 + 8 * q + 4);
              const unsigned long long rr[4] = {r01.x, r01.y, r23.x, r23.y};
              const unsigned long long bb[4] = {b01.x, b01.y, b23.x, b23.y};
              float y[8];
              const bool gelu = args.epilogue == OQ_EPI_GELU;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const unsigned long long acc2 =
                    f2_pack(__uint_as_float(v[8 * q + 2 * j]), __uint_as_float(v[8 * q + 2 * j + 1]));
                unsigned long long y2 = f2_fma(f2_mul(acc2, as2), rr[j], bb[j]);
                if (gelu) y2 = gelu2(y2);
                f2_unpack(y2, y[2 * j], y[2 * j + 1]);
              }
              if (kind == 0) {
                sts_v4(blk + (uint32_t)(((j0 + q) ^ (rl & 7)) << 4),
                       make_uint4(bf16x2_rn(y[0], y[1]), bf16x2_rn(y[2], y[3]), bf16x2_rn(y[4], y[5]),
                                  bf16x2_rn(y[6], y[7])));
              } else {
                sts_v4(blk + (uint32_t)(((j0 + 2 * q) ^ (rl & 7)) << 4),
                       make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                                  __float_as_uint(y[3])));
                sts_v4(blk + (uint32_t)(((j0 + 2 * q + 1) ^ (rl & 7)) << 4),
                       make_uint4(__float_as_uint(y[4]), __float_as_uint(y[5]), __float_as_uint(y[6]),
                                  __float_as_uint(y[7])));
              }
            }
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // staging visible to the bulk copies
          epi_bar();
          if (leader) {
            const CUtensorMap* map = kind == 0 ? &map_y16 : &map_y32;
            for (int b = 0; b < S::kStageBlocks; ++b) {
              const int x = n0 + p0 + b * cpb;
              if (x < args.N && m0 < args.M) tma_store_2d(map, stage + (uint32_t)b * 16384u, x, m0);
            }
            bulk_commit();
          }
        }
      }
    }
    if (leader) bulk_wait_all();
  }

  // teardown: every role of both CTAs is done (or gave up); release TMEM
  __syncwarp();
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) {
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// ---- host side ----------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encode_fn(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  if (!cached) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
      return fail(OQ_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (%s)", cudaGetErrorString(e));
    cached = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = cached;
  return OQ_OK;
}

// Encodes a 2-D map from its cache key (no interleave, unit element strides).
int encode_2d(const TmapKey& k, void* out) {
  EncodeTiledFn enc;
  if (int rc = get_encode_fn(&enc)) return rc;
  cuuint64_t dims[2] = {(cuuint64_t)k.dim0, (cuuint64_t)k.dim1};
  cuuint64_t strides[1] = {(cuuint64_t)k.stride1};
  cuuint32_t box[2] = {(cuuint32_t)k.box0, (cuuint32_t)k.box1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(static_cast<CUtensorMap*>(out), (CUtensorMapDataType)k.type, 2, const_cast<void*>(k.base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, (CUtensorMapSwizzle)k.swizzle,
                   (CUtensorMapL2promotion)k.promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(OQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return OQ_OK;
}

// 2-D map over packed codes: [rows][row_bytes] uint8, box = (64 codes, box_rows).
int make_code_map(CUtensorMap* map, const void* base, int rows, int row_bytes, int box_bytes, int box_rows) {
  static_assert(sizeof(CUtensorMap) == 128, "tensor map size");
  TmapKey k{base, (unsigned long long)row_bytes, (unsigned long long)rows, (unsigned long long)row_bytes,
            (unsigned)box_bytes, (unsigned)box_rows, (int)CU_TENSOR_MAP_DATA_TYPE_UINT8,
            (int)CU_TENSOR_MAP_SWIZZLE_NONE, (int)CU_TENSOR_MAP_L2_PROMOTION_L2_128B};
  return cached_tensor_map(k, map, encode_2d);
}

// Row-major M x N output, written in 128-row boxes of 128 bytes with the
// 128-byte swizzle that the epilogue's staging layout uses.
int make_out_map(CUtensorMap* map, void* base, int M, int N, CUtensorMapDataType type, int esize) {
  TmapKey k{base, (unsigned long long)N, (unsigned long long)M, (unsigned long long)N * (unsigned long long)esize,
            (unsigned)(128 / esize), 128u, (int)type, (int)CU_TENSOR_MAP_SWIZZLE_128B,
            (int)CU_TENSOR_MAP_L2_PROMOTION_NONE};
  return cached_tensor_map(k, map, encode_2d);
}

using GemmKernel = void (*)(GemmArgs, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap);

template <int BA, int BW, bool PAIR, int NG>
int launch_t(GemmArgs& a, const uint8_t* a_codes, const uint8_t* w_codes, int nsm, cudaStream_t stream) {
  using S = Smem<BA, BW, PAIR, NG>;
  CUtensorMap ma, mb;
  if (int rc = make_code_map(&ma, a_codes, a.M, a.K * BA / 8, PackedUnit<BA, BW>::kRowA, BM)) return rc;
  if (int rc = make_code_map(&mb, w_codes, a.N, a.K * BW / 8, PackedUnit<BA, BW>::kRowB, S::kBnCta)) return rc;
  if ((a.K / BK) % PackedUnit<BA, BW>::KP != 0)
    return fail(OQ_ERR_UNSUPPORTED, "3-bit codes need d %% 128 == 0 (d=%d)", a.K);
  CUtensorMap my16, my32;
  memset(&my16, 0, sizeof(my16));
  memset(&my32, 0, sizeof(my32));
  if (a.y16)
    if (int rc = make_out_map(&my16, a.y16, a.M, a.N, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2)) return rc;
  if (a.y32)
    if (int rc = make_out_map(&my32, a.y32, a.M, a.N, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4)) return rc;
  GemmKernel k = cbgemm_kernel<BA, BW, PAIR, NG>;
  const int smem = S::kAlloc;
  const int tile_m = PAIR ? 2 * BM : BM;
  a.tiles_m = (a.M + tile_m - 1) / tile_m;
  a.num_tiles = a.tiles_m * ((a.N + BN - 1) / BN);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  int units = std::min(a.num_tiles, nsm);
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  if (PAIR) {
    attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
    attr[cfg.numAttrs].val.clusterDim.x = 2;
    attr[cfg.numAttrs].val.clusterDim.y = 1;
    attr[cfg.numAttrs].val.clusterDim.z = 1;
    cfg.numAttrs += 1;
    int max_clusters = 0;
    if (int rc = occupancy(reinterpret_cast<const void*>(k), smem, NUM_THREADS, 2, &max_clusters)) return rc;
    if (max_clusters < 1) return fail(OQ_ERR_UNSUPPORTED, "no CTA pair of the GEMM fits on this device");
    units = std::min(std::min(a.num_tiles, max_clusters), nsm / 2);  // one CTA per SM
    cfg.gridDim = dim3(2 * units, 1, 1);
  } else {
    int per_sm = 0;
    if (int rc = occupancy(reinterpret_cast<const void*>(k), smem, NUM_THREADS, 0, &per_sm)) return rc;
    if (per_sm < 1) return fail(OQ_ERR_UNSUPPORTED, "the GEMM's CTA does not fit on this device");
    cfg.gridDim = dim3(units, 1, 1);
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, k, a, ma, mb, my16, my32);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "GEMM launch: %s", cudaGetErrorString(e));
  return OQ_OK;
}

template <int BA, int BW>
int launch_pick(GemmArgs& a, const uint8_t* a_codes, const uint8_t* w_codes, int nsm, cudaStream_t stream) {
  // CTA pairs halve the operand expansion per tensor-core flop; one CTA suffices
  // when a single 128-row tile covers M.  GELU tiles of short K (at most 32
  // k-steps) with bf16-only output take three converter groups and eight
  // epilogue warps: there the epilogue's arithmetic, not the expansion, sets
  // the pace.
  if (a.M > BM) {
    if (a.epilogue == OQ_EPI_GELU && a.y16 != nullptr && a.y32 == nullptr && a.K <= 32 * BK)
      return launch_t<BA, BW, true, 3>(a, a_codes, w_codes, nsm, stream);
    return launch_t<BA, BW, true, 4>(a, a_codes, w_codes, nsm, stream);
  }
  return launch_t<BA, BW, false, 4>(a, a_codes, w_codes, nsm, stream);
}

}  // namespace

int launch_cbgemm(int d, oq_codebook_t cb_a, oq_codebook_t cb_w, const uint8_t* a_codes, const float* a_norm, int M,
                  const uint8_t* w_codes, const uint16_t* w_norm, int N, const uint16_t* bias, int epilogue,
                  float* Y_f32, uint16_t* Y_bf16, void* stream) {
  int* status;
  if (int rc = device_status_word(&status)) return rc;
  int nsm;
  if (int rc = sm_count(&nsm)) return rc;
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.a_norm = a_norm;
  a.w_norm = w_norm;
  a.bias = bias;
  a.y32 = Y_f32;
  a.y16 = Y_bf16;
  a.status = status;
  a.M = M;
  a.N = N;
  a.K = d;
  a.epilogue = epilogue;
  // the two tables are fp16(sqrt(d_cb) c): the product carries d_cb (= d unless
  // the codebooks are for the block)
  a.inv_d = (float)(1.0 / std::sqrt((double)cb_a->d * (double)cb_w->d));
  a.stall = take_test_stall(2);
  for (int i = 0; i < 32; ++i) {
    auto entry = [](oq_codebook_t cb, int k) -> uint32_t {
      return k < (int)cb->lut.size() ? cb->lut[k] : 0u;
    };
    a.lut_a[i] = entry(cb_a, 2 * i) | (entry(cb_a, 2 * i + 1) << 16);
    a.lut_w[i] = entry(cb_w, 2 * i) | (entry(cb_w, 2 * i + 1) << 16);
  }
  // The 4-bit expansion reads only the negative half of each table and flips
  // the sign bit for the rest.
  for (oq_codebook_t cb : {cb_a, cb_w}) {
    const int L = 1 << cb->bits;
    for (int k = 0; k < L; ++k)
      if ((uint16_t)cb->lut[L - 1 - k] != (uint16_t)(cb->lut[k] ^ 0x8000u))
        return fail(OQ_ERR_UNSUPPORTED, "codebook table is not odd (entry %d)", k);
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int ba = cb_a->bits, bw = cb_w->bits;
#define OQ_GEMM_CASE(X, Y) \
  if (ba == X && bw == Y) return launch_pick<X, Y>(a, a_codes, w_codes, nsm, s);
  OQ_GEMM_CASE(4, 4)
  OQ_GEMM_CASE(4, 2)
  OQ_GEMM_CASE(6, 4)
  OQ_GEMM_CASE(2, 2)
  OQ_GEMM_CASE(2, 4)
  OQ_GEMM_CASE(4, 6)
  OQ_GEMM_CASE(6, 6)
  OQ_GEMM_CASE(6, 2)
  OQ_GEMM_CASE(2, 6)
  OQ_GEMM_CASE(3, 3)
#undef OQ_GEMM_CASE
  return fail(OQ_ERR_UNSUPPORTED, "no GEMM kernel for bits a=%d w=%d", ba, bw);
}

}  // namespace oq
