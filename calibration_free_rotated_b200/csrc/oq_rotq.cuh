// Rotate+quantize kernel template (kernel 1), shared by the translation units
// that instantiate it (one per configuration, compiled in parallel) and the
// launcher in oq_rotq.cu.  The design notes are at the top of oq_rotq.cu.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "oq_internal.h"

namespace oq {
namespace rotq {

constexpr unsigned long long kWaitLimitNs = 1000000000ull;

struct Args {
  const uint16_t* X;
  uint8_t* codes;
  float* norm_f32;
  uint16_t* norm_bf16;
  const uint32_t* perm2;  // pi as uint16 pairs: word k = pi(2k) | pi(2k+1) << 16
  const uint32_t* signs;  // sign words [d/32]
  const uint32_t* qtable;
  int* status;
  int M, d, P, groups, qtable_len, seg_log;
  uint32_t bar_off, part_off, qt_off, ring_off;  // byte offsets in dynamic shared memory
  float alpha_h;                                 // alpha / sqrt(h)
  float nb;                                      // buckets of the search table
  int stall;                                     // test hook: issue no copies (the waits run out)
};

// Kernel configurations: pair-buffer stride (IBS) and gather-address form.
//   0: P*d <= 6144,  IBS = 24 KB, byte addresses
//   1: d <= 12288,   IBS = 48 KB, byte addresses
//   2: d <= 16384,   IBS = 64 KB, word addresses (16-bit byte addresses overflow)
template <int CFG>
struct Cfg {
  static constexpr uint32_t IBS = CFG == 0 ? 0x6000u : (CFG == 1 ? 0xC000u : 0x10000u);
  static constexpr uint32_t HALF = IBS / 2;  // ring: second row of each pair
  static constexpr bool WORD_ADDR = CFG == 2;
  static constexpr int STAGES = CFG == 2 ? 1 : 2;  // ring slots (compile-time: slot and phase are shifts)
};

// Programmatic dependent launch: let the next kernel in the stream launch, and
// wait until the previous one has completed (no-ops without the attribute).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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

// Bounded wait: gives up after ~1 s, records OQ_ERR_TIMEOUT and returns false.
static __device__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0 && global_ns() - t0 > kWaitLimitNs) {
      atomicExch(status, OQ_ERR_TIMEOUT);
      return false;
    }
  }
}

// One stage = R = 2P rows; row 2p lands at slot + p*2d, row 2p+1 at slot + HALF + p*2d.
// Warp 0 issues it: lane 0 posts the byte count, then the lanes share the copies.
template <int CFG>
__device__ __forceinline__ void issue_stage_load(const Args& a, uint32_t ring, uint32_t bars, int it, int lane) {
  const int grp = blockIdx.x + it * gridDim.x;
  if (grp >= a.groups || a.stall) return;
  const int slot = it % Cfg<CFG>::STAGES;
  const int R = 2 * a.P;
  const int row0 = grp * R;
  const int nrows = min(R, a.M - row0);
  const uint32_t rowb = (uint32_t)a.d * 2u;
  const uint32_t bar = bars + 8u * slot;
  const uint32_t dst0 = ring + (uint32_t)slot * Cfg<CFG>::IBS;
  if (lane == 0)
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"((uint32_t)nrows * rowb)
                 : "memory");
  __syncwarp();
  for (int r = lane; r < nrows; r += 32) {
    const uint32_t dst = dst0 + (uint32_t)(r & 1) * Cfg<CFG>::HALF + (uint32_t)(r >> 1) * rowb;
    const uint16_t* src = a.X + (size_t)(row0 + r) * a.d;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(rowb), "r"(bar)
        : "memory");
  }
}

// ---- packed f32x2 arithmetic ---------------------------------------------------
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ unsigned long long u2_pack(uint32_t lo, uint32_t hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ void u2_unpack(unsigned long long v, uint32_t& lo, uint32_t& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long f2_sub(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_u128(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

// Stores 32 codes packed in BITS words (code i at bits [i*BITS, (i+1)*BITS)).
template <int BITS>
__device__ __forceinline__ void store_words(uint8_t* dst, const uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else if constexpr (BITS == 6) {
    uint2* p = reinterpret_cast<uint2*>(dst);
    p[0] = make_uint2(w[0], w[1]);
    p[1] = make_uint2(w[2], w[3]);
    p[2] = make_uint2(w[4], w[5]);
  } else {
    uint32_t* p = reinterpret_cast<uint32_t*>(dst);
#pragma unroll
    for (int k = 0; k < BITS; ++k) p[k] = w[k];
  }
}

// Adds code i (low BITS bits of c, higher bits ignored) to the row's words.
// Widths dividing 32: funnel the code in from the top of its word, so after
// the word's last code every code sits at its own position.
template <int BITS>
__device__ __forceinline__ void put_code(uint32_t (&w)[BITS], int i, uint32_t c) {
  if constexpr (32 % BITS == 0) {
    constexpr int PER = 32 / BITS;
    w[i / PER] = __funnelshift_r(w[i / PER], c, BITS);
  } else {
    c &= (1u << BITS) - 1u;
    const int bit = i * BITS, wi = bit >> 5, sh = bit & 31;
    w[wi] |= c << sh;
    if (sh + BITS > 32) w[wi + 1] |= c >> (32 - sh);
  }
}

// Gather step of one stage, for pair buffer BUF (0 or 1; a compile-time
// offset of BUF * IBS on every shared-memory address).
template <int CFG, int LOGHB>
struct Gather {
  // Gathers the 32 pair words of this thread from pair buffer BUF, applies the
  // signs, splits them into f32x2 (row 2p, row 2p+1) and accumulates squares.
  template <int BUF>
  static __device__ __forceinline__ void run(unsigned long long (&v)[32], unsigned long long& ss2,
                                             const uint32_t (&offw)[16], const uint32_t (&sb)[8], uint32_t s_base) {
    unsigned long long sq[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      uint32_t a0, a1;
      if constexpr (Cfg<CFG>::WORD_ADDR) {
        a0 = s_base + ((offw[k] & 0xFFFFu) << 2);
        a1 = s_base + ((offw[k] >> 16) << 2);
      } else {
        a0 = offw[k] & 0xFFFFu;
        a1 = offw[k] >> 16;
      }
      const uint32_t w0 = lds_u32(a0 + BUF * Cfg<CFG>::IBS);
      const uint32_t w1 = lds_u32(a1 + BUF * Cfg<CFG>::IBS);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * k + e;
        const uint32_t w = e ? w1 : w0;
        // sign byte of coordinate i moved to bit 31 (0 or 0x80000000)
        const uint32_t sg = __byte_perm(sb[i >> 2], 0u, 0x0444u | ((uint32_t)(i & 3) << 12));
        const uint32_t ra = (w << 16) + sg;          // row 2p   (add == xor on bit 31)
        const uint32_t rb = (w & 0xFFFF0000u) ^ sg;  // row 2p+1
        v[i] = u2_pack(ra, rb);
        sq[i & 3] = f2_fma(v[i], v[i], sq[i & 3]);
      }
    }
    ss2 = f2_add(f2_add(sq[0], sq[1]), f2_add(sq[2], sq[3]));
  }
};

// Gather step without a permutation (Block-RHT, Full RHT): thread (p, g)
// reads its own 32 columns of both rows of pair p straight from ring slot SLOT
// (no pair buffer, no interleave pass) and applies the signs while widening.
template <int CFG>
struct Direct {
  template <int SLOT>
  static __device__ __forceinline__ void run(unsigned long long (&v)[32], unsigned long long& ss2, uint32_t src,
                                             const uint32_t (&sb)[8]) {
    constexpr uint32_t OFF = SLOT * Cfg<CFG>::IBS, HALF = Cfg<CFG>::HALF;
    unsigned long long sq[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 A = lds_u128(src + OFF + 16u * c);
      const uint4 B = lds_u128(src + OFF + HALF + 16u * c);
      const uint32_t wa[4] = {A.x, A.y, A.z, A.w}, wb[4] = {B.x, B.y, B.z, B.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 8 * c + 2 * m + e;
          const uint32_t sg = __byte_perm(sb[i >> 2], 0u, 0x0444u | ((uint32_t)(i & 3) << 12));
          const uint32_t ra = e ? ((wa[m] & 0xFFFF0000u) ^ sg) : ((wa[m] << 16) + sg);
          const uint32_t rb = e ? ((wb[m] & 0xFFFF0000u) ^ sg) : ((wb[m] << 16) + sg);
          v[i] = u2_pack(ra, rb);
          sq[i & 3] = f2_fma(v[i], v[i], sq[i & 3]);
        }
      }
    }
    ss2 = f2_add(f2_add(sq[0], sq[1]), f2_add(sq[2], sq[3]));
  }
};

// Gather step without a permutation for the block-transposed FWHT: group t of
// lane bl is columns 32 (t ^ bl) + R bl + [0, R) of the block, read for both
// rows of the pair straight from ring slot SLOT (src = the block's first
// column + 2 R bl bytes in slot 0).
template <int CFG, int LOGHB>
struct DirectX {
  template <int SLOT>
  static __device__ __forceinline__ void run(unsigned long long (&v)[32], unsigned long long& ss2, uint32_t src, int bl,
                                             const uint32_t (&sb)[8]) {
    constexpr int L = 1 << LOGHB, R = 32 / L;
    constexpr uint32_t OFF = SLOT * Cfg<CFG>::IBS, HALF = Cfg<CFG>::HALF;
    unsigned long long sq[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int t = 0; t < L; ++t) {
      const uint32_t at = src + OFF + 64u * (uint32_t)(t ^ bl);
      uint32_t wa[R / 2], wb[R / 2];  // R bf16 of each row
      if constexpr (R >= 8) {
#pragma unroll
        for (int c = 0; c < R / 8; ++c) {
          const uint4 A = lds_u128(at + 16u * c), B = lds_u128(at + HALF + 16u * c);
          wa[4 * c] = A.x, wa[4 * c + 1] = A.y, wa[4 * c + 2] = A.z, wa[4 * c + 3] = A.w;
          wb[4 * c] = B.x, wb[4 * c + 1] = B.y, wb[4 * c + 2] = B.z, wb[4 * c + 3] = B.w;
        }
      } else {
        uint32_t x0, x1, y0, y1;
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(x0), "=r"(x1) : "r"(at));
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(y0), "=r"(y1) : "r"(at + HALF));
        wa[0] = x0, wa[1] = x1, wb[0] = y0, wb[1] = y1;
      }
#pragma unroll
      for (int m = 0; m < R / 2; ++m) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = R * t + 2 * m + e;
          const uint32_t sgb = __byte_perm(sb[i >> 2], 0u, 0x0444u | ((uint32_t)(i & 3) << 12));
          const uint32_t ra = e ? ((wa[m] & 0xFFFF0000u) ^ sgb) : ((wa[m] << 16) + sgb);
          const uint32_t rb = e ? ((wb[m] & 0xFFFF0000u) ^ sgb) : ((wb[m] << 16) + sgb);
          v[i] = u2_pack(ra, rb);
          sq[i & 3] = f2_fma(v[i], v[i], sq[i & 3]);
        }
      }
    }
    ss2 = f2_add(f2_add(sq[0], sq[1]), f2_add(sq[2], sq[3]));
  }
};

// Unnormalised Walsh-Hadamard transform (Sylvester order) of the blocks of h =
// 32 << LOGHB coordinates that span lanes 2^LOGHB-aligned: coordinate 32 l + i
// of the block sits in v[i] of lane l (f32x2: both rows of a pair).  Five
// in-thread stages over bits 0..4 of the block index, then LOGHB xor-shuffle
// stages over bits 5.. (the lane bits).
template <int LOGHB>
__device__ __forceinline__ void fwht_pairs(unsigned long long (&v)[32], int lane) {
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & s) == 0) {
        const unsigned long long x0 = v[i], x1 = v[i + s];
        v[i] = f2_add(x0, x1);
        v[i + s] = f2_sub(x0, x1);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < LOGHB; ++k) {
    const float sg = ((lane >> k) & 1) ? -1.0f : 1.0f;
    const unsigned long long sg2 = f2_pack(sg, sg);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float lo, hi;
      f2_unpack(v[i], lo, hi);
      const float olo = __shfl_xor_sync(0xFFFFFFFFu, lo, 1 << k);
      const float ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, 1 << k);
      v[i] = f2_fma(v[i], sg2, f2_pack(olo, ohi));
    }
  }
}

// ---- block-transposed FWHT ------------------------------------------------------
// For blocks of h = 32 L coordinates (L = 2^LOGHB lanes) the lane-crossing
// stages run in-thread too, with one register transpose between two layouts.
// Registers come in L groups of R = 32 / L pairs; lane l of the block holds
//   layout A (after the gather): group t = coordinates 32 (t ^ l) + R l + [0, R)
//   layout B (after the transpose): group u = coordinates 32 l + R (u ^ l) + [0, R)
// A's stages run over bits 5.. of the block coordinate (its group index, XOR-
// relabelled by l), B's over bits 0..4.  Group t of lane l is exactly what lane
// l ^ t needs in B's group t, so the transpose is one xor-shuffle per pair of
// groups t != 0 and group 0 stays in place: (L - 1) R pairs move instead of
// 32 LOGHB, with compile-time register indices.  A stage over a relabelled
// bit s swaps the roles of the two inputs in lanes whose bit s of l is set;
// that is folded into a sign, so both outputs are one FMA each:
//   x0' = x0 * sg + x1,   x1' = x0 - x1 * sg   (sg = -1 where bit s of l is 1).
template <int BITS, int LOGHB>
struct Xch {
  static constexpr int L = 1 << LOGHB, R = 32 / L, LOGR = 5 - LOGHB;
  static constexpr int CB = R * BITS;  // bits of one group's codes
  // The packed codes of a group are moved between positions u and u ^ l; each
  // level k swaps neighbouring runs of CB << k bits, which this supports when
  // every run is whole words, a half / byte / nibble of a word, or half of a
  // three-word group (48 bits, 3- and 6-bit codes).
  static constexpr bool level_ok(int S) {
    return S % 32 == 0 || S == 16 || S == 8 || S == 4 || (S == 48 && BITS % 3 == 0);
  }
  static constexpr bool ok() {
    bool r = LOGHB >= 1 && LOGHB <= 3;
    for (int k = 0; k < 3; ++k) r = r && (k >= LOGHB || level_ok(CB << k));
    return r;
  }
};

// The relabelled stages over the group index of a layout (A or B).
template <int LOGHB>
__device__ __forceinline__ void groups_stages(unsigned long long (&v)[32], const unsigned long long (&sg)[3],
                                              const unsigned long long (&nsg)[3]) {
  constexpr int L = 1 << LOGHB, R = 32 / L;
#pragma unroll
  for (int s = 0; s < LOGHB; ++s) {
#pragma unroll
    for (int t = 0; t < L; ++t) {
      if ((t >> s) & 1) continue;
      const int t1 = t | (1 << s);
#pragma unroll
      for (int b = 0; b < R; ++b) {
        const unsigned long long x0 = v[R * t + b], x1 = v[R * t1 + b];
        v[R * t + b] = f2_fma(x0, sg[s], x1);
        v[R * t1 + b] = f2_fma(x1, nsg[s], x0);
      }
    }
  }
}

template <int LOGHB>
__device__ __forceinline__ void fwht_xch(unsigned long long (&v)[32], const unsigned long long (&sg)[3],
                                         const unsigned long long (&nsg)[3]) {
  constexpr int L = 1 << LOGHB, R = 32 / L;
  groups_stages<LOGHB>(v, sg, nsg);  // layout A: coordinate bits 5 .. 4 + LOGHB
#pragma unroll
  for (int t = 1; t < L; ++t) {
#pragma unroll
    for (int b = 0; b < R; ++b) {
      float lo, hi;
      f2_unpack(v[R * t + b], lo, hi);
      lo = __shfl_xor_sync(0xFFFFFFFFu, lo, t);
      hi = __shfl_xor_sync(0xFFFFFFFFu, hi, t);
      v[R * t + b] = f2_pack(lo, hi);
    }
  }
  // layout B: coordinate bits 0 .. 4 - LOGHB (standard), then the group bits
#pragma unroll
  for (int s = 1; s < R; s <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & s) == 0) {
        const unsigned long long x0 = v[i], x1 = v[i + s];
        v[i] = f2_add(x0, x1);
        v[i + s] = f2_sub(x0, x1);
      }
    }
  }
  groups_stages<LOGHB>(v, sg, nsg);
}

// Swaps every pair of neighbouring runs of S bits of the packed row when sw.
template <int BITS, int S>
__device__ __forceinline__ void swap_runs(uint32_t (&w)[BITS], bool sw) {
  if constexpr (S % 32 == 0) {
    constexpr int WS = S / 32;
#pragma unroll
    for (int c = 0; c < BITS; c += 2 * WS) {
#pragma unroll
      for (int j = 0; j < WS; ++j) {
        const uint32_t a = w[c + j], b = w[c + WS + j];
        w[c + j] = sw ? b : a;
        w[c + WS + j] = sw ? a : b;
      }
    }
  } else if constexpr (S == 48) {  // halves of each three-word group
#pragma unroll
    for (int c = 0; c < BITS; c += 3) {
      const uint32_t m0 = __byte_perm(w[c + 1], w[c + 2], 0x5432), m1 = __byte_perm(w[c + 2], w[c], 0x5432),
                     m2 = __byte_perm(w[c], w[c + 1], 0x5432);
      w[c] = sw ? m0 : w[c];
      w[c + 1] = sw ? m1 : w[c + 1];
      w[c + 2] = sw ? m2 : w[c + 2];
    }
  } else if constexpr (S == 16 || S == 8) {
    const uint32_t sel = sw ? (S == 16 ? 0x1032u : 0x2301u) : 0x3210u;
#pragma unroll
    for (int j = 0; j < BITS; ++j) w[j] = __byte_perm(w[j], 0u, sel);
  } else {
    static_assert(S == 4, "unsupported run width");
#pragma unroll
    for (int j = 0; j < BITS; ++j) {
      const uint32_t x = ((w[j] >> 4) & 0x0F0F0F0Fu) | ((w[j] & 0x0F0F0F0Fu) << 4);
      w[j] = sw ? x : w[j];
    }
  }
}

// Moves the packed codes of group u (CB bits at u * CB) to group u ^ l: level
// k swaps runs of CB << k bits where bit k of l is set.
template <int BITS, int LOGHB, int K = 0>
__device__ __forceinline__ void xor_groups(uint32_t (&w)[BITS], int l) {
  if constexpr (K < LOGHB) {
    swap_runs<BITS, (Xch<BITS, LOGHB>::CB << K)>(w, ((l >> K) & 1) != 0);
    xor_groups<BITS, LOGHB, K + 1>(w, l);
  }
}

// Centroid search and packing of the 32 coordinates of both rows held in v:
// y = sat(x * A + 1/2) (A folds the row scale and 1/sqrt(h) into the table's
// alpha), bucket q = round(y * nb) read from the low mantissa bits of
// fma(y, nb, 1.5 * 2^23), table entry q = the bucket's boundary with the codes
// below it in its low bits, code = entry + (y > boundary) from the sign of
// (boundary - y); qkey is the table's shared address minus the bucket key of
// q = 0.  wa / wb receive the packed codes of rows a / b.
template <int BITS>
__device__ __forceinline__ void search_pack(const unsigned long long (&v)[32], float A_a, float A_b, float nb,
                                            uint32_t qkey, uint32_t (&wa)[BITS], uint32_t (&wb)[BITS]) {
  const unsigned long long NB2 = f2_pack(nb, nb);
  const unsigned long long C2 = f2_pack(12582912.0f, 12582912.0f);  // 1.5 * 2^23
#pragma unroll
  for (int k = 0; k < BITS; ++k) wa[k] = wb[k] = 0u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float xa, xb;
    f2_unpack(v[i], xa, xb);
    const float ya = fma_sat(xa, A_a, 0.5f), yb = fma_sat(xb, A_b, 0.5f);
    const unsigned long long y1 = f2_pack(ya, yb);
    uint32_t qa, qb;
    u2_unpack(f2_fma(y1, NB2, C2), qa, qb);
    const uint32_t ea = lds_u32((qa << 2) + qkey), eb = lds_u32((qb << 2) + qkey);
    uint32_t da, db;
    u2_unpack(f2_sub(u2_pack(ea, eb), y1), da, db);
    put_code<BITS>(wa, i, ea + (da >> 31));
    put_code<BITS>(wb, i, eb + (db >> 31));
  }
}

// Per-thread constants of the kernel (all registers).
struct Thread {
  int tid, lane, pr, g, spr, nparts;
  bool active;
  uint32_t s_base, s_bars, s_ring, qkey;
  uint32_t src_pair;  // ring: row 2pr, columns 32g.., with the lane's chunk rotation
  uint32_t src_direct;  // ring slot 0: row 2pr, columns 32g.. (no rotation)
  uint32_t ib_w0, ib_w1;
  float2* partial;
  int bl;                          // lane within the Hadamard block (block-transposed FWHT)
  uint32_t src_blk;                // ring slot 0: row 2pr, start of the block + 2 R bl (no permutation)
  unsigned long long sg[3], nsg[3];  // (s, s) and (-s, -s), s = -1 where bit k of bl is set
};

// Interleave stage `it` (ring slot it % STAGES) into pair buffer it & 1.
template <int CFG>
__device__ __forceinline__ bool interleave(const Args& a, const Thread& t, int it) {
  constexpr uint32_t IBS = Cfg<CFG>::IBS, HALF = Cfg<CFG>::HALF;
  const int slot = it % Cfg<CFG>::STAGES;
  const uint32_t parity = (uint32_t)(it / Cfg<CFG>::STAGES) & 1u;
  if (!mbar_wait_bounded(t.s_bars + 8u * slot, parity, a.status)) return false;
  const uint32_t src = t.s_ring + (uint32_t)slot * IBS + t.src_pair;
  const uint32_t boff = (uint32_t)(it & 1) * IBS;
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const uint32_t s_a = src ^ (16u * n);
    const uint4 A = lds_u128(s_a);
    const uint4 B = lds_u128(s_a + HALF);
    sts_u128((t.ib_w0 ^ (32u * n)) + boff, __byte_perm(A.x, B.x, 0x5410), __byte_perm(A.x, B.x, 0x7632),
             __byte_perm(A.y, B.y, 0x5410), __byte_perm(A.y, B.y, 0x7632));
    sts_u128((t.ib_w1 ^ (32u * n)) + boff, __byte_perm(A.z, B.z, 0x5410), __byte_perm(A.z, B.z, 0x7632),
             __byte_perm(A.w, B.w, 0x5410), __byte_perm(A.w, B.w, 0x7632));
  }
  return true;
}

// Gather + signs + FWHT of stage `it`, and the segment partials of its squared norms.
template <int BITS, int LOGHB, int CFG, bool PERM>
__device__ __forceinline__ void transform(const Args& a, const Thread& t, int it, unsigned long long (&v)[32],
                                          const uint32_t (&offw)[16], const uint32_t (&sb)[8]) {
  constexpr bool XCH = Xch<BITS, LOGHB>::ok();
  unsigned long long ss2;
  if constexpr (PERM) {
    if (it & 1)
      Gather<CFG, LOGHB>::template run<1>(v, ss2, offw, sb, t.s_base);
    else
      Gather<CFG, LOGHB>::template run<0>(v, ss2, offw, sb, t.s_base);
  } else if constexpr (XCH) {
    static_assert(Cfg<CFG>::STAGES <= 2, "slot offsets are unrolled for two slots");
    if (it % Cfg<CFG>::STAGES == 1)
      DirectX<CFG, LOGHB>::template run<1>(v, ss2, t.src_blk, t.bl, sb);
    else
      DirectX<CFG, LOGHB>::template run<0>(v, ss2, t.src_blk, t.bl, sb);
  } else {
    static_assert(Cfg<CFG>::STAGES <= 2, "slot offsets are unrolled for two slots");
    if (it % Cfg<CFG>::STAGES == 1)
      Direct<CFG>::template run<1>(v, ss2, t.src_direct, sb);
    else
      Direct<CFG>::template run<0>(v, ss2, t.src_direct, sb);
  }
  {
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      if (k < a.seg_log) {
        float lo, hi;
        f2_unpack(ss2, lo, hi);
        ss2 = f2_add(ss2, f2_pack(__shfl_xor_sync(0xFFFFFFFFu, lo, 1 << k), __shfl_xor_sync(0xFFFFFFFFu, hi, 1 << k)));
      }
    }
    float lo, hi;
    f2_unpack(ss2, lo, hi);
    if ((t.lane & ((1 << a.seg_log) - 1)) == 0)
      t.partial[(it & 1) * t.nparts + (t.tid >> a.seg_log)] = make_float2(lo, hi);
  }
  if constexpr (XCH)
    fwht_xch<LOGHB>(v, t.sg, t.nsg);
  else
    fwht_pairs<LOGHB>(v, t.lane);
}

// Normalise, search, pack and store stage `it`.
template <int BITS, int LOGHB>
__device__ __forceinline__ void quantize(const Args& a, const Thread& t, int it, const unsigned long long (&v)[32]) {
  constexpr bool XCH = Xch<BITS, LOGHB>::ok();
  const int R = 2 * a.P;
  const int grp = blockIdx.x + it * gridDim.x;
  const int row0 = grp * R;
  const int nrows = min(R, a.M - row0);
  const bool row_a = t.active && 2 * t.pr < nrows, row_b = t.active && 2 * t.pr + 1 < nrows;
  if (!row_a) return;
  float sum_a = 0.0f, sum_b = 0.0f;
  {
    const float2* src = t.partial + (it & 1) * t.nparts + ((t.pr * t.spr) >> a.seg_log);
    const int cnt = t.spr >> a.seg_log;
    for (int k = 0; k < cnt; ++k) {
      const float2 p = src[k];
      sum_a += p.x;
      sum_b += p.y;
    }
  }
  const float A_a = sum_a > 0.0f ? a.alpha_h * rsqrtf(sum_a) : 0.0f;
  const float A_b = sum_b > 0.0f ? a.alpha_h * rsqrtf(sum_b) : 0.0f;
  uint32_t wa[BITS], wb[BITS];
  search_pack<BITS>(v, A_a, A_b, a.nb, t.qkey, wa, wb);
  if constexpr (XCH) {  // register group u holds the codes of group u ^ bl
    xor_groups<BITS, LOGHB>(wa, t.bl);
    xor_groups<BITS, LOGHB>(wb, t.bl);
  }
  const int row = row0 + 2 * t.pr;
  const size_t rb = (size_t)(a.d / 8 * BITS);
  uint8_t* dst = a.codes + (size_t)row * rb + (size_t)t.g * (4 * BITS);
  store_words<BITS>(dst, wa);
  if (row_b) store_words<BITS>(dst + rb, wb);
  if (t.g == 0) {
    const float s_a = sqrtf(sum_a), s_b = sqrtf(sum_b);
    if (a.norm_f32) {
      a.norm_f32[row] = s_a;
      if (row_b) a.norm_f32[row + 1] = s_b;
    }
    if (a.norm_bf16) {
      const __nv_bfloat16 ha = __float2bfloat16_rn(s_a), hb = __float2bfloat16_rn(s_b);
      a.norm_bf16[row] = *reinterpret_cast<const uint16_t*>(&ha);
      if (row_b) a.norm_bf16[row + 1] = *reinterpret_cast<const uint16_t*>(&hb);
    }
  }
}

template <int BITS, int LOGHB, int CFG, bool PERM>
__global__ void __launch_bounds__(CFG == 2 ? 512 : 384, 1) rotq_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  pdl_launch_dependents();
  const int d = a.d, P = a.P;
  Thread t;
  t.tid = threadIdx.x;
  t.lane = t.tid & 31;
  const int warp = t.tid >> 5;
  t.spr = d >> 5;  // 32-coordinate segments per row
  t.active = t.tid < P * t.spr;
  t.pr = t.active ? t.tid / t.spr : 0;  // row pair (inactive threads shadow pair 0, never store)
  t.g = t.active ? t.tid - t.pr * t.spr : 0;
  t.nparts = (int)(blockDim.x >> a.seg_log);
  t.s_base = smem_u32(smem);
  t.s_bars = t.s_base + a.bar_off;
  t.s_ring = t.s_base + a.ring_off;
  t.partial = reinterpret_cast<float2*>(smem + a.part_off);
  uint32_t* qtab = reinterpret_cast<uint32_t*>(smem + a.qt_off);
  t.qkey = smem_u32(qtab) - 0x2D000000u;  // = qtab - 4 * bits(1.5 * 2^23)

  // The address arithmetic below relies on a 128-byte aligned shared window
  // base and (byte-address forms) on every pair-buffer address fitting 16 bits.
  if ((t.s_base & 127u) != 0u || (!Cfg<CFG>::WORD_ADDR && t.s_base + 4u * (uint32_t)(P * d) > 0xFFFFu)) {
    if (t.tid == 0) atomicExch(a.status, OQ_ERR_UNSUPPORTED);
    return;
  }

  if (t.tid == 0) {
    for (int s = 0; s < Cfg<CFG>::STAGES; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(t.s_bars + 8u * s) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // The first stages' copies start now, so their HBM latency overlaps the
  // table loads below (only warp 0, which made the barriers, touches them
  // before the CTA barrier).  X may be written by the previous kernel in the
  // stream, and the codes and norms read by it: warp 0 waits for that kernel
  // first (every other thread's global accesses before the CTA barrier are
  // to the handles' tables; its writes come after data that warp 0 requested).
  if (warp == 0) {
    pdl_wait();
    __syncwarp();
    for (int s = 0; s < Cfg<CFG>::STAGES; ++s) issue_stage_load<CFG>(a, t.s_ring, t.s_bars, s, t.lane);
  }
  for (int k = t.tid; k < a.qtable_len; k += blockDim.x) qtab[k] = __ldg(a.qtable + k);

  // gather addresses: pair word of column c of pair pr sits at word
  // pr*d + swz(c) of a pair buffer, swz swapping the 16-byte halves of odd
  // 32-column segments (conflict-free interleave stores)
  // Register r of a thread holds coordinate col(r) of its row pair: 32 g + r,
  // or, with the block-transposed FWHT, layout A's
  // 32 (g - bl) + 32 ((r / XR) ^ bl) + XR bl + r % XR.
  constexpr bool XCH = Xch<BITS, LOGHB>::ok();
  constexpr int XR = XCH ? (32 >> LOGHB) : 32;
  t.bl = XCH ? (t.g & ((1 << LOGHB) - 1)) : 0;
  auto col = [&](int r) -> uint32_t {
    return 32u * (uint32_t)(t.g - t.bl) + 32u * (uint32_t)((r / XR) ^ t.bl) + (uint32_t)(XR * t.bl + r % XR);
  };
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const float sgn = ((t.bl >> k) & 1) ? -1.0f : 1.0f;
    t.sg[k] = f2_pack(sgn, sgn);
    t.nsg[k] = f2_pack(-sgn, -sgn);
  }
  t.src_blk = t.s_ring + (uint32_t)t.pr * (uint32_t)d * 2u + 64u * (uint32_t)(t.g - t.bl) + 2u * (uint32_t)(XR * t.bl);
  uint32_t offw[16];
  if constexpr (PERM) {
    const uint32_t rowbase = (uint32_t)t.pr * (uint32_t)d;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t pw = __ldg(a.perm2 + (col(2 * k) >> 1));  // col(2k) is even, col(2k + 1) = col(2k) + 1
      uint32_t c0 = pw & 0xFFFFu, c1 = pw >> 16;
      c0 ^= ((c0 >> 5) & 1u) << 2;
      c1 ^= ((c1 >> 5) & 1u) << 2;
      uint32_t o0 = rowbase + c0, o1 = rowbase + c1;  // word indices
      if constexpr (!Cfg<CFG>::WORD_ADDR) {
        o0 = t.s_base + 4u * o0;
        o1 = t.s_base + 4u * o1;
      }
      offw[k] = (o0 & 0xFFFFu) | (o1 << 16);
    }
  }
  // sign bytes: byte m of sb[q] is 0x80 when coordinate col(4q + m) is negated
  // (a register group's coordinates share one sign word)
  uint32_t sb[8];
  {
    uint32_t sw[32 / XR];
#pragma unroll
    for (int t2 = 0; t2 < 32 / XR; ++t2) sw[t2] = __ldg(a.signs + (col(XR * t2) >> 5));
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t x = 0;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = 4 * q + m;
        x |= ((sw[r / XR] >> (col(r) & 31u)) & 1u) << (8 * m + 7);
      }
      sb[q] = x;
    }
  }
  // interleave addresses: 16-byte chunk c = n ^ rot of the thread's 32 columns
  // (lane-rotated, conflict-free ring reads); odd segments swap halves
  {
    const uint32_t rot16 = (uint32_t)((t.g >> 1) & 3) << 4;
    t.src_pair = ((uint32_t)t.pr * (uint32_t)d * 2u + (uint32_t)t.g * 64u) ^ rot16;
    const uint32_t ib_seg = t.s_base + 4u * ((uint32_t)t.pr * (uint32_t)d + 32u * (uint32_t)t.g);
    const uint32_t h0 = (uint32_t)(t.g & 1) << 4;
    t.ib_w0 = (ib_seg + h0) ^ (rot16 << 1);
    t.ib_w1 = (ib_seg + (16u - h0)) ^ (rot16 << 1);
    t.src_direct = t.s_ring + (uint32_t)t.pr * (uint32_t)d * 2u + (uint32_t)t.g * 64u;
  }
  __syncthreads();

  const int n_it = a.groups > (int)blockIdx.x ? (a.groups - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  if (n_it == 0) return;
  unsigned long long v[32];

  if constexpr (PERM) {
    // prologue: stage 0
    bool ok = interleave<CFG>(a, t, 0);
    if (__syncthreads_or(!ok)) return;
    if (warp == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_stage_load<CFG>(a, t.s_ring, t.s_bars, Cfg<CFG>::STAGES, t.lane);
    }
    transform<BITS, LOGHB, CFG, PERM>(a, t, 0, v, offw, sb);
    for (int it = 0; it < n_it; ++it) {
      const bool more = it + 1 < n_it;
      ok = more ? interleave<CFG>(a, t, it + 1) : true;
      if (__syncthreads_or(!ok)) return;  // partials of `it`, pair buffer of it+1, ring slot released
      if (more && warp == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_stage_load<CFG>(a, t.s_ring, t.s_bars, it + 1 + Cfg<CFG>::STAGES, t.lane);
      }
      quantize<BITS, LOGHB>(a, t, it, v);
      if (more) transform<BITS, LOGHB, CFG, PERM>(a, t, it + 1, v, offw, sb);
    }
  } else {
    // no permutation: each stage is read straight from its ring slot, which is
    // released at the barrier that follows its transform
    bool ok = mbar_wait_bounded(t.s_bars, 0u, a.status);
    if (ok) transform<BITS, LOGHB, CFG, PERM>(a, t, 0, v, offw, sb);
    for (int it = 0; it < n_it; ++it) {
      if (__syncthreads_or(!ok)) return;  // partials of `it`; ring slot of `it` released
      if (warp == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_stage_load<CFG>(a, t.s_ring, t.s_bars, it + Cfg<CFG>::STAGES, t.lane);
      }
      quantize<BITS, LOGHB>(a, t, it, v);
      if (it + 1 < n_it) {
        const int nx = it + 1;
        ok = mbar_wait_bounded(t.s_bars + 8u * (nx % Cfg<CFG>::STAGES), (uint32_t)(nx / Cfg<CFG>::STAGES) & 1u,
                               a.status);
        if (ok) transform<BITS, LOGHB, CFG, PERM>(a, t, nx, v, offw, sb);
      }
    }
  }
}

using KernelFn = void (*)(Args);

// Kernels of configuration CFG for bits 1..6 and log2(h/32) 0..5 (nullptr otherwise),
// with (RPBH) or without (Block-RHT, Full RHT) the permutation.
KernelFn pick_cfg0(int bits, int loghb);
KernelFn pick_cfg1(int bits, int loghb);
KernelFn pick_cfg2(int bits, int loghb);
KernelFn pick_cfg0_np(int bits, int loghb);
KernelFn pick_cfg1_np(int bits, int loghb);
KernelFn pick_cfg2_np(int bits, int loghb);

#define OQ_ROTQ_DEFINE_PICK(NAME, CFG, PERM)                \
  template <int BITS>                                       \
  static KernelFn NAME##_loghb(int loghb) {                 \
    switch (loghb) {                                        \
      case 0: return rotq_kernel<BITS, 0, CFG, PERM>;       \
      case 1: return rotq_kernel<BITS, 1, CFG, PERM>;       \
      case 2: return rotq_kernel<BITS, 2, CFG, PERM>;       \
      case 3: return rotq_kernel<BITS, 3, CFG, PERM>;       \
      case 4: return rotq_kernel<BITS, 4, CFG, PERM>;       \
      case 5: return rotq_kernel<BITS, 5, CFG, PERM>;       \
    }                                                       \
    return nullptr;                                         \
  }                                                         \
  KernelFn NAME(int bits, int loghb) {                      \
    switch (bits) {                                         \
      case 1: return NAME##_loghb<1>(loghb);                \
      case 2: return NAME##_loghb<2>(loghb);                \
      case 3: return NAME##_loghb<3>(loghb);                \
      case 4: return NAME##_loghb<4>(loghb);                \
      case 5: return NAME##_loghb<5>(loghb);                \
      case 6: return NAME##_loghb<6>(loghb);                \
    }                                                       \
    return nullptr;                                         \
  }

}  // namespace rotq
}  // namespace oq
