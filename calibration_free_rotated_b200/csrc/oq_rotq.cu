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
// Design (HBM-bound; every step below is sized to keep the SM's issue slots and
// shared-memory wavefronts under the HBM time of a row):
//   * Persistent CTAs.  A stage is R = 2P rows (P row pairs, P = max(1, 8192/d)).
//     A 3-deep ring of stage buffers is filled by 1-D bulk async copies
//     (cp.async.bulk + mbarrier transaction counts).
//   * Interleave pass: each landed stage is rewritten so that word j of row pair
//     p holds (x[2p][j], x[2p+1][j]); one 32-bit gather then feeds both rows.
//   * Thread t owns row pair p = t div (d/32) and segment g = t mod (d/32)
//     (output coordinates j = 32 g .. 32 g + 31 of both rows).  Its 32 gather
//     offsets pi(j) and 32 sign bits stay in registers.
//   * The Rademacher sign is applied while splitting the gathered word into two
//     floats; the two rows travel as f32x2 pairs, so the FWHT butterflies, the
//     sum of squares and the scaling run as packed f32x2 instructions.
//   * FWHT: 5 butterfly stages inside the thread, then log2(h/32) xor-shuffle
//     stages across the h/32 lanes of a block.
//   * Row norms from the gathered values (||Pi x|| = ||x||), reduced in a fixed
//     order (deterministic).
//   * Centroid search: y = fma(t, G, C) leaves the bucket index in y's low
//     mantissa bits; one shared-memory table load gives the bucket's only
//     boundary with the count of boundaries below it in its low bits, and one
//     compare finishes: code = (e & (2^b - 1)) + (t > e).  Ties take the lower
//     centroid.  (The host builds the table; see build_qtable.)
//   * The 32 codes of a segment fill exactly b 32-bit words per row, stored
//     with vector stores (coalesced across the warp).
//   * Every mbarrier wait is bounded (~1 s) and reports OQ_ERR_TIMEOUT.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "oq_internal.h"

namespace oq {
namespace {

constexpr int kMaxStages = 3;
constexpr int kPairElems = 8192;  // d * P per stage (elements per row of the pair)
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

struct RotqArgs {
  const uint16_t* X;
  uint8_t* codes;
  float* norm_f32;
  uint16_t* norm_bf16;
  const uint16_t* perm;
  const uint32_t* signs;
  const uint32_t* qtable;
  int* status;
  int M, d, P, groups, pairs_per_warp, qtable_len, stages;
  float inv_sqrt_h;
  float qt_scale, qt_offset;
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

// Bounded wait: gives up after ~1 s, records OQ_ERR_TIMEOUT and returns false.
__device__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int* status) {
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

__device__ __forceinline__ void issue_stage_load(const RotqArgs& a, uint32_t ring, uint32_t bars, int it) {
  const int grp = blockIdx.x + it * gridDim.x;
  if (grp >= a.groups) return;
  const int slot = it % a.stages;
  const int R = 2 * a.P;
  const int row0 = grp * R;
  const int nrows = min(R, a.M - row0);
  const uint32_t bytes = (uint32_t)nrows * (uint32_t)a.d * 2u;
  const uint32_t bar = bars + 8u * slot;
  const uint32_t dst = ring + (uint32_t)slot * (uint32_t)R * (uint32_t)a.d * 2u;
  const uint16_t* src = a.X + (size_t)row0 * a.d;
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// ---- packed f32x2 arithmetic ---------------------------------------------------
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
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

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

// Code of one value: bucket from y's bits, one table entry, one compare.  The
// bucket index is clamped so that a non-finite input cannot read past the table.
template <int BITS>
__device__ __forceinline__ uint32_t code_of(float t, float y, uint32_t qt_base, uint32_t qt_last) {
  constexpr uint32_t LOW = (1u << BITS) - 1u;
  const uint32_t q = min(__float_as_uint(y) - 0x4B400000u, qt_last);  // bits(y) - bits(1.5 * 2^23)
  const uint32_t e = lds_u32(qt_base + 4u * q);
  return (e & LOW) + (t > __uint_as_float(e) ? 1u : 0u);
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

template <int BITS>
__device__ __forceinline__ void put_code(uint32_t (&w)[BITS], int i, uint32_t c) {
  const int bit = i * BITS, wi = bit >> 5, sh = bit & 31;
  w[wi] |= c << sh;
  if (sh + BITS > 32) w[wi + 1] |= c >> (32 - sh);
}

template <int BITS, int LOGHB>
__global__ void __launch_bounds__(512, 1) rotq_kernel(const __grid_constant__ RotqArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int d = a.d, P = a.P, R = 2 * P;
  const int nwarps = blockDim.x >> 5;
  // layout: bars | partial[2][nwarps][ppw][2] | qtable | ibuf[P][d] u32 | ring[stages][R][d] u16
  const uint32_t s_bars = smem_u32(smem);
  float* partial = reinterpret_cast<float*>(smem + 64);
  const size_t part_bytes = ((size_t)2 * nwarps * a.pairs_per_warp * 2 * 4 + 127) & ~(size_t)127;
  uint32_t* qtab = reinterpret_cast<uint32_t*>(smem + 64 + part_bytes);
  const size_t qt_bytes = ((size_t)a.qtable_len * 4 + 127) & ~(size_t)127;
  unsigned char* ibuf = smem + 64 + part_bytes + qt_bytes;
  const uint32_t s_ibuf = smem_u32(ibuf);
  const uint32_t s_ring = s_ibuf + (uint32_t)P * (uint32_t)d * 4u;
  const uint32_t s_qtab = smem_u32(qtab);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int spr = d >> 5;  // segments per row
  const bool active = tid < P * spr;
  const int pr = active ? tid / spr : P;  // row pair (inactive threads: past the last)
  const int g = active ? tid - pr * spr : 0;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(s_bars + 8u * s) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int k = tid; k < a.qtable_len; k += blockDim.x) qtab[k] = __ldg(a.qtable + k);

  // gather offsets: byte offsets inside ibuf, (pr * d + pi(j)) * 4; reloaded per
  // stage from the (L1-resident) permutation so they do not hold registers
  const uint4* perm4 = reinterpret_cast<const uint4*>(a.perm + 32 * g);
  const uint32_t obase = 4u * (uint32_t)(active ? pr : 0) * (uint32_t)d;
  const uint32_t sw = __ldg(a.signs + g);
  const unsigned long long G2 = f2_pack(a.qt_scale, a.qt_scale);
  const unsigned long long C2 = f2_pack(a.qt_offset, a.qt_offset);
  const uint32_t qt_last = (uint32_t)a.qtable_len - 1u;
  __syncthreads();

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) issue_stage_load(a, s_ring, s_bars, s);
  }

  for (int it = 0;; ++it) {
    const int grp = blockIdx.x + it * gridDim.x;
    if (grp >= a.groups) break;
    const int slot = it % a.stages;
    const uint32_t parity = (uint32_t)(it / a.stages) & 1u;
    if (!mbar_wait_bounded(s_bars + 8u * slot, parity, a.status)) return;
    const int row0 = grp * R;
    const int nrows = min(R, a.M - row0);

    // interleave pass: natural rows (ring slot) -> word j of pair p = (x[2p][j], x[2p+1][j]).
    // Unit = 4 columns of a pair: two 8-byte loads, one 16-byte store; consecutive
    // lanes touch consecutive addresses (no bank conflicts).
    {
      const uint32_t src = s_ring + (uint32_t)slot * (uint32_t)R * (uint32_t)d * 2u;
      for (int p = 0; p < P; ++p) {
        const bool va = 2 * p < nrows, vb = 2 * p + 1 < nrows;
        const uint32_t ra0 = src + (uint32_t)(2 * p) * (uint32_t)d * 2u;
        const uint32_t dp = s_ibuf + (uint32_t)p * (uint32_t)d * 4u;
        for (int k = tid; k < (d >> 2); k += blockDim.x) {
          uint32_t a0 = 0, a1 = 0, b0 = 0, b1 = 0;
          if (va) asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(a0), "=r"(a1) : "r"(ra0 + 8u * k));
          if (vb)
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(ra0 + (uint32_t)d * 2u + 8u * k));
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dp + 16u * k), "r"(__byte_perm(a0, b0, 0x5410)),
                       "r"(__byte_perm(a0, b0, 0x7632)), "r"(__byte_perm(a1, b1, 0x5410)),
                       "r"(__byte_perm(a1, b1, 0x7632))
                       : "memory");
        }
      }
    }
    __syncthreads();  // ibuf ready; the ring slot is free again
    if (tid == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_stage_load(a, s_ring, s_bars, it + a.stages);
    }

    // gather (permutation) + signs -> f32x2 pairs (row 2p, row 2p+1), sums of squares
    unsigned long long v[32];
    unsigned long long ss2 = 0ull;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 pq = __ldg(perm4 + q);
      const uint32_t pw[4] = {pq.x, pq.y, pq.z, pq.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = 8 * q + k;
        const uint32_t pj = (k & 1) ? (pw[k >> 1] >> 16) : (pw[k >> 1] & 0xFFFFu);
        const uint32_t w = lds_u32(s_ibuf + obase + 4u * pj);
        const uint32_t sgn = ((sw >> i) & 1u) << 31;
        v[i] = f2_pack(__uint_as_float((w << 16) ^ sgn), __uint_as_float((w & 0xFFFF0000u) ^ sgn));
        ss2 = f2_fma(v[i], v[i], ss2);
      }
    }

    // per-warp partial sums of every row pair this warp touches (fixed order)
    const int par = it & 1;
    {
      float s_lo, s_hi;
      f2_unpack(ss2, s_lo, s_hi);
      const int wp0 = (warp * 32) / spr;
      const int wp1 = min((warp * 32 + 31) / spr, P - 1);
      for (int p = wp0; p <= wp1; ++p) {
        const bool mine = active && pr == p;
        const float x0 = warp_sum(mine ? s_lo : 0.0f);
        const float x1 = warp_sum(mine ? s_hi : 0.0f);
        if (lane == 0) {
          float* dst = partial + ((par * nwarps + warp) * a.pairs_per_warp + (p - wp0)) * 2;
          dst[0] = x0;
          dst[1] = x1;
        }
      }
    }
    __syncthreads();  // every gather from ibuf is done; partials visible

    // in-thread Walsh-Hadamard butterflies over bits 0..4 of the block index
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
    // across the h/32 lanes of a block: bits 5.. of the block index
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

    const bool row_a = active && 2 * pr < nrows, row_b = active && 2 * pr + 1 < nrows;
    if (!row_a) continue;
    // row norms from the partials of the warps covering this pair, in order
    float sum_a = 0.0f, sum_b = 0.0f;
    {
      const int w_lo = (pr * spr) >> 5, w_hi = (pr * spr + spr - 1) >> 5;
      for (int w = w_lo; w <= w_hi; ++w) {
        const int p0 = (w * 32) / spr;
        const float* src = partial + ((par * nwarps + w) * a.pairs_per_warp + (pr - p0)) * 2;
        sum_a += src[0];
        sum_b += src[1];
      }
    }
    const float s_a = sqrtf(sum_a), s_b = sqrtf(sum_b);
    const unsigned long long scale2 = f2_pack(a.inv_sqrt_h / (s_a + 1e-12f), a.inv_sqrt_h / (s_b + 1e-12f));

    uint32_t wa[BITS], wb[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) wa[k] = wb[k] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const unsigned long long t2 = f2_mul(v[i], scale2);
      const unsigned long long y2 = f2_fma(t2, G2, C2);
      float ta, tb, ya, yb;
      f2_unpack(t2, ta, tb);
      f2_unpack(y2, ya, yb);
      put_code<BITS>(wa, i, code_of<BITS>(ta, ya, s_qtab, qt_last));
      put_code<BITS>(wb, i, code_of<BITS>(tb, yb, s_qtab, qt_last));
    }
    const int row = row0 + 2 * pr;
    const size_t rb = (size_t)(d / 8 * BITS);
    uint8_t* dst = a.codes + (size_t)row * rb + (size_t)g * (4 * BITS);
    store_words<BITS>(dst, wa);
    if (row_b) store_words<BITS>(dst + rb, wb);
    if (g == 0) {
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
}

using RotqKernel = void (*)(RotqArgs);

template <int BITS>
RotqKernel pick_loghb(int loghb) {
  switch (loghb) {
    case 0: return rotq_kernel<BITS, 0>;
    case 1: return rotq_kernel<BITS, 1>;
    case 2: return rotq_kernel<BITS, 2>;
    case 3: return rotq_kernel<BITS, 3>;
    case 4: return rotq_kernel<BITS, 4>;
    case 5: return rotq_kernel<BITS, 5>;
  }
  return nullptr;
}

RotqKernel pick_kernel(int bits, int loghb) {
  switch (bits) {
    case 1: return pick_loghb<1>(loghb);
    case 2: return pick_loghb<2>(loghb);
    case 3: return pick_loghb<3>(loghb);
    case 4: return pick_loghb<4>(loghb);
    case 5: return pick_loghb<5>(loghb);
    case 6: return pick_loghb<6>(loghb);
  }
  return nullptr;
}

}  // namespace

int launch_rotq(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, uint8_t* codes, float* norm_f32,
                uint16_t* norm_bf16, void* stream) {
  const int d = r->d, h = r->h, bits = cb->bits;
  int loghb = 0;
  while ((32 << loghb) < h) ++loghb;
  RotqKernel kern = pick_kernel(bits, loghb);
  if (!kern) return fail(OQ_ERR_UNSUPPORTED, "no rotate+quantize kernel for bits=%d h=%d", bits, h);

  const uint16_t* perm;
  const uint32_t* signs;
  if (int rc = rpbh_device_tables(r, &perm, &signs)) return rc;
  const uint32_t* qtable;
  if (int rc = codebook_device_qtable(cb, &qtable)) return rc;
  int* status;
  if (int rc = device_status_word(&status)) return rc;
  int nsm;
  if (int rc = sm_count(&nsm)) return rc;

  RotqArgs a;
  memset(&a, 0, sizeof(a));
  a.X = static_cast<const uint16_t*>(X);
  a.codes = codes;
  a.norm_f32 = norm_f32;
  a.norm_bf16 = norm_bf16;
  a.perm = perm;
  a.signs = signs;
  a.qtable = qtable;
  a.status = status;
  a.M = M;
  a.d = d;
  a.P = d >= kPairElems ? 1 : kPairElems / d;
  a.groups = (M + 2 * a.P - 1) / (2 * a.P);
  const int spr = d / 32;
  a.pairs_per_warp = (spr >= 32 ? 2 : 32 / spr + 2);
  a.qtable_len = (int)cb->qtable.size();
  a.inv_sqrt_h = (float)(1.0 / std::sqrt((double)h));
  a.stages = (size_t)2 * a.P * d * 2 > 49152 ? 2 : kMaxStages;  // keep d = 16384 under 227 KB
  a.qt_scale = cb->qt_scale;
  a.qt_offset = cb->qt_offset;

  const int threads = ((a.P * spr + 31) / 32) * 32;
  const int nwarps = threads / 32;
  const size_t part_bytes = ((size_t)2 * nwarps * a.pairs_per_warp * 2 * 4 + 127) & ~(size_t)127;
  const size_t qt_bytes = ((size_t)a.qtable_len * 4 + 127) & ~(size_t)127;
  const size_t smem = 64 + part_bytes + qt_bytes + (size_t)a.P * d * 4 + (size_t)a.stages * 2 * a.P * d * 2;

  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
  if (per_sm < 1) return fail(OQ_ERR_UNSUPPORTED, "rotate+quantize kernel does not fit (d=%d)", d);
  const int grid = std::min(a.groups, nsm * per_sm);
  kern<<<grid, threads, smem, (cudaStream_t)stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "rotate+quantize launch: %s", cudaGetErrorString(e));
  return OQ_OK;
}

}  // namespace oq
