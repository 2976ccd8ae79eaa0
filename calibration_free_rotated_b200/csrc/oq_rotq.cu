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
// Design (HBM-bound):
//   * Persistent CTAs.  Each CTA owns R = max(1, 8192/d) rows per stage; a
//     3-deep ring of stage buffers in shared memory is filled by 1-D bulk
//     async copies (cp.async.bulk + mbarrier transaction counts), so HBM reads
//     for the next stages overlap the arithmetic on the current one.
//   * Thread t of the CTA owns segment g = t mod (d/32) of row t div (d/32):
//     output coordinates j = 32 g .. 32 g + 31.  Its 32 gather indices pi(j)
//     and 32 sign bits stay in registers for the whole kernel.
//   * The permutation is a gather from the shared-memory copy of the row; the
//     Rademacher sign is folded into the bf16 -> fp32 conversion.
//   * The row norm is taken from the gathered values (||Pi x|| = ||x|| since
//     Pi is orthogonal) with a fixed-order (deterministic) reduction.
//   * FWHT: 5 butterfly stages inside the thread, then log2(h/32) stages across
//     the h/32 lanes that hold one block (xor shuffles).  Blocks are aligned
//     lane groups because d/32 is a multiple of h/32.
//   * Branchless centroid search: for b <= 4, a select tree over the positive
//     boundaries held in registers (the codebook is exactly antisymmetric);
//     for b >= 5, a fixed-depth binary search over all boundaries in shared
//     memory.  Ties go to the lower centroid.
//   * The 32 codes of a segment fill exactly b 32-bit words, stored with one
//     vector store (coalesced across the warp).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "oq_internal.h"

namespace oq {
namespace {

constexpr int kStages = 3;
constexpr int kStageElems = 8192;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

struct RotqArgs {
  const uint16_t* X;
  uint8_t* codes;
  float* norm_f32;
  uint16_t* norm_bf16;
  const uint16_t* perm;
  const uint32_t* signs;
  int* status;
  int M, d, R, groups, rows_per_warp;
  float inv_sqrt_h;
  float bpos[32];    // positive boundaries ascending (2^(b-1) - 1 used)
  float bounds[64];  // all boundaries ascending (2^b - 1 used)
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
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicExch(status, OQ_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void issue_stage_load(const RotqArgs& a, uint16_t* rows, uint64_t* bars, int it) {
  const int grp = blockIdx.x + it * gridDim.x;
  if (grp >= a.groups) return;
  const int slot = it % kStages;
  const int row0 = grp * a.R;
  const int nrows = min(a.R, a.M - row0);
  const uint32_t bytes = (uint32_t)nrows * (uint32_t)a.d * 2u;
  const uint32_t bar = smem_u32(&bars[slot]);
  const uint32_t dst = smem_u32(rows + (size_t)slot * a.R * a.d);
  const uint16_t* src = a.X + (size_t)row0 * a.d;
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

template <int BITS>
__device__ __forceinline__ uint32_t quantize_one(float t, const float* bpos, const float* sb) {
  if constexpr (BITS <= 4) {
    constexpr uint32_t H = 1u << (BITS - 1);
    const bool neg = !(t > 0.0f);
    // |t|, nudged up one ulp on the non-positive side so that a strict
    // compare implements ">=" there: ties always take the lower centroid.
    const float a = __uint_as_float((__float_as_uint(t) & 0x7FFFFFFFu) + (neg ? 1u : 0u));
    uint32_t c = 0;
    if constexpr (BITS == 2) {
      c = a > bpos[0] ? 1u : 0u;
    } else if constexpr (BITS == 3) {
      const bool p1 = a > bpos[1];
      const float t0 = p1 ? bpos[2] : bpos[0];
      c = (p1 ? 2u : 0u) | (a > t0 ? 1u : 0u);
    } else if constexpr (BITS == 4) {
      const bool p2 = a > bpos[3];
      const float t1 = p2 ? bpos[5] : bpos[1];
      const bool p1 = a > t1;
      const float t0 = p2 ? (p1 ? bpos[6] : bpos[4]) : (p1 ? bpos[2] : bpos[0]);
      c = (p2 ? 4u : 0u) | (p1 ? 2u : 0u) | (a > t0 ? 1u : 0u);
    }
    return (c | H) ^ (neg ? (2u * H - 1u) : 0u);
  } else {
    // count of boundaries strictly below t, over the sorted array sb[2^b - 1]
    uint32_t idx = 0;
#pragma unroll
    for (int step = 1 << (BITS - 1); step > 0; step >>= 1)
      idx += (t > sb[idx + step - 1]) ? (uint32_t)step : 0u;
    return idx;
  }
}

// Quantize 32 values and pack their codes: the 32 codes fill exactly BITS
// 32-bit words (code i at bits [i*BITS, (i+1)*BITS) of the segment).
template <int BITS>
__device__ __forceinline__ void store_codes(uint8_t* dst, const float (&v)[32], float scale, const float* bpos,
                                            const float* sb) {
  uint32_t w[BITS];
#pragma unroll
  for (int k = 0; k < BITS; ++k) w[k] = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t c = quantize_one<BITS>(v[i] * scale, bpos, sb);
    const int bit = i * BITS, wi = bit >> 5, sh = bit & 31;
    w[wi] |= c << sh;
    if (sh + BITS > 32) w[wi + 1] |= c >> (32 - sh);
  }
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

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

template <int BITS, int LOGHB>
__global__ void __launch_bounds__(512, 1) rotq_kernel(const __grid_constant__ RotqArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int d = a.d, R = a.R;
  const int nwarps = blockDim.x >> 5;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  float* sb = reinterpret_cast<float*>(smem + 64);                  // 64 floats
  float* partial = reinterpret_cast<float*>(smem + 64 + 256);      // [2][nwarps][rows_per_warp]
  const size_t part_bytes = ((size_t)2 * nwarps * a.rows_per_warp * 4 + 127) & ~(size_t)127;
  uint16_t* rows = reinterpret_cast<uint16_t*>(smem + 64 + 256 + part_bytes);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int spr = d >> 5;  // segments per row
  const bool active = tid < R * spr;
  const int row_local = active ? tid / spr : R;  // inactive threads: past the last row
  const int g = active ? tid - row_local * spr : 0;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[s])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int k = tid; k < 64; k += blockDim.x) sb[k] = a.bounds[k];
  float bpos[BITS <= 4 ? 8 : 1];
#pragma unroll
  for (int k = 0; k < (BITS <= 4 ? 8 : 1); ++k) bpos[k] = a.bpos[k];

  // Gather offsets: byte offsets inside a stage buffer (row_local*d + pi(j)) * 2,
  // two 16-bit offsets per register (R*d*2 <= 32768 always fits).
  uint32_t off2[16];
  {
    const uint4* p4 = reinterpret_cast<const uint4*>(a.perm + 32 * g);
    const uint32_t base = 2u * (uint32_t)(active ? row_local : 0) * (uint32_t)d;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = __ldg(p4 + q);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t lo = base + 2u * (w[k] & 0xFFFFu), hi = base + 2u * (w[k] >> 16);
        off2[4 * q + k] = lo | (hi << 16);
      }
    }
  }
  const uint32_t sw = __ldg(a.signs + g);
  __syncthreads();

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) issue_stage_load(a, rows, bars, s);
  }

  for (int it = 0;; ++it) {
    const int grp = blockIdx.x + it * gridDim.x;
    if (grp >= a.groups) break;
    const int slot = it % kStages;
    const uint32_t parity = (uint32_t)(it / kStages) & 1u;
    if (!mbar_wait_bounded(smem_u32(&bars[slot]), parity, a.status)) return;

    const int row0 = grp * R;
    const int nrows = min(R, a.M - row0);
    const bool valid = active && row_local < nrows;
    const uint32_t buf = smem_u32(rows + (size_t)slot * R * d);

    // gather (permutation) + signs + sum of squares
    float v[32];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t o = (i & 1) ? (off2[i >> 1] >> 16) : (off2[i >> 1] & 0xFFFFu);
      uint32_t raw = 0u;
      if (valid) asm volatile("ld.shared.u16 %0, [%1];" : "=r"(raw) : "r"(buf + o));
      v[i] = __uint_as_float((raw << 16) ^ (((sw >> i) & 1u) << 31));
      ss = fmaf(v[i], v[i], ss);
    }

    // per-warp partial sums of every row this warp touches (fixed order)
    const int par = it & 1;
    {
      const int wr0 = (warp * 32) / spr;
      const int wr1 = min((warp * 32 + 31) / spr, R - 1);
      for (int r = wr0; r <= wr1; ++r) {
        const float x = warp_sum((active && row_local == r) ? ss : 0.0f);
        if (lane == 0) partial[(par * nwarps + warp) * a.rows_per_warp + (r - wr0)] = x;
      }
    }
    __syncthreads();  // every gather from this slot is done; partials visible
    if (tid == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_stage_load(a, rows, bars, it + kStages);
    }

    // in-thread Walsh-Hadamard butterflies over bits 0..4 of the block index
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if ((i & s) == 0) {
          const float x0 = v[i], x1 = v[i + s];
          v[i] = x0 + x1;
          v[i + s] = x0 - x1;
        }
      }
    }
    // across the h/32 lanes of a block: bits 5.. of the block index
#pragma unroll
    for (int k = 0; k < LOGHB; ++k) {
      const float sgn = ((lane >> k) & 1) ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float o = __shfl_xor_sync(0xFFFFFFFFu, v[i], 1 << k);
        v[i] = fmaf(v[i], sgn, o);
      }
    }

    if (!valid) continue;
    // row norm from the partials of the warps covering this row, in order
    float sum = 0.0f;
    {
      const int w_lo = (row_local * spr) >> 5, w_hi = (row_local * spr + spr - 1) >> 5;
      for (int w = w_lo; w <= w_hi; ++w) {
        const int r0 = (w * 32) / spr;
        sum += partial[(par * nwarps + w) * a.rows_per_warp + (row_local - r0)];
      }
    }
    const float s = sqrtf(sum);
    const float scale = a.inv_sqrt_h / (s + 1e-12f);

    const int row = row0 + row_local;
    uint8_t* dst = a.codes + (size_t)row * (size_t)(d / 8 * BITS) + (size_t)g * (4 * BITS);
    store_codes<BITS>(dst, v, scale, bpos, sb);
    if (g == 0) {
      if (a.norm_f32) a.norm_f32[row] = s;
      if (a.norm_bf16) {
        const __nv_bfloat16 hb = __float2bfloat16_rn(s);
        a.norm_bf16[row] = *reinterpret_cast<const uint16_t*>(&hb);
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
  a.status = status;
  a.M = M;
  a.d = d;
  a.R = d >= kStageElems ? 1 : kStageElems / d;
  a.groups = (M + a.R - 1) / a.R;
  const int spr = d / 32;
  a.rows_per_warp = (spr >= 32 ? 2 : 32 / spr + 2);
  a.inv_sqrt_h = (float)(1.0 / std::sqrt((double)h));
  const int L = 1 << bits, H = L / 2;
  for (int k = 0; k < 64; ++k) a.bounds[k] = k < L - 1 ? (float)cb->bounds[k] : 3.0e38f;
  for (int k = 0; k < 32; ++k) a.bpos[k] = k < H - 1 ? (float)cb->bounds[H + k] : 3.0e38f;

  const int threads = ((a.R * spr + 31) / 32) * 32;
  const int nwarps = threads / 32;
  const size_t part_bytes = ((size_t)2 * nwarps * a.rows_per_warp * 4 + 127) & ~(size_t)127;
  const size_t smem = 64 + 256 + part_bytes + (size_t)kStages * a.R * d * 2;

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
