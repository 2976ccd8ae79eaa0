// Composed RPBH rounds + norm + quantize + pack (rotation handles with k > 1
// rounds).
//
// "Quantizing With Randomized Hadamard Transforms: Efficient Heuristic Now
// Proven", Methodology and Key contributions 1 and 3: composing k randomized
// Hadamard transforms makes every coordinate of any input close to Gaussian
// (k = 2) and decorrelates the coordinates (k = 3).  With OrbitQuant's block
// rotation each round is a full RPBH round, Pi_r = blkdiag(H_h D_r) P_r, and
// the rows are rotated by Pi_k ... Pi_1 before the norm and the Lloyd-Max
// search ("OrbitQuant", Methodology, "Online Activation Quantization").
//
// One CTA works on one row pair at a time (persistent over pairs); thread g
// owns coordinates 32 g .. 32 g + 31 of both rows, the layout the butterflies
// and the search of the one-round kernel use:
//   * the rows of the CTA's next pairs stream into a ring of shared-memory
//     slots by 1-D bulk async copies with mbarrier transaction counts (two
//     slots, one for the widest rows), so HBM latency overlaps the rounds of
//     the pair at hand; a slot is refilled as soon as its pair is unpacked;
//   * the pair is unpacked from its slot (128-bit loads) into a shared array
//     of d 4-byte words, word j holding (x_a[j], x_b[j]) as bf16; a thread's
//     32 words form a 128-byte run whose 16-byte chunks are rotated by the
//     thread index, so the 128-bit writes are free of bank conflicts;
//   * round 1 gathers those words (one 32-bit load feeds both rows) and widens
//     them to f32 while flipping its signs; later rounds gather f32 pairs from
//     a shared array F of 8-byte slots, which the previous round wrote between
//     two CTA barriers; each round reads through a table of precomputed slot
//     indices and runs the unnormalised block transform in registers;
//   * where a round stores each coordinate is chosen on the host (a table of
//     store slots): every half-warp's store of one register, and the next
//     round's gather of it, fall on 16 different bank pairs (an edge colouring
//     of the store-group / gather-group graph), so both move in the minimum
//     two wavefronts instead of conflicting at random;
//   * the sum of squares comes from round 1's gathered input (the rotation is
//     orthogonal); the k factors sqrt(h) of the unnormalised transforms are
//     folded into the search multiplier;
//   * for blocks of 64..256 coordinates (where the packed codes allow it) each
//     round runs the block-transposed transform of the one-round kernel: the
//     slot and sign tables are then in each thread's register order (layout A
//     of that transform), a later round's slots point at where the previous
//     round stored each coordinate from layout B, and the codes of the last
//     round are moved back to coordinate order before the store.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "oq_rotq.cuh"

namespace oq {
namespace rotq {

struct ComposedArgs {
  const uint16_t* X;
  uint8_t* codes;
  float* norm_f32;
  uint16_t* norm_bf16;
  const uint16_t* slots;  // [rounds][d]: slot that round r's register reads (round 1: 4-byte words)
  const uint16_t* store;  // [rounds][d]: slot that round r's register is stored to (rounds before the last)
  const uint32_t* signs;  // [rounds][d / 32]: sign words
  const uint32_t* qtable;
  int* status;
  int M, d, rounds, pairs, qtable_len, stages;
  uint32_t qt_off, part_off, bar_off, ring_off;  // byte offsets in dynamic shared memory
  float alpha;                // search multiplier / h^(rounds / 2)
  float nb;
};

__device__ __forceinline__ unsigned long long lds_u64(uint32_t addr) {
  unsigned long long v;
  asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}

// Writes the 32 f32 pairs of this thread to their 8-byte slots of F, from its
// 32 store-slot indices (16-bit each, four 128-bit words).
__device__ __forceinline__ void store_round(uint32_t fbase, const uint4* st, const unsigned long long (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 S = st[q];
    const uint32_t s4[4] = {S.x, S.y, S.z, S.w};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int i = 8 * q + m;
      const uint32_t slot = (s4[m >> 1] >> (16 * (m & 1))) & 0xFFFFu;
      uint32_t lo, hi;
      u2_unpack(v[i], lo, hi);
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(fbase + 8u * slot), "r"(lo), "r"(hi) : "memory");
    }
  }
}

// One round's gather of this thread's 32 coordinates with its signs applied:
// round 1 (FIRST) from bf16 pair words (row a low, row b high), later rounds
// from f32 pairs.  sl: the thread's 32 slot indices, sw: its sign word.
template <bool FIRST>
__device__ __forceinline__ void gather_round(unsigned long long (&v)[32], const uint4* sl, uint32_t sw,
                                             uint32_t fbase) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 S = sl[q];
    const uint32_t s4[4] = {S.x, S.y, S.z, S.w};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int i = 8 * q + m;
      const uint32_t slot = (s4[m >> 1] >> (16 * (m & 1))) & 0xFFFFu;
      const uint32_t flip = (sw << (31 - i)) & 0x80000000u;  // sign of coordinate i
      if constexpr (FIRST) {
        const uint32_t w = lds_u32(fbase + 4u * slot);
        v[i] = u2_pack((w << 16) ^ flip, (w & 0xFFFF0000u) ^ flip);
      } else {
        uint32_t lo, hi;
        u2_unpack(lds_u64(fbase + 8u * slot), lo, hi);
        v[i] = u2_pack(lo ^ flip, hi ^ flip);
      }
    }
  }
}

// Copies CTA-local pair k (rows 2 pk, 2 pk + 1 with pk = blockIdx + k grid)
// into ring slot k % stages: lane 0 posts the byte count, lanes 0 and 1 issue
// one row each.  Called by warp 0 only.
__device__ __forceinline__ void issue_pair(const ComposedArgs& a, uint32_t ring, uint32_t bars, int k, int lane) {
  const int pk = blockIdx.x + k * gridDim.x;
  if (pk >= a.pairs) return;
  const int slot = k % a.stages;
  const int row = 2 * pk, nrows = min(2, a.M - row);
  const uint32_t rowb = (uint32_t)a.d * 2u;
  const uint32_t bar = bars + 8u * (uint32_t)slot;
  if (lane == 0)
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"((uint32_t)nrows * rowb)
                 : "memory");
  __syncwarp();
  if (lane < nrows) {
    const uint32_t dst = ring + (uint32_t)slot * 2u * rowb + (uint32_t)lane * rowb;
    const uint16_t* src = a.X + (size_t)(row + lane) * a.d;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(rowb), "r"(bar)
        : "memory");
  }
}

template <int BITS, int LOGHB>
__global__ void __launch_bounds__(512, 1) rotq_composed_kernel(const __grid_constant__ ComposedArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.d / 32;  // threads that own coordinates
  const bool active = tid < T;
  const uint32_t fbase = smem_u32(smem);
  uint32_t* qtab = reinterpret_cast<uint32_t*>(smem + a.qt_off);
  float2* part = reinterpret_cast<float2*>(smem + a.part_off);
  for (int i = tid; i < a.qtable_len; i += blockDim.x) qtab[i] = a.qtable[i];
  const uint32_t qkey = smem_u32(qtab) - 0x2D000000u;  // = qtab - 4 * bits(1.5 * 2^23)
  const int nwarps = blockDim.x >> 5;
  const uint32_t rowb = (uint32_t)a.d * 2u;  // bytes of a bf16 row
  const uint32_t ring = fbase + a.ring_off, bars = fbase + a.bar_off;
  constexpr bool XCH = Xch<BITS, LOGHB>::ok();
  const int bl = lane & ((1 << LOGHB) - 1);  // lane within the Hadamard block
  unsigned long long sg[3], nsg[3];          // block-transposed stages: (s, s), (-s, -s)
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const float s = ((bl >> k) & 1) ? -1.0f : 1.0f;
    sg[k] = f2_pack(s, s);
    nsg[k] = f2_pack(-s, -s);
  }

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bars + 8u * (uint32_t)s) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {  // the first pairs' copies start now, before the CTA barrier
    __syncwarp();
    for (int k = 0; k < a.stages; ++k) issue_pair(a, ring, bars, k, lane);
  }
  __syncthreads();  // barriers initialised and the search table loaded before any thread waits or reads

  int it = 0;
  for (int pr = blockIdx.x; pr < a.pairs; pr += gridDim.x, ++it) {
    const int row = 2 * pr;
    const bool has_b = row + 1 < a.M;
    const int slot = it % a.stages;
    // the previous pair's readers of F and of the partials are done, and this
    // pair's rows have landed (a give-up anywhere is agreed on and ends the CTA)
    const bool ok = mbar_wait_bounded(bars + 8u * (uint32_t)slot, (uint32_t)(it / a.stages) & 1u, a.status);
    if (__syncthreads_or(!ok)) return;
    if (active) {
      const uint32_t ra = ring + (uint32_t)slot * 2u * rowb + 64u * (uint32_t)tid, rb = ra + rowb;
      const uint32_t run1 = fbase + 128u * (uint32_t)tid, rot1 = (uint32_t)tid & 7u;
#pragma unroll
      for (int n = 0; n < 4; ++n) {  // 8 columns -> two 16-byte chunks of pair words
        const uint32_t q = ((uint32_t)n + (uint32_t)tid) & 3u;  // rotated: 2-way conflicts at most
        const uint4 A = lds_u128(ra + 16u * q);
        const uint4 B = has_b ? lds_u128(rb + 16u * q) : make_uint4(0u, 0u, 0u, 0u);
        sts_u128(run1 + (((2u * q) ^ rot1) << 4), __byte_perm(A.x, B.x, 0x5410), __byte_perm(A.x, B.x, 0x7632),
                 __byte_perm(A.y, B.y, 0x5410), __byte_perm(A.y, B.y, 0x7632));
        sts_u128(run1 + (((2u * q + 1u) ^ rot1) << 4), __byte_perm(A.z, B.z, 0x5410), __byte_perm(A.z, B.z, 0x7632),
                 __byte_perm(A.w, B.w, 0x5410), __byte_perm(A.w, B.w, 0x7632));
      }
    }
    __syncthreads();  // pair words ready; the ring slot is free
    if (warp == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_pair(a, ring, bars, it + a.stages, lane);
    }

    unsigned long long v[32];
    unsigned long long sq[4] = {0ull, 0ull, 0ull, 0ull};
    for (int r = 0; r < a.rounds; ++r) {
      if (active) {
        const uint4* sl = reinterpret_cast<const uint4*>(a.slots + (size_t)r * a.d) + 4 * tid;
        const uint32_t sw = a.signs[(size_t)r * T + tid];
        if (r == 0)
          gather_round<true>(v, sl, sw, fbase);
        else
          gather_round<false>(v, sl, sw, fbase);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0ull;
      }
      if (r == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sq[i & 3] = f2_fma(v[i], v[i], sq[i & 3]);
      }
      if constexpr (XCH)
        fwht_xch<LOGHB>(v, sg, nsg);
      else
        fwht_pairs<LOGHB>(v, lane);
      if (r + 1 < a.rounds) {
        __syncthreads();  // every thread has gathered this round's input
        if (active) store_round(fbase, reinterpret_cast<const uint4*>(a.store + (size_t)r * a.d) + 4 * tid, v);
        __syncthreads();
      }
    }

    // norms: per-warp shuffle sums, then the warps' partials in a fixed order
    unsigned long long ss2 = f2_add(f2_add(sq[0], sq[1]), f2_add(sq[2], sq[3]));
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) {
      float lo, hi;
      f2_unpack(ss2, lo, hi);
      ss2 = f2_add(ss2, f2_pack(__shfl_xor_sync(0xFFFFFFFFu, lo, k), __shfl_xor_sync(0xFFFFFFFFu, hi, k)));
    }
    if (lane == 0) {
      float lo, hi;
      f2_unpack(ss2, lo, hi);
      part[warp] = make_float2(lo, hi);
    }
    __syncthreads();
    float sum_a = 0.0f, sum_b = 0.0f;
    for (int w = 0; w < nwarps; ++w) {
      const float2 p = part[w];
      sum_a += p.x;
      sum_b += p.y;
    }
    if (active) {
      const float A_a = sum_a > 0.0f ? a.alpha * rsqrtf(sum_a) : 0.0f;
      const float A_b = sum_b > 0.0f ? a.alpha * rsqrtf(sum_b) : 0.0f;
      uint32_t wa[BITS], wb[BITS];
      search_pack<BITS>(v, A_a, A_b, a.nb, qkey, wa, wb);
      if constexpr (XCH) {  // register group u holds the codes of group u ^ bl
        xor_groups<BITS, LOGHB>(wa, bl);
        xor_groups<BITS, LOGHB>(wb, bl);
      }
      const size_t cb = (size_t)(a.d / 8 * BITS);
      uint8_t* dst = a.codes + (size_t)row * cb + (size_t)tid * (4 * BITS);
      store_words<BITS>(dst, wa);
      if (has_b) store_words<BITS>(dst + cb, wb);
      if (tid == 0) {
        const float s_a = sqrtf(sum_a), s_b = sqrtf(sum_b);
        if (a.norm_f32) {
          a.norm_f32[row] = s_a;
          if (has_b) a.norm_f32[row + 1] = s_b;
        }
        if (a.norm_bf16) {
          const __nv_bfloat16 ha = __float2bfloat16_rn(s_a), hb = __float2bfloat16_rn(s_b);
          a.norm_bf16[row] = *reinterpret_cast<const uint16_t*>(&ha);
          if (has_b) a.norm_bf16[row + 1] = *reinterpret_cast<const uint16_t*>(&hb);
        }
      }
    }
  }
}

using ComposedFn = void (*)(ComposedArgs);

// Whether rotq_composed_kernel<bits, loghb> runs the block-transposed transform
// (and so reads the register-order tables).
template <int BITS>
bool composed_xch_bits(int loghb) {
  switch (loghb) {
    case 1: return Xch<BITS, 1>::ok();
    case 2: return Xch<BITS, 2>::ok();
    case 3: return Xch<BITS, 3>::ok();
    default: return false;
  }
}

bool composed_xch(int bits, int loghb) {
  switch (bits) {
    case 1: return composed_xch_bits<1>(loghb);
    case 2: return composed_xch_bits<2>(loghb);
    case 3: return composed_xch_bits<3>(loghb);
    case 4: return composed_xch_bits<4>(loghb);
    case 5: return composed_xch_bits<5>(loghb);
    case 6: return composed_xch_bits<6>(loghb);
    default: return false;
  }
}

template <int BITS>
ComposedFn pick_composed_bits(int loghb) {
  switch (loghb) {
    case 0: return rotq_composed_kernel<BITS, 0>;
    case 1: return rotq_composed_kernel<BITS, 1>;
    case 2: return rotq_composed_kernel<BITS, 2>;
    case 3: return rotq_composed_kernel<BITS, 3>;
    case 4: return rotq_composed_kernel<BITS, 4>;
    case 5: return rotq_composed_kernel<BITS, 5>;
    default: return nullptr;
  }
}

ComposedFn pick_composed(int bits, int loghb) {
  switch (bits) {
    case 1: return pick_composed_bits<1>(loghb);
    case 2: return pick_composed_bits<2>(loghb);
    case 3: return pick_composed_bits<3>(loghb);
    case 4: return pick_composed_bits<4>(loghb);
    case 5: return pick_composed_bits<5>(loghb);
    case 6: return pick_composed_bits<6>(loghb);
    default: return nullptr;
  }
}

}  // namespace rotq

int launch_rotq_composed(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, uint8_t* codes, float* norm_f32,
                         uint16_t* norm_bf16, void* stream) {
  const int d = r->d, h = r->h, bits = cb->bits;
  int loghb = 0;
  while ((32 << loghb) < h) ++loghb;
  if (h < 32 || d % 32 != 0 || d > 16384)
    return fail(OQ_ERR_UNSUPPORTED, "composed rotation kernel: d=%d h=%d (needs h >= 32, d <= 16384)", d, h);
  const int qlen = (int)cb->qtable.size();
  if (qlen > 4097) return fail(OQ_ERR_UNSUPPORTED, "codebook d=%d bits=%d needs a %d-entry search table", cb->d, bits, qlen);
  rotq::ComposedFn kern = rotq::pick_composed(bits, loghb);
  if (!kern) return fail(OQ_ERR_UNSUPPORTED, "no composed rotate+quantize kernel for bits=%d h=%d", bits, h);
  const uint16_t *slots, *store;
  const uint32_t* signs;
  if (int rc = rpbh_composed_tables(r, &slots, &store, &signs, rotq::composed_xch(bits, loghb))) return rc;
  const uint32_t* qtable;
  if (int rc = codebook_device_qtable(cb, &qtable)) return rc;
  int nsm;
  if (int rc = sm_count(&nsm)) return rc;

  const int threads = (d / 32 + 31) / 32 * 32;
  rotq::ComposedArgs a;
  memset(&a, 0, sizeof(a));
  a.X = static_cast<const uint16_t*>(X);
  a.codes = codes;
  a.norm_f32 = norm_f32;
  a.norm_bf16 = norm_bf16;
  a.slots = slots;
  a.store = store;
  a.signs = signs;
  a.qtable = qtable;
  a.M = M;
  a.d = d;
  a.rounds = r->rounds;
  a.pairs = (M + 1) / 2;
  a.qtable_len = qlen;
  int* status;
  if (int rc = device_status_word(&status)) return rc;
  a.status = status;
  a.qt_off = (uint32_t)threads * 256u;  // F: 32 8-byte slots per thread (round 1 uses the first half as words)
  a.part_off = (a.qt_off + 4u * (uint32_t)qlen + 15u) & ~15u;
  a.bar_off = (a.part_off + (uint32_t)(threads / 32) * 8u + 15u) & ~15u;
  a.ring_off = (a.bar_off + 16u + 127u) & ~127u;
  // Ring slots of a row pair each: two where the second costs no resident CTA
  // (the kernel is bound by its rounds, so residency matters more than depth).
  const uint32_t slot_bytes = 4u * (uint32_t)d;
  const size_t smem1 = (size_t)a.ring_off + slot_bytes, smem2 = smem1 + slot_bytes;
  int occ1 = 0, occ2 = 0;
  if (int rc = occupancy(reinterpret_cast<const void*>(kern), (int)smem1, threads, 0, &occ1)) return rc;
  if (smem2 <= 200u * 1024u)
    if (int rc = occupancy(reinterpret_cast<const void*>(kern), (int)smem2, threads, 0, &occ2)) return rc;
  a.stages = occ2 >= occ1 && occ2 > 0 ? 2 : 1;
  a.alpha = (float)((double)cb->qt_alpha / std::pow((double)h, 0.5 * r->rounds));
  a.nb = (float)cb->qt_nb;
  const size_t smem = a.stages == 2 ? smem2 : smem1;
  const int per_sm = a.stages == 2 ? occ2 : occ1;
  if (per_sm < 1) return fail(OQ_ERR_UNSUPPORTED, "composed rotate+quantize kernel does not fit (d=%d)", d);
  const int grid = std::min(a.pairs, nsm * per_sm);
  kern<<<grid, threads, smem, (cudaStream_t)stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "composed rotate+quantize launch: %s", cudaGetErrorString(e));
  return OQ_OK;
}

}  // namespace oq
