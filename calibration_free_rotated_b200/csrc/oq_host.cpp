// Host side of the C ABI: handles, RPBH planning, the Lloyd-Max codebook,
// argument checks, per-device tables and the device status word.
//
// Sources: "OrbitQuant: Data-Agnostic Quantization for Image and Video
// Diffusion Transformers" ([OQ]) -- Methodology (RPBH, offline weight and
// online activation quantization), Theoretical Basis (f_d, codebook, q_hat);
// "TurboQuant: Online Vector Quantization with Near-optimal Distortion Rate"
// ([TQ]) slides 14-16 (sphere marginal, continuous k-means).
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "oq_internal.h"

namespace oq {

static thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

void clear_error() { g_last_error.clear(); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SplitMix64 (Steele, Lea & Flood 2014): state += golden gamma, then a
// bijective 64-bit mix of the new state.
uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// ---------------------------------------------------------------------------
// Lloyd-Max for f_d.  Integrals of t^p f_d(t) dt are taken in theta = asin t,
// where f_d(t) dt = C cos(theta)^(d-2) dtheta (smooth for d >= 3), on equal
// panels of width <= 0.25/sqrt(d-2) over |theta| <= min(pi/2, 40/sqrt(d-2)),
// each panel (or part of one) by 16-point Gauss-Legendre.
// ---------------------------------------------------------------------------
namespace {

constexpr int kGL = 16;

void gauss_legendre(int n, double* x, double* w) {
  // Newton iteration on P_n from the usual cosine initial guesses.
  for (int i = 0; i < n; ++i) {
    double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
    double dp = 1.0;
    for (int it = 0; it < 100; ++it) {
      double p0 = 1.0, p1 = z;
      for (int k = 2; k <= n; ++k) {
        double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
        p0 = p1;
        p1 = p2;
      }
      dp = n * (z * p1 - p0) / (z * z - 1.0);
      double dz = p1 / dp;
      z -= dz;
      if (std::fabs(dz) < 1e-16) break;
    }
    double p0 = 1.0, p1 = z;
    for (int k = 2; k <= n; ++k) {
      double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
      p0 = p1;
      p1 = p2;
    }
    dp = n * (z * p1 - p0) / (z * z - 1.0);
    x[i] = z;
    w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
  }
}

struct ThetaIntegrator {
  int d;
  double logC, tmax, width;
  int npan;
  double gx[kGL], gw[kGL];
  std::vector<double> panel[3];

  explicit ThetaIntegrator(int d_) : d(d_) {
    logC = std::lgamma(d / 2.0) - 0.5 * std::log(M_PI) - std::lgamma((d - 1) / 2.0);
    tmax = std::fmin(M_PI / 2.0, 40.0 / std::sqrt(d - 2.0));
    double wmax = 0.25 / std::sqrt(d - 2.0);
    int per_side = (int)std::ceil(tmax / wmax);
    if (per_side < 1) per_side = 1;
    npan = 2 * per_side;
    width = 2.0 * tmax / npan;
    gauss_legendre(kGL, gx, gw);
    for (int p = 0; p < 3; ++p) {
      panel[p].resize(npan);
      for (int q = 0; q < npan; ++q) panel[p][q] = gl(edge(q), edge(q + 1), p);
    }
  }
  double edge(int q) const { return q == npan ? tmax : -tmax + q * width; }
  double gl(double a, double b, int p) const {
    double half = 0.5 * (b - a), mid = 0.5 * (b + a), s = 0.0;
    for (int i = 0; i < kGL; ++i) {
      double th = mid + half * gx[i];
      double c = std::cos(th);
      double f = c > 0.0 ? std::exp(logC + (d - 2) * std::log(c)) : 0.0;
      double sn = std::sin(th);
      double g = p == 0 ? 1.0 : (p == 1 ? sn : sn * sn);
      s += gw[i] * f * g;
    }
    return half * s;
  }
  double to_theta(double t) const {
    double th = std::asin(std::fmax(-1.0, std::fmin(1.0, t)));
    return std::fmax(-tmax, std::fmin(tmax, th));
  }
  int panel_of(double th) const {
    int q = (int)std::floor((th + tmax) / width);
    return q < 0 ? 0 : (q >= npan ? npan - 1 : q);
  }
  // int_{ta}^{tb} t^p f_d(t) dt
  double cell(double ta, double tb, int p) const {
    double a = to_theta(ta), b = to_theta(tb);
    int pa = panel_of(a), pb = panel_of(b);
    if (pa == pb) return gl(a, b, p);
    long double s = gl(a, edge(pa + 1), p);
    for (int q = pa + 1; q < pb; ++q) s += panel[p][q];
    s += gl(edge(pb), b, p);
    return (double)s;
  }
};

}  // namespace

void lloyd_max(int d, int bits, std::vector<double>& c, std::vector<double>& beta, int& iterations,
               double& distortion) {
  const int L = 1 << bits;
  ThetaIntegrator integ(d);
  const double sd = std::sqrt((double)d);
  const double a = std::fmin(3.0 / sd, 0.9);
  c.resize(L);
  for (int k = 0; k < L; ++k) c[k] = L == 1 ? 0.0 : -a + 2.0 * a * k / (L - 1);
  std::vector<double> e(L + 1), cn(L);
  const double tol = 1e-13;
  const int max_iters = 200000;
  int it = 0;
  for (it = 1; it <= max_iters; ++it) {
    e[0] = -1.0;
    e[L] = 1.0;
    for (int k = 1; k < L; ++k) e[k] = 0.5 * (c[k - 1] + c[k]);  // nearest-neighbour condition
    double delta = 0.0;
    for (int k = 0; k < L; ++k) {                                  // centroid condition
      double m0 = integ.cell(e[k], e[k + 1], 0);
      double m1 = integ.cell(e[k], e[k + 1], 1);
      cn[k] = m1 / m0;
      delta = std::fmax(delta, std::fabs(cn[k] - c[k]));
    }
    c.swap(cn);
    if (delta * sd < tol) break;
  }
  if (it > max_iters) it = max_iters;
  iterations = it;
  // exact antisymmetry: the optimum for the symmetric f_d is symmetric
  for (int k = 0; k < L / 2; ++k) {
    double v = 0.5 * (c[L - 1 - k] - c[k]);
    c[L - 1 - k] = v;
    c[k] = -v;
  }
  beta.resize(L - 1);
  for (int k = 0; k + 1 < L; ++k) beta[k] = 0.5 * (c[k] + c[k + 1]);
  double dist = 0.0;
  for (int k = 0; k < L; ++k) {
    double lo = k == 0 ? -1.0 : beta[k - 1], hi = k == L - 1 ? 1.0 : beta[k];
    double m0 = integ.cell(lo, hi, 0), m1 = integ.cell(lo, hi, 1), m2 = integ.cell(lo, hi, 2);
    dist += m2 - 2.0 * c[k] * m1 + c[k] * c[k] * m0;
  }
  distortion = dist;
}

// IEEE binary16 bits of v rounded to nearest, ties to even (finite |v| < 65520).
uint16_t double_to_fp16_rne(double v) {
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e;
  double m = std::frexp(a, &e);  // a = m 2^e, 0.5 <= m < 1
  if (e - 1 < -14) {             // subnormal: multiples of 2^-24
    double q = std::nearbyint(a * 16777216.0);
    return (uint16_t)(sign | (uint16_t)q);  // q == 1024 becomes the smallest normal
  }
  double q = std::nearbyint(m * 2048.0);  // 11 significant bits
  if (q >= 2048.0) {
    q *= 0.5;
    e += 1;
  }
  int exp_field = e - 1 + 15;
  if (exp_field >= 31) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | (exp_field << 10) | ((uint16_t)q & 0x3FF));
}

// ---------------------------------------------------------------------------
// Bucket table for the rotate+quantize kernel's centroid search.
//
// The kernel maps a normalised coordinate t into the unit interval,
// y = sat(t * alpha + 1/2) (fp32), and reads the bucket q = round(y * NB) from
// the low mantissa bits of fma(y, NB, 1.5 * 2^23).  Bucket q covers
// y * NB in [q - 1/2, q + 1/2).  alpha maps every boundary into (0, 1) with a
// little room; NB (a power of two) is large enough that consecutive fp32
// boundaries are >= 1.25 buckets apart (at most one boundary per bucket), and
// alpha is nudged until no boundary lies within 0.02 bucket of a bucket edge
// (a y that rounds to either neighbour at an edge then gets the same answer).
// Entry q: the bucket's boundary in y (or 3e38 if none) with its low b
// mantissa bits replaced by base_q = #{boundaries below the bucket}; the code
// is base_q + (y > entry).  Replacing those bits moves a threshold by fewer
// than 2^b fp32 ulps of y < 1 (below 4e-6 in y, a few 1e-7 in t), far inside
// the 1e-5 boundary band of the parity rule.  The middle boundary of an even
// codebook is t = 0, i.e. y = 1/2 exactly, whose low mantissa bits are zero:
// its entry is >= 1/2, so t = 0 takes the lower centroid as the tie rule says.
// ---------------------------------------------------------------------------
void build_qtable(oq_codebook_t cb) {
  const int L = 1 << cb->bits;
  std::vector<double> b(L - 1);
  double bmax = 0.0, gap = 1e300;
  for (int k = 0; k < L - 1; ++k) {
    b[k] = (double)(float)cb->bounds[k];
    bmax = std::fmax(bmax, std::fabs(b[k]));
    if (k > 0) gap = std::fmin(gap, b[k] - b[k - 1]);
  }
  double T = bmax > 0.0 ? bmax * 1.02 + 1e-6 : 1.0;
  int NB = 2;
  while (NB < (1 << 16) && 1.25 * (2.0 * T / NB) > gap) NB *= 2;
  float alpha = 0.0f;
  std::vector<double> yb(L - 1);
  for (int attempt = 0; attempt < 100000; ++attempt) {
    alpha = (float)(0.5 / T);
    bool ok = true;
    for (int k = 0; k < L - 1; ++k) {
      yb[k] = (double)(float)(b[k] * (double)alpha + 0.5);
      const double z = yb[k] * NB;
      if (std::fabs(z - std::floor(z) - 0.5) < 0.02) ok = false;
    }
    if (ok) break;
    T *= 1.0007;
  }
  cb->qtable.assign(NB + 1, 0u);
  const uint32_t lowmask = (uint32_t)L - 1u;
  for (int q = 0; q <= NB; ++q) {
    const double lo = (q - 0.5) / NB, hi = (q + 0.5) / NB;
    uint32_t base = 0;
    float thr = 3.0e38f;
    for (int k = 0; k < L - 1; ++k) {
      if (yb[k] < lo) ++base;
      else if (yb[k] < hi) thr = (float)yb[k];
    }
    uint32_t bits;
    std::memcpy(&bits, &thr, 4);
    cb->qtable[q] = (bits & ~lowmask) | base;
  }
  cb->qt_alpha = alpha;
  cb->qt_nb = NB;
}

// ---------------------------------------------------------------------------
// Device state
// ---------------------------------------------------------------------------
static std::atomic<long long> g_dev_allocs{0};

// Every device allocation of the library goes through here, so that
// oq_device_allocations() can report how many there have been.
static cudaError_t dev_malloc(void** p, size_t bytes) {
  cudaError_t e = cudaMalloc(p, bytes);
  if (e == cudaSuccess) g_dev_allocs.fetch_add(1, std::memory_order_relaxed);
  return e;
}

static std::mutex g_dev_mu;
static int* g_status[OQ_MAX_DEVICES] = {};
static int g_sms[OQ_MAX_DEVICES] = {};

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (*dev < 0 || *dev >= OQ_MAX_DEVICES) return fail(OQ_ERR_UNSUPPORTED, "device index %d too large", *dev);
  return OQ_OK;
}

int device_status_word(int** status) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_status[dev]) {
    int* p = nullptr;
    cudaError_t e = dev_malloc(reinterpret_cast<void**>(&p), sizeof(int));
    if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "cudaMalloc(status): %s", cudaGetErrorString(e));
    e = cudaMemset(p, 0, sizeof(int));
    if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "cudaMemset(status): %s", cudaGetErrorString(e));
    g_status[dev] = p;
  }
  *status = g_status[dev];
  return OQ_OK;
}

int device_status_word_if_present(int** status) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_status[dev]) return OQ_ERR_ARG;
  *status = g_status[dev];
  return OQ_OK;
}

int sm_count(int* n) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_sms[dev]) {
    int v = 0;
    cudaError_t e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    g_sms[dev] = v;
  }
  *n = g_sms[dev];
  return OQ_OK;
}

namespace {
struct OccEntry {
  const void* fn;
  int dev, smem, threads, cluster, value;
};
std::mutex g_occ_mu;
std::vector<OccEntry> g_occ;
std::vector<std::pair<const void*, int>> g_smem_raised;  // (kernel, device)

struct TmapEntry {
  TmapKey key;
  int dev;
  alignas(64) unsigned char map[128];
};
constexpr int kTmapSlots = 64;
std::mutex g_tmap_mu;
TmapEntry g_tmap[kTmapSlots];
int g_tmap_used = 0, g_tmap_next = 0;
}  // namespace

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("OQ_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}

int occupancy(const void* kernel, int smem, int threads, int cluster, int* value) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lk(g_occ_mu);
  for (const OccEntry& e : g_occ)
    if (e.fn == kernel && e.dev == dev && e.smem == smem && e.threads == threads && e.cluster == cluster) {
      *value = e.value;
      return OQ_OK;
    }
  bool raised = false;
  for (const auto& p : g_smem_raised) raised |= p.first == kernel && p.second == dev;
  if (!raised) {
    int optin = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kernel);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "raising the shared-memory limit: %s", cudaGetErrorString(e));
    g_smem_raised.emplace_back(kernel, dev);
  }
  int v = 0;
  cudaError_t e;
  if (cluster == 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, threads, (size_t)smem);
  } else {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.gridDim = dim3((unsigned)cluster, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    e = cudaOccupancyMaxActiveClusters(&v, kernel, &cfg);
  }
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(e));
  g_occ.push_back(OccEntry{kernel, dev, smem, threads, cluster, v});
  *value = v;
  return OQ_OK;
}

int cached_tensor_map(const TmapKey& key, void* map128, int (*encode)(const TmapKey&, void*)) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lk(g_tmap_mu);
  for (int i = 0; i < g_tmap_used; ++i)
    if (g_tmap[i].dev == dev && g_tmap[i].key == key) {
      std::memcpy(map128, g_tmap[i].map, 128);
      return OQ_OK;
    }
  if (int rc = encode(key, map128)) return rc;
  TmapEntry& slot = g_tmap[g_tmap_next];  // round-robin replacement
  slot.key = key;
  slot.dev = dev;
  std::memcpy(slot.map, map128, 128);
  g_tmap_next = (g_tmap_next + 1) % kTmapSlots;
  if (g_tmap_used < kTmapSlots) ++g_tmap_used;
  return OQ_OK;
}

static int upload_rpbh(oq_rpbh_t r, int dev) {
  std::vector<uint16_t> p16(r->d);
  for (int j = 0; j < r->d; ++j) p16[j] = (uint16_t)r->perm[j];
  uint16_t* dp = nullptr;
  uint32_t* ds = nullptr;
  cudaError_t e = dev_malloc(reinterpret_cast<void**>(&dp), sizeof(uint16_t) * r->d);
  if (e == cudaSuccess) e = dev_malloc(reinterpret_cast<void**>(&ds), sizeof(uint32_t) * r->sign_bits.size());
  if (e == cudaSuccess) e = cudaMemcpy(dp, p16.data(), sizeof(uint16_t) * r->d, cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(ds, r->sign_bits.data(), sizeof(uint32_t) * r->sign_bits.size(), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(dp);
    cudaFree(ds);
    return fail(OQ_ERR_CUDA, "uploading RPBH tables: %s", cudaGetErrorString(e));
  }
  r->dev_perm[dev] = dp;
  r->dev_signs[dev] = ds;
  return OQ_OK;
}

int codebook_device_qtable(oq_codebook_t cb, const uint32_t** qtable) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lk(cb->mu);
  if (!cb->dev_qtable[dev]) {
    uint32_t* p = nullptr;
    const size_t bytes = sizeof(uint32_t) * cb->qtable.size();
    cudaError_t e = dev_malloc(reinterpret_cast<void**>(&p), bytes);
    if (e == cudaSuccess) e = cudaMemcpy(p, cb->qtable.data(), bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaFree(p);
      return fail(OQ_ERR_CUDA, "uploading the search table: %s", cudaGetErrorString(e));
    }
    cb->dev_qtable[dev] = p;
  }
  *qtable = cb->dev_qtable[dev];
  return OQ_OK;
}

// Shared-memory slot of coordinate c in the composed kernel: thread c / 32
// owns a run of 32 slots whose 16-byte chunks are rotated by the thread index.
// Round 1 reads 4-byte bf16 pair words (chunk (c / 4) % 8 at position
// chunk ^ (thread % 8)); later rounds 8-byte f32 pairs (chunk (c / 2) % 16 at
// position chunk ^ (thread % 16)).
static uint16_t composed_slot(uint32_t c, bool first_round) {
  const uint32_t g = c >> 5;
  if (first_round) {
    const uint32_t ch = (c >> 2) & 7u;
    return (uint16_t)((g << 5) | ((ch ^ (g & 7u)) << 2) | (c & 3u));
  }
  const uint32_t ch = (c >> 1) & 15u;
  return (uint16_t)((g << 5) | ((ch ^ (g & 15u)) << 1) | (c & 1u));
}

// Register order of the block-transposed FWHT for blocks of L = h / 32 lanes
// (R = 32 / L): thread g (lane l = g mod L of its block) gathers into register
// r coordinate 32 (g - l) + 32 ((r / R) ^ l) + R l + r mod R (layout A), and
// holds output coordinate 32 g + R (u ^ l) + b in register R u + b (layout B).
static uint32_t xch_gather_coord(uint32_t g, uint32_t r, uint32_t L) {
  const uint32_t R = 32u / L, l = g & (L - 1u);
  return 32u * (g - l) + 32u * ((r / R) ^ l) + R * l + r % R;
}
static uint32_t xch_output_reg(uint32_t c, uint32_t L) {  // the register that holds output coordinate c
  const uint32_t R = 32u / L, l = (c >> 5) & (L - 1u), i = c & 31u;
  return R * ((i / R) ^ l) + i % R;
}

// Splits the edges `ids` of a bipartite multigraph in which every vertex has
// an even number of them into two halves that give every vertex half of its
// edges each (bit[e] = 0 or 1): closed walks over unused edges, labelled
// alternately.  A closed walk in a bipartite graph has even length, so every
// pass through a vertex, the start included, uses one edge of each label.
static void euler_split(int nv, const std::vector<std::pair<int, int>>& E, const std::vector<int>& ids,
                        std::vector<uint8_t>& bit) {
  std::vector<std::vector<int>> adj((size_t)nv);
  for (int e : ids) {
    adj[(size_t)E[e].first].push_back(e);
    adj[(size_t)E[e].second].push_back(e);
  }
  std::vector<uint8_t> used(E.size(), 0);
  std::vector<size_t> next((size_t)nv, 0);
  auto take = [&](int x) -> int {  // an unused edge at x, or -1
    auto& a = adj[(size_t)x];
    size_t& i = next[(size_t)x];
    while (i < a.size() && used[(size_t)a[i]]) ++i;
    return i < a.size() ? a[i] : -1;
  };
  for (int s = 0; s < nv; ++s) {
    while (take(s) >= 0) {
      int cur = s;
      uint8_t label = 0;
      for (int e = take(cur); e >= 0; e = take(cur)) {
        used[(size_t)e] = 1;
        bit[(size_t)e] = label;
        label ^= 1u;
        cur = E[e].first == cur ? E[e].second : E[e].first;
      }
    }
  }
}

// Shared-memory layout of one round's output for the composed kernel, free of
// bank conflicts on both sides.  Coordinate c is stored by one register of
// one thread (the store group: half-warp and register) and gathered by one
// register of one thread of the next round (the load group); each group is
// at most 16 lanes.  An 8-byte slot s sits on bank pair s mod 16, so a group
// whose 16 slots fall on 16 different bank pairs moves in the minimum two
// wavefronts.  Colouring the bipartite (store group, load group) multigraph
// with 16 colours, one per bank pair, such that no group repeats a colour is
// an edge colouring of a graph of degree 16, which always exists (Konig);
// padded with dummy edges to exactly degree 16, four levels of Euler splits
// find one.  Returns sigma[c], the slot of coordinate c, all below 32 * TP.
static std::vector<uint16_t> conflict_free_layout(int d, const std::vector<uint32_t>& store_group,
                                                  const std::vector<uint32_t>& load_group, int ngroups) {
  std::vector<std::pair<int, int>> E;  // vertices: store groups 0.., load groups ngroups..
  E.reserve((size_t)ngroups * 16);
  std::vector<int> ds((size_t)ngroups, 0), dl((size_t)ngroups, 0);
  for (int c = 0; c < d; ++c) {
    E.emplace_back((int)store_group[(size_t)c], ngroups + (int)load_group[(size_t)c]);
    ++ds[store_group[(size_t)c]];
    ++dl[load_group[(size_t)c]];
  }
  // pad to degree 16 (both sides miss the same number of edges)
  for (int u = 0, v = 0; u < ngroups; ++u) {
    while (ds[(size_t)u] < 16) {
      while (dl[(size_t)v] >= 16) ++v;
      E.emplace_back(u, ngroups + v);
      ++ds[(size_t)u];
      ++dl[(size_t)v];
    }
  }
  std::vector<uint8_t> colour(E.size(), 0), bit(E.size(), 0);
  std::vector<std::vector<int>> classes(1);
  for (size_t e = 0; e < E.size(); ++e) classes[0].push_back((int)e);
  for (int level = 0; level < 4; ++level) {
    std::vector<std::vector<int>> split;
    for (const auto& ids : classes) {
      euler_split(2 * ngroups, E, ids, bit);
      std::vector<int> a, b;
      for (int e : ids) {
        (bit[(size_t)e] ? b : a).push_back(e);
        colour[(size_t)e] = (uint8_t)(colour[(size_t)e] | (bit[(size_t)e] << level));
      }
      split.push_back(std::move(a));
      split.push_back(std::move(b));
    }
    classes.swap(split);
  }
  std::vector<uint16_t> sigma((size_t)d);
  int fill[16] = {};
  for (int c = 0; c < d; ++c) {
    const int k = colour[(size_t)c];
    sigma[(size_t)c] = (uint16_t)(16 * fill[k]++ + k);
  }
  return sigma;
}

// The composed kernel's tables for one register order (coordinate order, or
// the block-transposed layout's):
//   gather[k][32 g + r]: the slot register r of thread g reads in round k
//                        (round 1: the interleaved bf16 pair words; later
//                        rounds: where the previous round stored it);
//   store[k][32 g + r]:  the slot it stores its output to (rounds before the last);
//   signs[k][g]:         bit r = the sign of the coordinate register r gathers.
static void build_composed_tables(const oq_rpbh_s* r, bool xch, std::vector<uint16_t>& gather,
                                  std::vector<uint16_t>& store, std::vector<uint32_t>& signs) {
  const int d = r->d, T = d / 32, words = (d + 31) / 32, rounds = r->rounds;
  const uint32_t L = (uint32_t)r->h / 32u, R = xch ? 32u / L : 32u;
  gather.assign((size_t)rounds * d, 0);
  store.assign((size_t)rounds * d, 0);
  signs.assign((size_t)rounds * words, 0u);
  auto in_j = [&](uint32_t g, uint32_t reg) { return xch ? xch_gather_coord(g, reg, L) : 32u * g + reg; };
  auto out_c = [&](uint32_t g, uint32_t reg) {
    return xch ? 32u * g + R * ((reg / R) ^ (g & (L - 1u))) + reg % R : 32u * g + reg;
  };
  const int ngroups = ((T + 15) / 16) * 32;  // (half-warp, register)
  std::vector<uint16_t> sigma;  // slots of the previous round's output
  for (int k = 0; k < rounds; ++k) {
    const int32_t* perm = k == 0 ? r->perm.data() : r->perm_more.data() + (size_t)(k - 1) * d;
    const uint32_t* bits = k == 0 ? r->sign_bits.data() : r->sign_bits_more.data() + (size_t)(k - 1) * words;
    for (uint32_t g = 0; g < (uint32_t)T; ++g) {
      for (uint32_t reg = 0; reg < 32u; ++reg) {
        const uint32_t j = in_j(g, reg), c = (uint32_t)perm[j];
        gather[(size_t)k * d + 32u * g + reg] = k == 0 ? composed_slot(c, true) : sigma[c];
        if ((bits[j >> 5] >> (j & 31u)) & 1u) signs[(size_t)k * words + g] |= 1u << reg;
      }
    }
    if (k + 1 == rounds) break;
    // this round's output layout, chosen against the next round's gathers
    const int32_t* pnext = r->perm_more.data() + (size_t)k * d;
    std::vector<uint32_t> sgrp((size_t)d), lgrp((size_t)d);
    for (uint32_t g = 0; g < (uint32_t)T; ++g)
      for (uint32_t reg = 0; reg < 32u; ++reg) {
        sgrp[out_c(g, reg)] = (g >> 4) * 32u + reg;
        lgrp[(uint32_t)pnext[in_j(g, reg)]] = (g >> 4) * 32u + reg;
      }
    sigma = conflict_free_layout(d, sgrp, lgrp, ngroups);
    for (uint32_t g = 0; g < (uint32_t)T; ++g)
      for (uint32_t reg = 0; reg < 32u; ++reg) store[(size_t)k * d + 32u * g + reg] = sigma[out_c(g, reg)];
  }
}

int rpbh_composed_tables(oq_rpbh_t r, const uint16_t** slots, const uint16_t** store, const uint32_t** signs,
                         bool xch) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  const uint32_t L = (uint32_t)r->h / 32u;
  const bool xch_ok = L >= 2 && L <= 8 && r->d % 32 == 0;
  if (xch && !xch_ok) return fail(OQ_ERR_UNSUPPORTED, "no block-transposed layout for block %d", r->h);
  std::lock_guard<std::mutex> lk(r->mu);
  if (!r->dev_ctab[0][dev]) {  // both register orders at once, so no later launch allocates
    for (int v = 0; v < (xch_ok ? 2 : 1); ++v) {
      std::vector<uint16_t> gather, st;
      std::vector<uint32_t> sg;
      build_composed_tables(r, v == 1, gather, st, sg);
      // one allocation: gather slots, store slots, sign words
      const size_t nslot = gather.size(), bytes = sizeof(uint16_t) * 2 * nslot + sizeof(uint32_t) * sg.size();
      unsigned char* dbuf = nullptr;
      cudaError_t e = dev_malloc(reinterpret_cast<void**>(&dbuf), bytes);
      if (e == cudaSuccess) e = cudaMemcpy(dbuf, gather.data(), sizeof(uint16_t) * nslot, cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(dbuf + sizeof(uint16_t) * nslot, st.data(), sizeof(uint16_t) * nslot, cudaMemcpyHostToDevice);
      if (e == cudaSuccess)
        e = cudaMemcpy(dbuf + sizeof(uint16_t) * 2 * nslot, sg.data(), sizeof(uint32_t) * sg.size(),
                       cudaMemcpyHostToDevice);
      if (e != cudaSuccess) {
        cudaFree(dbuf);
        if (v == 1) {  // keep the pair all-or-nothing
          cudaFree(r->dev_ctab[0][dev]);
          r->dev_ctab[0][dev] = nullptr;
        }
        return fail(OQ_ERR_CUDA, "uploading composed rotation tables: %s", cudaGetErrorString(e));
      }
      r->dev_ctab[v][dev] = dbuf;
    }
  }
  const int v = xch ? 1 : 0;
  const size_t nslot = (size_t)r->rounds * r->d;
  unsigned char* base = r->dev_ctab[v][dev];
  *slots = reinterpret_cast<const uint16_t*>(base);
  *store = reinterpret_cast<const uint16_t*>(base + sizeof(uint16_t) * nslot);
  *signs = reinterpret_cast<const uint32_t*>(base + sizeof(uint16_t) * 2 * nslot);
  return OQ_OK;
}

int rpbh_tables_if_present(oq_rpbh_t r, int dev) {
  std::lock_guard<std::mutex> lk(r->mu);
  return r->dev_perm[dev] && (r->rounds == 1 || r->dev_ctab[0][dev]) ? OQ_OK : OQ_ERR_ARG;
}

int codebook_qtable_if_present(oq_codebook_t cb, int dev) {
  std::lock_guard<std::mutex> lk(cb->mu);
  return cb->dev_qtable[dev] ? OQ_OK : OQ_ERR_ARG;
}

int rpbh_device_tables(oq_rpbh_t r, const uint16_t** perm, const uint32_t** signs) {
  int dev;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lk(r->mu);
  if (!r->dev_perm[dev]) {
    if (int rc = upload_rpbh(r, dev)) return rc;
  }
  *perm = r->dev_perm[dev];
  *signs = r->dev_signs[dev];
  return OQ_OK;
}

// Host span of an entry point for timeline tools (NVTX; a no-op unless a tool
// such as ncu --nvtx is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

static std::atomic<int> g_test_stall{0};

int take_test_stall(int kernel) {
  int expected = kernel;
  return g_test_stall.compare_exchange_strong(expected, 0) ? 1 : 0;
}

// One round of draws from the SplitMix64 stream `st`: the Fisher-Yates
// permutation of 0..d-1 (for i = d-1 .. 1: j = next() mod (i+1), swap), then
// d Rademacher signs (sign_j = -1 when the top bit of next() is set).
static void draw_round(uint64_t& st, int d, int32_t* perm, uint32_t* sign_bits) {
  for (int j = 0; j < d; ++j) perm[j] = j;
  for (int i = d - 1; i >= 1; --i) {
    const uint64_t j = splitmix64_next(st) % (uint64_t)(i + 1);
    const int32_t tmp = perm[i];
    perm[i] = perm[j];
    perm[j] = tmp;
  }
  for (int w = 0; w < (d + 31) / 32; ++w) sign_bits[w] = 0u;
  for (int j = 0; j < d; ++j)
    if (splitmix64_next(st) >> 63) sign_bits[j >> 5] |= 1u << (j & 31);
}

// Rotation handle of `rounds` rounds drawn in order from SplitMix64(seed).
static int make_rotation(uint64_t seed, int d, int block, int kind, int rounds, oq_rpbh_t* out) {
  if (!out) return fail(OQ_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (d < 1) return fail(OQ_ERR_ARG, "d must be >= 1 (got %d)", d);
  if (kind != OQ_ROT_RPBH && kind != OQ_ROT_BLOCK_RHT && kind != OQ_ROT_FULL_RHT)
    return fail(OQ_ERR_ARG, "unknown rotation kind %d", kind);
  if (kind == OQ_ROT_FULL_RHT && block != 0 && block != (d & -d))
    return fail(OQ_ERR_ARG, "a full RHT of d=%d has block %d (got %d)", d, d & -d, block);
  int h = block == 0 ? (d & -d) : block;
  if (h < 1 || (h & (h - 1)) != 0 || d % h != 0)
    return fail(OQ_ERR_ARG, "block %d must be a power of two dividing d=%d", block, d);
  // the composed kernel's limits, checked here so that no handle is made (and
  // uploaded) that no kernel can run
  if (rounds > 1 && (h < 32 || d % 32 != 0 || d > 16384))
    return fail(OQ_ERR_UNSUPPORTED, "composed rotation kernel: d=%d h=%d (needs h >= 32, d <= 16384)", d, h);
  oq_rpbh_t r = new (std::nothrow) oq_rpbh_s;
  if (!r) return fail(OQ_ERR_NOMEM, "allocating the RPBH handle");
  r->seed = seed;
  r->d = d;
  r->h = h;
  r->kind = kind;
  r->rounds = rounds;
  const size_t words = (size_t)(d + 31) / 32;
  r->perm.resize(d);
  r->sign_bits.resize(words);
  r->perm_more.resize((size_t)(rounds - 1) * d);
  r->sign_bits_more.resize((size_t)(rounds - 1) * words);
  uint64_t st = seed;
  draw_round(st, d, r->perm.data(), r->sign_bits.data());
  // Block-RHT and Full RHT: the same draws (so the same signs), identity permutation
  if (kind != OQ_ROT_RPBH)
    for (int j = 0; j < d; ++j) r->perm[j] = j;
  for (int k = 1; k < rounds; ++k)  // later rounds continue the same stream
    draw_round(st, d, r->perm_more.data() + (size_t)(k - 1) * d, r->sign_bits_more.data() + (size_t)(k - 1) * words);
  // Upload to the current device now when one is present; otherwise lazily.
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0 && d <= 65536) {
    int dev;
    if (cudaGetDevice(&dev) == cudaSuccess && dev < OQ_MAX_DEVICES) {
      if (int rc = upload_rpbh(r, dev)) {
        delete r;
        return rc;
      }
      if (rounds > 1) {
        const uint16_t *sl, *st;
        const uint32_t* sg;
        if (int rc = rpbh_composed_tables(r, &sl, &st, &sg)) {
          oq_free_rpbh(r);
          return rc;
        }
      }
    }
  } else {
    cudaGetLastError();  // no device here: clear the sticky "no device" error
  }
  *out = r;
  return OQ_OK;
}

}  // namespace oq

// ===========================================================================
// C ABI
// ===========================================================================
using namespace oq;

extern "C" {

int oq_version(void) { return OQ_VERSION; }

long long oq_device_allocations(void) { return g_dev_allocs.load(std::memory_order_relaxed); }

// Synchronous checking (OQ_DEBUG=1 in the environment, or oq_set_debug): each
// launching entry point then waits for its stream and returns the device status
// word itself, so an asynchronous give-up is reported by the call that caused
// it.  Off by default, when the calls stay asynchronous.
static std::atomic<int> g_debug{-1};  // -1: the environment is not read yet

static bool debug_on() {
  int v = g_debug.load();
  if (v < 0) {
    const char* e = std::getenv("OQ_DEBUG");
    v = (e && e[0] && e[0] != '0') ? 1 : 0;
    int expected = -1;
    g_debug.compare_exchange_strong(expected, v);
    v = g_debug.load();
  }
  return v != 0;
}

static int finish(int rc, void* stream) {
  if (rc != OQ_OK || !debug_on()) return rc;
  return oq_get_device_status(stream);
}

int oq_set_debug(int on) {
  clear_error();
  g_debug.store(on ? 1 : 0);
  return OQ_OK;
}

int oq_test_composed_tables(oq_rpbh_t r, int xch, uint16_t* gather, uint16_t* store, uint32_t* signs) {
  clear_error();
  if (!r || !gather || !store || !signs) return fail(OQ_ERR_ARG, "NULL argument");
  if (r->rounds < 2) return fail(OQ_ERR_ARG, "not a composed rotation");
  const uint32_t L = (uint32_t)r->h / 32u;
  if (xch && !(L >= 2 && L <= 8)) return fail(OQ_ERR_UNSUPPORTED, "no block-transposed layout for block %d", r->h);
  std::vector<uint16_t> g, st;
  std::vector<uint32_t> sg;
  {
    std::lock_guard<std::mutex> lk(r->mu);
    build_composed_tables(r, xch != 0, g, st, sg);
  }
  std::memcpy(gather, g.data(), sizeof(uint16_t) * g.size());
  std::memcpy(store, st.data(), sizeof(uint16_t) * st.size());
  std::memcpy(signs, sg.data(), sizeof(uint32_t) * sg.size());
  return OQ_OK;
}

int oq_test_stall_next(int kernel) {
  clear_error();
  if (kernel < 0 || kernel > 2) return fail(OQ_ERR_ARG, "kernel must be 0 (disarm), 1 or 2 (got %d)", kernel);
  g_test_stall.store(kernel);
  return OQ_OK;
}

const char* oq_last_error(void) { return g_last_error.c_str(); }

int oq_get_device_status(void* stream) {
  clear_error();
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  int* st;
  if (int rc = device_status_word(&st)) return rc;
  int v = 0;
  e = cudaMemcpy(&v, st, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(st, 0, sizeof(int));
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, "reading device status: %s", cudaGetErrorString(e));
  if (v != OQ_OK) return fail(v, "a kernel reported device status %d (bounded wait gave up)", v);
  return OQ_OK;
}

int oq_make_rotation(uint64_t seed, int d, int block, int kind, oq_rpbh_t* out) {
  clear_error();
  return make_rotation(seed, d, block, kind, 1, out);
}

int oq_make_rpbh(uint64_t seed, int d, int block, oq_rpbh_t* out) {
  return oq_make_rotation(seed, d, block, OQ_ROT_RPBH, out);
}

int oq_make_composed_rpbh(uint64_t seed, int d, int block, int rounds, oq_rpbh_t* out) {
  clear_error();
  if (rounds < 1 || rounds > 3) {
    if (out) *out = nullptr;
    return fail(OQ_ERR_ARG, "rounds must be 1, 2 or 3 (got %d)", rounds);
  }
  return make_rotation(seed, d, block, OQ_ROT_RPBH, rounds, out);
}

int oq_rotation_rounds(oq_rpbh_t r, int* rounds) {
  clear_error();
  if (!r || !rounds) return fail(OQ_ERR_ARG, "NULL argument");
  *rounds = r->rounds;
  return OQ_OK;
}

int oq_rpbh_export_round(oq_rpbh_t r, int round, int32_t* perm, uint32_t* sign_bits) {
  clear_error();
  if (!r) return fail(OQ_ERR_ARG, "NULL rpbh handle");
  if (round < 1 || round > r->rounds) return fail(OQ_ERR_ARG, "round %d of a %d-round rotation", round, r->rounds);
  const size_t words = r->sign_bits.size();
  const int32_t* p = round == 1 ? r->perm.data() : r->perm_more.data() + (size_t)(round - 2) * r->d;
  const uint32_t* b = round == 1 ? r->sign_bits.data() : r->sign_bits_more.data() + (size_t)(round - 2) * words;
  if (perm) std::memcpy(perm, p, sizeof(int32_t) * r->d);
  if (sign_bits) std::memcpy(sign_bits, b, sizeof(uint32_t) * words);
  return OQ_OK;
}

int oq_rotation_kind(oq_rpbh_t r, int* kind) {
  clear_error();
  if (!r || !kind) return fail(OQ_ERR_ARG, "NULL argument");
  *kind = r->kind;
  return OQ_OK;
}

int oq_rpbh_info(oq_rpbh_t r, int* d, int* block) {
  clear_error();
  if (!r) return fail(OQ_ERR_ARG, "NULL rpbh handle");
  if (d) *d = r->d;
  if (block) *block = r->h;
  return OQ_OK;
}

int oq_rpbh_export(oq_rpbh_t r, int32_t* perm, uint32_t* sign_bits) {
  clear_error();
  if (!r) return fail(OQ_ERR_ARG, "NULL rpbh handle");
  if (perm) std::memcpy(perm, r->perm.data(), sizeof(int32_t) * r->d);
  if (sign_bits) std::memcpy(sign_bits, r->sign_bits.data(), sizeof(uint32_t) * r->sign_bits.size());
  return OQ_OK;
}

void oq_free_rpbh(oq_rpbh_t r) {
  if (!r) return;
  int prev = -1;
  bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
  for (int dev = 0; dev < OQ_MAX_DEVICES; ++dev) {
    if (!r->dev_perm[dev] && !r->dev_signs[dev] && !r->dev_ctab[0][dev] && !r->dev_ctab[1][dev]) continue;
    if (cudaSetDevice(dev) == cudaSuccess) {
      cudaFree(r->dev_perm[dev]);
      cudaFree(r->dev_signs[dev]);
      cudaFree(r->dev_ctab[0][dev]);
      cudaFree(r->dev_ctab[1][dev]);
    }
  }
  if (have_prev) cudaSetDevice(prev);
  delete r;
}

int oq_build_codebook(int d, int bits, oq_codebook_t* out) {
  clear_error();
  if (!out) return fail(OQ_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (d < 3) return fail(OQ_ERR_ARG, "d must be >= 3 (got %d)", d);
  if (bits < 1 || bits > 8) return fail(OQ_ERR_ARG, "bits must be in 1..8 (got %d)", bits);
  oq_codebook_t cb = new (std::nothrow) oq_codebook_s;
  if (!cb) return fail(OQ_ERR_NOMEM, "allocating the codebook handle");
  cb->d = d;
  cb->bits = bits;
  lloyd_max(d, bits, cb->centroids, cb->bounds, cb->iterations, cb->distortion);
  cb->lut.resize(cb->centroids.size());
  const double sd = std::sqrt((double)d);
  for (size_t k = 0; k < cb->centroids.size(); ++k) cb->lut[k] = double_to_fp16_rne(sd * cb->centroids[k]);
  build_qtable(cb);
  // Upload the search table to the current device now when one is present.
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0) {
    const uint32_t* t;
    if (int rc = codebook_device_qtable(cb, &t)) {
      delete cb;
      return rc;
    }
  } else {
    cudaGetLastError();
  }
  *out = cb;
  return OQ_OK;
}

int oq_codebook_info(oq_codebook_t cb, int* d, int* bits) {
  clear_error();
  if (!cb) return fail(OQ_ERR_ARG, "NULL codebook handle");
  if (d) *d = cb->d;
  if (bits) *bits = cb->bits;
  return OQ_OK;
}

int oq_codebook_export(oq_codebook_t cb, double* centroids, double* bounds, uint16_t* lut_fp16, int* iterations,
                       double* distortion) {
  clear_error();
  if (!cb) return fail(OQ_ERR_ARG, "NULL codebook handle");
  if (centroids) std::memcpy(centroids, cb->centroids.data(), sizeof(double) * cb->centroids.size());
  if (bounds) std::memcpy(bounds, cb->bounds.data(), sizeof(double) * cb->bounds.size());
  if (lut_fp16) std::memcpy(lut_fp16, cb->lut.data(), sizeof(uint16_t) * cb->lut.size());
  if (iterations) *iterations = cb->iterations;
  if (distortion) *distortion = cb->distortion;
  return OQ_OK;
}

void oq_free_codebook(oq_codebook_t cb) {
  if (!cb) return;
  int prev = -1;
  bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
  for (int dev = 0; dev < OQ_MAX_DEVICES; ++dev) {
    if (!cb->dev_qtable[dev]) continue;
    if (cudaSetDevice(dev) == cudaSuccess) cudaFree(cb->dev_qtable[dev]);
  }
  if (have_prev) cudaSetDevice(prev);
  delete cb;
}

static int check_quant_args(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, const void* codes,
                            const void* norms) {
  if (!r || !cb) return fail(OQ_ERR_ARG, "NULL handle");
  if (M < 0) return fail(OQ_ERR_ARG, "M must be >= 0 (got %d)", M);
  // The codebook is C^(d,b) for the row width d; C^(h,b) for the rotation's
  // block h is accepted too (the literal reading of a "codebook for d = h" on
  // rows of width d: the rows are unit vectors either way).
  if (cb->d != r->d && cb->d != r->h)
    return fail(OQ_ERR_ARG, "codebook d=%d is neither the rows' d=%d nor the block %d", cb->d, r->d, r->h);
  if (r->d % 32 != 0 || r->d > 16384)
    return fail(OQ_ERR_UNSUPPORTED, "kernels need d %% 32 == 0 and d <= 16384 (d=%d)", r->d);
  if (r->h < 32 || r->h > 1024) return fail(OQ_ERR_UNSUPPORTED, "kernels need 32 <= block <= 1024 (h=%d)", r->h);
  if (cb->bits > 6) return fail(OQ_ERR_UNSUPPORTED, "kernels need bits <= 6 (bits=%d)", cb->bits);
  if (M == 0) return OQ_OK;
  if (!X || !codes || !norms) return fail(OQ_ERR_ARG, "NULL buffer");
  if (!aligned16(X) || !aligned16(codes) || !aligned16(norms))
    return fail(OQ_ERR_ALIGN, "X, codes and norms must be 16-byte aligned");
  return OQ_OK;
}

int oq_quantize_act(oq_rpbh_t r, oq_codebook_t cb, const void* X, int M, uint8_t* codes, float* norms,
                    void* stream) {
  clear_error();
  NvtxRange nvtx("oq_quantize_act");
  if (int rc = check_quant_args(r, cb, X, M, codes, norms)) return rc;
  if (M == 0) return OQ_OK;
  return finish(launch_rotq(r, cb, X, M, codes, norms, nullptr, stream), stream);
}

int oq_row_flatness(const void* X, int M, int d, float* rho3, float* rhoinf, float* batch_max, void* stream) {
  clear_error();
  NvtxRange nvtx("oq_row_flatness");
  if (M < 0) return fail(OQ_ERR_ARG, "M must be >= 0 (got %d)", M);
  if (d < 8 || d % 8 != 0) return fail(OQ_ERR_UNSUPPORTED, "the flatness check needs d %% 8 == 0 (d=%d)", d);
  if (M > 0 && !X) return fail(OQ_ERR_ARG, "X is NULL");
  if (!aligned16(X)) return fail(OQ_ERR_ALIGN, "X must be 16-byte aligned");
  if (!rho3 && !rhoinf && !batch_max) return fail(OQ_ERR_ARG, "no output requested");
  if ((rho3 && ((uintptr_t)rho3 & 3u)) || (rhoinf && ((uintptr_t)rhoinf & 3u)) ||
      (batch_max && ((uintptr_t)batch_max & 3u)))
    return fail(OQ_ERR_ALIGN, "outputs must be 4-byte aligned");
  return finish(launch_flatness(X, M, d, rho3, rhoinf, batch_max, stream), stream);
}

int oq_quantize_weight(oq_rpbh_t r, oq_codebook_t cb, const void* W, int N, uint8_t* codes, void* norms_bf16,
                       void* stream) {
  clear_error();
  NvtxRange nvtx("oq_quantize_weight");
  if (int rc = check_quant_args(r, cb, W, N, codes, norms_bf16)) return rc;
  if (N == 0) return OQ_OK;
  return finish(launch_rotq(r, cb, W, N, codes, nullptr, (uint16_t*)norms_bf16, stream), stream);
}

size_t oq_linear_workspace_bytes(int M, int d, int bits_a) {
  if (M <= 0 || d <= 0 || bits_a <= 0) return 0;
  size_t code_bytes = ((size_t)M * (size_t)d * (size_t)bits_a + 7) / 8;
  code_bytes = (code_bytes + 255) & ~(size_t)255;
  return code_bytes + 4 * (size_t)M;
}

static int check_linear_args(int d, oq_codebook_t cb_a, oq_codebook_t cb_w, int M, const void* w_codes,
                             const void* w_norm, int N, const void* bias, int epilogue, const void* Y_f32,
                             const void* Y_bf16) {
  if (!cb_a || !cb_w) return fail(OQ_ERR_ARG, "NULL codebook handle");
  if (cb_a->d != cb_w->d || cb_a->d <= 0 || d % cb_a->d != 0)
    return fail(OQ_ERR_ARG, "codebook dims (%d, %d) must be equal and divide d=%d", cb_a->d, cb_w->d, d);
  if (M < 0 || N < 0) return fail(OQ_ERR_ARG, "M and N must be >= 0");
  if (epilogue != OQ_EPI_NONE && epilogue != OQ_EPI_GELU) return fail(OQ_ERR_ARG, "unknown epilogue %d", epilogue);
  if (d % 64 != 0) return fail(OQ_ERR_UNSUPPORTED, "the GEMM needs d %% 64 == 0 (d=%d)", d);
  if (N % 16 != 0) return fail(OQ_ERR_UNSUPPORTED, "the GEMM needs N %% 16 == 0 (N=%d)", N);
  auto ok_bits = [](int b) { return b == 2 || b == 4 || b == 6; };
  const bool w3a3 = cb_a->bits == 3 && cb_w->bits == 3;
  if (!w3a3 && (!ok_bits(cb_a->bits) || !ok_bits(cb_w->bits)))
    return fail(OQ_ERR_UNSUPPORTED, "the GEMM needs bits in {2,4,6}, or 3 for both (a=%d, w=%d)", cb_a->bits,
                cb_w->bits);
  if (w3a3 && d % 128 != 0) return fail(OQ_ERR_UNSUPPORTED, "3-bit codes need d %% 128 == 0 (d=%d)", d);
  if (M == 0 || N == 0) return OQ_OK;
  if (!Y_f32 && !Y_bf16) return fail(OQ_ERR_ARG, "at least one of Y_f32 / Y_bf16 is needed");
  if (!w_codes || !w_norm) return fail(OQ_ERR_ARG, "NULL weight buffer");
  if (!aligned16(w_codes) || !aligned16(w_norm) || (bias && !aligned16(bias)) || (Y_f32 && !aligned16(Y_f32)) ||
      (Y_bf16 && !aligned16(Y_bf16)))
    return fail(OQ_ERR_ALIGN, "GEMM buffers must be 16-byte aligned");
  return OQ_OK;
}

int oq_linear_codes(int d, oq_codebook_t cb_a, oq_codebook_t cb_w, const uint8_t* a_codes, const float* a_norm,
                    int M, const uint8_t* w_codes, const void* w_norm, int N, const void* bias, int epilogue,
                    float* Y_f32, void* Y_bf16, void* stream) {
  clear_error();
  NvtxRange nvtx("oq_linear_codes");
  if (int rc = check_linear_args(d, cb_a, cb_w, M, w_codes, w_norm, N, bias, epilogue, Y_f32, Y_bf16)) return rc;
  if (M == 0 || N == 0) return OQ_OK;
  if (!a_codes || !a_norm) return fail(OQ_ERR_ARG, "NULL activation buffer");
  if (!aligned16(a_codes) || !aligned16(a_norm)) return fail(OQ_ERR_ALIGN, "activation buffers must be 16-byte aligned");
  return finish(launch_cbgemm(d, cb_a, cb_w, a_codes, a_norm, M, w_codes, (const uint16_t*)w_norm, N,
                              (const uint16_t*)bias, epilogue, Y_f32, (uint16_t*)Y_bf16, stream),
                stream);
}

int oq_linear(oq_rpbh_t r, oq_codebook_t cb_a, oq_codebook_t cb_w, const void* X, int M, const uint8_t* w_codes,
              const void* w_norm, int N, const void* bias, int epilogue, float* Y_f32, void* Y_bf16,
              void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  NvtxRange nvtx("oq_linear");
  if (!r) return fail(OQ_ERR_ARG, "NULL rpbh handle");
  if (int rc = check_linear_args(r->d, cb_a, cb_w, M, w_codes, w_norm, N, bias, epilogue, Y_f32, Y_bf16)) return rc;
  if (M == 0 || N == 0) return OQ_OK;
  size_t need = oq_linear_workspace_bytes(M, r->d, cb_a->bits);
  if (!workspace || workspace_bytes < need)
    return fail(OQ_ERR_ARG, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(OQ_ERR_ALIGN, "workspace must be 16-byte aligned");
  uint8_t* a_codes = (uint8_t*)workspace;
  size_t code_bytes = need - 4 * (size_t)M;
  float* a_norm = (float*)((uint8_t*)workspace + code_bytes);
  if (int rc = check_quant_args(r, cb_a, X, M, a_codes, a_norm)) return rc;
  if (int rc = finish(launch_rotq(r, cb_a, X, M, a_codes, a_norm, nullptr, stream), stream)) return rc;
  return finish(launch_cbgemm(r->d, cb_a, cb_w, a_codes, a_norm, M, w_codes, (const uint16_t*)w_norm, N,
                              (const uint16_t*)bias, epilogue, Y_f32, (uint16_t*)Y_bf16, stream),
                stream);
}

}  // extern "C"
