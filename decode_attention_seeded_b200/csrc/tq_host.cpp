// Host side of libtq: context, seeded tables, Lloyd-Max codebooks, argument
// checks and launch plumbing for the C ABI declared in include/tq.h.
//
// The seeded tables and the codebooks are computed here, on the host, in
// double precision, and uploaded once (cold path).

#include "tq.h"
#include "tq_internal.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

namespace {

// ---------------------------------------------------------------- SplitMix64
// Steele, Lea & Flood, "Fast splittable pseudorandom number generators"
// (OOPSLA 2014): the state advances by the golden gamma, each output is the
// 64-bit finaliser of the new state. Output j of seed s mixes s + (j+1)*gamma.
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
inline uint64_t splitmix_at(uint64_t seed, uint64_t j) { return mix64(seed + (j + 1) * kGamma); }

// ------------------------------------------------------- binary16 conversion
// Round a double to the nearest IEEE binary16 (ties to even); returns the bits.
uint16_t to_half_bits(double x) {
  const uint16_t sign = std::signbit(x) ? 0x8000u : 0u;
  const double a = std::fabs(x);
  if (std::isnan(x)) return 0x7E00u;
  if (a >= 65520.0) return sign | 0x7C00u;           // at or past the midpoint to infinity
  int e2 = 0;
  std::frexp(a, &e2);                                 // a = f * 2^e2, f in [0.5, 1)
  int E = e2 - 1;                                     // a = 1.m * 2^E
  if (a == 0.0) return sign;
  if (E < -14) {                                      // subnormal: quantum 2^-24
    const double r = std::nearbyint(std::ldexp(a, 24));
    return sign | static_cast<uint16_t>(r);           // r == 1024 is the smallest normal
  }
  double r = std::nearbyint(std::ldexp(a, 10 - E));  // in [1024, 2048]
  uint32_t mant = static_cast<uint32_t>(r);
  if (mant == 2048u) { mant = 1024u; ++E; }
  if (E > 15) return sign | 0x7C00u;
  return sign | static_cast<uint16_t>(((E + 15) << 10) | (mant - 1024u));
}

double half_bits_to_double(uint16_t h) {
  const int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = std::ldexp(static_cast<double>(m), -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp(static_cast<double>(m + 1024), e - 25);
  return s ? -v : v;
}

// --------------------------------------------------------- Lloyd-Max (host)
// Density of one coordinate of a uniform point on S^(d-1): (1 - t^2)^k,
// k = (d - 3) / 2, on [-1, 1]. Cell masses by composite Gauss-Legendre
// quadrature, first moments in closed form: the integral of t (1-t^2)^k is
// -(1-t^2)^(k+1) / (2(k+1)). The normalising constant cancels in the
// conditional means.
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));   // Tricomi initial guess
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;                            // Legendre recurrence
        for (int k = 2; k <= n; ++k) {
          const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        const double dp = n * (z * p1 - p0) / (z * z - 1.0);
        const double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) {
          x[i] = z;
          w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
          break;
        }
        x[i] = z;
        w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
      }
    }
  }
};

double cell_mass(double a, double b, double k) {
  static const GaussLegendre gl(24);
  const int panels = 48;
  const double h = (b - a) / panels;
  double sum = 0.0;
  for (int p = 0; p < panels; ++p) {
    const double mid = a + (p + 0.5) * h;
    double part = 0.0;
    for (size_t i = 0; i < gl.x.size(); ++i) {
      const double t = mid + 0.5 * h * gl.x[i];
      const double u = 1.0 - t * t;
      part += gl.w[i] * (u > 0.0 ? std::pow(u, k) : 0.0);
    }
    sum += 0.5 * h * part;
  }
  return sum;
}

double cell_moment1(double a, double b, double k) {
  const double ua = std::max(0.0, 1.0 - a * a), ub = std::max(0.0, 1.0 - b * b);
  return (std::pow(ua, k + 1.0) - std::pow(ub, k + 1.0)) / (2.0 * (k + 1.0));
}

// Positive-half Lloyd-Max centroids for 2*levels cells.
std::vector<double> lloyd_positive(int d, int levels) {
  const double k = 0.5 * (d - 3);
  const double half = cell_mass(0.0, 1.0, k);
  std::vector<double> c(levels);
  for (int j = 0; j < levels; ++j) {                 // start at the level quantiles
    const double target = half * (j + 0.5) / levels;
    double lo = 0.0, hi = 1.0;
    for (int it = 0; it < 80; ++it) {
      const double mid = 0.5 * (lo + hi);
      (cell_mass(0.0, mid, k) < target ? lo : hi) = mid;
    }
    c[j] = 0.5 * (lo + hi);
  }
  double best = INFINITY;
  int stall = 0;
  std::vector<double> b(levels + 1);
  for (int it = 0; it < 200000; ++it) {
    b[0] = 0.0;
    b[levels] = 1.0;
    for (int j = 1; j < levels; ++j) b[j] = 0.5 * (c[j - 1] + c[j]);
    double delta = 0.0, cmax = 0.0;
    for (int j = 0; j < levels; ++j) {
      const double nc = cell_moment1(b[j], b[j + 1], k) / cell_mass(b[j], b[j + 1], k);
      delta = std::max(delta, std::fabs(nc - c[j]));
      c[j] = nc;
      cmax = std::max(cmax, std::fabs(nc));
    }
    if (delta <= 16.0 * 2.220446049250313e-16 * cmax) {
      stall = (delta >= best) ? stall + 1 : 0;
      best = std::min(best, delta);
      if (delta == 0.0 || stall >= 3) break;
    }
  }
  return c;
}

struct StoredCodebook {
  std::vector<uint16_t> half_bits;   // ascending fp16 centroids
  std::vector<float> thresholds;     // midpoints, fp32-exact
  bool ok = false;
};

StoredCodebook make_codebook(int bits, int d) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, StoredCodebook> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(bits, d);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  StoredCodebook cb;
  const int L = 1 << (bits - 1);
  std::vector<double> pos = lloyd_positive(d, L);
  std::vector<double> full(2 * L);
  for (int j = 0; j < L; ++j) {
    full[L + j] = pos[j];
    full[L - 1 - j] = -pos[j];
  }
  cb.half_bits.resize(2 * L);
  std::vector<double> c16(2 * L);
  for (int j = 0; j < 2 * L; ++j) {
    cb.half_bits[j] = to_half_bits(full[j]);
    c16[j] = half_bits_to_double(cb.half_bits[j]);
  }
  cb.ok = true;
  cb.thresholds.resize(2 * L - 1);
  for (int j = 0; j + 1 < 2 * L; ++j) {
    const double mid = 0.5 * (c16[j] + c16[j + 1]);
    cb.thresholds[j] = static_cast<float>(mid);
    if (static_cast<double>(cb.thresholds[j]) != mid) cb.ok = false;
    if (!(c16[j] < c16[j + 1])) cb.ok = false;
  }
  cache[key] = cb;
  return cb;
}

}  // namespace

// ====================================================================== context
struct tq_ctx {
  int device = 0;
  int sm_count = 0;                // streaming multiprocessors of the device (sizes decode grids)
  float sparse_tau = 0.0f;         // Sparse V threshold of the decode calls (0: dense)
  bool rot_ready = false, cb_ready = false;
  float* d_signs = nullptr;        // [2][128]: D_K then D_V
  uint16_t* d_sketch_t = nullptr;  // fp16 bits: S^T, M = S R_K (high, low) as decode A fragments, S as prefill B fragments
  unsigned* d_err = nullptr;
  tq::Tables tables;
};

namespace {

class DeviceGuard {               // make ctx->device current for the scope
 public:
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev_) != cudaSuccess) prev_ = -1;
    if (prev_ != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    if (prev_ >= 0) cudaSetDevice(prev_);
  }
 private:
  int prev_ = -1;
};

bool valid_bits(int b) { return b >= 2 && b <= 4; }
bool valid_key_bits(int b) { return valid_bits(b) || b == 8; }   // 8: q8_0 keys
size_t block_bytes_for(int bk, int bv) {
  return bk == 8 ? 2176u + 256u * bv + 32u : 256u * (bk + bv + 1) + 96u;
}

tq_status fill_codebook_tables(tq::Tables& t, int bk, int bv) {
  const bool q8 = bk == 8;                  // q8_0 keys carry no key codebook
  StoredCodebook ck = make_codebook(q8 ? 2 : bk, tq::kHeadDim), cv = make_codebook(bv, tq::kHeadDim);
  if (!ck.ok || !cv.ok) return TQ_ERR_UNSUPPORTED;
  std::memset(t.thr_k, 0, sizeof t.thr_k);
  std::memset(t.thr_v, 0, sizeof t.thr_v);
  std::memset(t.cen_k, 0, sizeof t.cen_k);
  std::memset(t.cen_v, 0, sizeof t.cen_v);
  std::memset(t.kq_hi, 0, sizeof t.kq_hi);
  std::memset(t.kq_lo, 0, sizeof t.kq_lo);
  std::memset(t.v_lo, 0, sizeof t.v_lo);
  std::memset(t.v_hi, 0, sizeof t.v_hi);
  const int nk = q8 ? 0 : 1 << bk, nv = 1 << bv;
  double kmax = 0.0;
  for (int j = 0; j < nk; ++j) {
    t.cen_k[j] = static_cast<float>(half_bits_to_double(ck.half_bits[j]));
    kmax = std::max(kmax, std::fabs(static_cast<double>(t.cen_k[j])));
    if (j + 1 < nk) t.thr_k[j] = ck.thresholds[j];
  }
  for (int j = 0; j < nv; ++j) {
    t.cen_v[j] = static_cast<float>(half_bits_to_double(cv.half_bits[j]));
    if (j + 1 < nv) t.thr_v[j] = cv.thresholds[j];
    const uint16_t h = cv.half_bits[j];
    t.v_lo[j >> 2] |= static_cast<uint32_t>(h & 0xFFu) << (8 * (j & 3));
    t.v_hi[j >> 2] |= static_cast<uint32_t>(h >> 8) << (8 * (j & 3));
  }
  // Key centroids as exact int16 values C = c * 2^E split C = 256*hi + lo.
  int E = q8 ? 0 : static_cast<int>(std::floor(std::log2(32639.0 / kmax)));
  for (int j = 0; j < nk; ++j) {
    const double C = std::ldexp(static_cast<double>(t.cen_k[j]), E);
    if (C != std::floor(C) || std::fabs(C) > 32639.0) return TQ_ERR_UNSUPPORTED;
    const int ci = static_cast<int>(C);
    const int hi = (ci + 128) >> 8;   // floor division
    const int lo = ci - 256 * hi;
    t.kq_hi[j >> 2] |= static_cast<uint32_t>(static_cast<uint8_t>(static_cast<int8_t>(hi))) << (8 * (j & 3));
    t.kq_lo[j >> 2] |= static_cast<uint32_t>(static_cast<uint8_t>(static_cast<int8_t>(lo))) << (8 * (j & 3));
  }
  t.k_exp = E;
  t.key_bits = bk;
  t.value_bits = bv;
  t.block_bytes = static_cast<int>(block_bytes_for(bk, bv));
  return TQ_OK;
}

tq_status check_device(const tq_ctx* ctx) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return TQ_ERR_CUDA;
  return cur == ctx->device ? TQ_OK : TQ_ERR_INVALID_ARG;
}

tq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

}  // namespace

namespace tq {

DecodePlan make_plan(int batch, int n_q, int n_kv, int max_seq_len, int sm_count) {
  DecodePlan p{};
  p.batch = batch;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.group = n_q / n_kv;
  p.n_hg = (p.group + 3) / 4;                    // groups of 4 query heads
  p.max_pages = std::max(1, (max_seq_len + kPage - 1) / kPage);
  const int pairs = batch * n_kv;
  p.n_pairs = pairs;
  // One resident CTA per SM: split each (sequence, KV head) into as many chunks
  // as keep every SM busy in one wave, each chunk at least kMinChunkPages pages
  // and at most kMaxChunkPages (its block-table window is cached in shared memory).
  int chunks = std::max(1, sm_count / pairs);
  int ppc = (p.max_pages + chunks - 1) / chunks;
  ppc = std::min(std::max(ppc, kMinChunkPages), kMaxChunkPages);
  p.pages_per_chunk = ppc;
  p.chunks = (p.max_pages + ppc - 1) / ppc;
  p.grid = p.chunks * pairs;
  // Balanced mode when the uniform split is SM-limited and leaves more than 5 % of
  // the SMs idle, or needs more than one wave: the split then follows the actual
  // (ragged) lengths, read on the device.
  const int sm_chunks = std::max(1, sm_count / pairs);
  const bool sm_limited = p.chunks == sm_chunks && pairs <= sm_count;
  const bool idle = sm_limited && (sm_count - p.chunks * pairs) * 20 > sm_count;
  p.balanced = 0;
  if ((idle || pairs > sm_count) && batch <= kMaxBalancedBatch) {
    const int seg_w = std::max(8, 36 / p.n_hg);
    const int64_t all = static_cast<int64_t>(pairs) * (p.max_pages + seg_w);
    const int64_t share = std::max<int64_t>(kMinShare, (all + sm_count - 1) / sm_count) + 2;
    if (share <= kMaxChunkPages) {
      p.balanced = 1;
      p.shares = sm_count;
      p.grid = sm_count;                           // one CTA per share
      p.seg_w = seg_w;
      p.min_share = kMinShare;
      p.pages_per_chunk = static_cast<int>(share);
    }
  }
  // records: uniform, one per (pair, chunk); balanced, one per segment, at slot
  // share + pair ordinal (below shares + pairs)
  const size_t records = p.balanced ? static_cast<size_t>(p.shares) + pairs : static_cast<size_t>(pairs) * p.chunks;
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  size_t off = 0;
  p.off_partial = off;
  off = al(off + records * p.n_hg * 4 * 132 * sizeof(float));
  p.off_counter = off;
  off = al(off + static_cast<size_t>(pairs) * sizeof(unsigned));
  p.total = off;
  return p;
}

}  // namespace tq

// ======================================================================== ABI
extern "C" {

int tq_version(void) { return 100; }

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported geometry or bit width";
    case TQ_ERR_WORKSPACE: return "workspace too small or misaligned";
    case TQ_ERR_CUDA: return "CUDA runtime error";
    case TQ_ERR_DEVICE: return "device error word set";
    case TQ_ERR_NOT_INITIALIZED: return "rotation or codebooks not initialised";
  }
  return "unknown status";
}

tq_status tq_host_sign_vector(uint64_t seed, int d, int8_t* out) {
  if (!out || d <= 0) return TQ_ERR_INVALID_ARG;
  for (int i = 0; i < d; ++i) out[i] = (splitmix_at(seed, i) >> 63) ? -1 : 1;
  return TQ_OK;
}

tq_status tq_host_gaussian_sketch(uint64_t seed, int m, int d, uint16_t* out) {
  if (!out || m <= 0 || d <= 0) return TQ_ERR_INVALID_ARG;
  const double two53 = 1.0 / 9007199254740992.0;   // 2^-53
  for (int64_t idx = 0; idx < static_cast<int64_t>(m) * d; ++idx) {
    const uint64_t w1 = splitmix_at(seed, 2 * idx), w2 = splitmix_at(seed, 2 * idx + 1);
    const double u1 = static_cast<double>(w1 >> 11) * two53 + two53;    // (0, 1]
    const double u2 = static_cast<double>(w2 >> 11) * two53;            // [0, 1)
    const double z = std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * M_PI * u2);
    out[idx] = to_half_bits(z);
  }
  return TQ_OK;
}

tq_status tq_host_codebook(int bits, int d, uint16_t* centroids, float* thresholds) {
  if (!centroids || !thresholds || bits < 1 || bits > 4 || d < 4) return TQ_ERR_INVALID_ARG;
  StoredCodebook cb = make_codebook(bits, d);
  if (!cb.ok) return TQ_ERR_UNSUPPORTED;
  std::memcpy(centroids, cb.half_bits.data(), cb.half_bits.size() * sizeof(uint16_t));
  std::memcpy(thresholds, cb.thresholds.data(), cb.thresholds.size() * sizeof(float));
  return TQ_OK;
}

tq_status tq_create(tq_ctx** out, int head_dim, int qjl_rows, int page_size, int device) {
  if (!out) return TQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (head_dim != tq::kHeadDim || qjl_rows != tq::kQjlRows || page_size != tq::kPage)
    return TQ_ERR_UNSUPPORTED;
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || device < 0 || device >= n) return TQ_ERR_CUDA;
  DeviceGuard guard(device);
  tq_ctx* c = new tq_ctx;
  c->device = device;
  cudaError_t e = cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, device);
  if (e == cudaSuccess && c->sm_count <= 0) e = cudaErrorInvalidDevice;
  if (e == cudaSuccess) e = cudaMalloc(&c->d_signs, 2 * tq::kHeadDim * sizeof(float));
  if (e == cudaSuccess) e = cudaMalloc(&c->d_sketch_t, 5 * tq::kQjlRows * tq::kHeadDim * sizeof(uint16_t));
  if (e == cudaSuccess) e = cudaMalloc(&c->d_err, sizeof(unsigned));
  if (e == cudaSuccess) e = cudaMemset(c->d_err, 0, sizeof(unsigned));
  if (e != cudaSuccess) {
    tq_destroy(c);
    return TQ_ERR_CUDA;
  }
  c->tables.signs_k = c->d_signs;
  c->tables.signs_v = c->d_signs + tq::kHeadDim;
  c->tables.sketch_t = c->d_sketch_t;
  c->tables.sketch_m = c->d_sketch_t + tq::kQjlRows * tq::kHeadDim;
  c->tables.sketch_qb = c->d_sketch_t + 3 * tq::kQjlRows * tq::kHeadDim;
  c->tables.sketch_umma = c->d_sketch_t + 4 * tq::kQjlRows * tq::kHeadDim;
  c->tables.err = c->d_err;
  *out = c;
  return TQ_OK;
}

void tq_destroy(tq_ctx* ctx) {
  if (!ctx) return;
  {
    DeviceGuard guard(ctx->device);
    if (ctx->d_signs) cudaFree(ctx->d_signs);
    if (ctx->d_sketch_t) cudaFree(ctx->d_sketch_t);
    if (ctx->d_err) cudaFree(ctx->d_err);
  }
  delete ctx;
}

tq_status tq_init_rotation(tq_ctx* ctx, uint64_t seed_k, uint64_t seed_v, uint64_t seed_s,
                           tq_stream stream) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  if (tq_status st = check_device(ctx)) return st;
  const int d = tq::kHeadDim, m = tq::kQjlRows;
  std::vector<int8_t> sk(d), sv(d);
  std::vector<uint16_t> s(m * d), st(5 * m * d);
  tq_host_sign_vector(seed_k, d, sk.data());
  tq_host_sign_vector(seed_v, d, sv.data());
  tq_host_gaussian_sketch(seed_s, m, d, s.data());
  std::vector<float> signs(2 * d);
  for (int i = 0; i < d; ++i) {
    signs[i] = sk[i];
    signs[d + i] = sv[i];
  }
  for (int r = 0; r < m; ++r)
    for (int c = 0; c < d; ++c) st[c * m + r] = s[r * d + c];   // S^T
  // M = S R_K with R_K = H D_K / sqrt(d), so that p = S q~ = M q needs no rotated
  // query: row r of S H is the Walsh-Hadamard transform of row r of S. M is kept
  // as fp16 high and low parts (M ~ hi + lo to about 22 bits) in m16n8k16 A
  // fragment order: warp w (rows 16w..16w+15), k-step ks (columns 16ks..16ks+15),
  // lane (g, t), register j -> row 16w + g + 8(j&1), fp16 pair at columns
  // 16ks + 2t + 8(j>>1) (+0, +1). Stored [hi/lo][w][ks][lane][j], so one warp's
  // register set for one k-step is 512 contiguous bytes.
  // S as m16n8k16 B fragments of the prefill product z = S u (tokens on rows):
  // coordinates and sketch rows both follow a lane's layout chunk. Coordinate
  // of k-step ks, k index kk: 16 ks + 4 tk + slot (tk = kk >> 1 mod 4, slot =
  // kk & 1, + 2 when kk >= 8); sketch row of n-tile nt, column c:
  // 32 (nt >> 2) + 16 ((nt >> 1) & 1) + 4 (c >> 1) + 2 (nt & 1) + (c & 1).
  // Stored [ks][nt][lane][2 regs], lane (g, t): reg 0 = k 2t, 2t+1, reg 1 = k
  // 2t+8, 2t+9, column g.
  uint16_t* qb = st.data() + 3 * m * d;
  for (int ks = 0; ks < d / 16; ++ks)
    for (int nt = 0; nt < m / 8; ++nt)
      for (int lane = 0; lane < 32; ++lane)
        for (int r = 0; r < 2; ++r)
          for (int h = 0; h < 2; ++h) {
            const int kk = 2 * (lane & 3) + 8 * r + h, c = lane >> 2;
            const int tk = (kk & 7) >> 1, slot = (kk & 1) + 2 * (kk >> 3);
            const int coord = 16 * ks + 4 * tk + slot;
            const int row = 32 * (nt >> 2) + 16 * ((nt >> 1) & 1) + 4 * (c >> 1) + 2 * (nt & 1) + (c & 1);
            qb[(((ks * (m / 8) + nt) * 32 + lane) * 2 + r) * 2 + h] = s[row * d + coord];
          }
  // S as the B operand of the tensor-core prefill product (K-major, no swizzle):
  // operand row n = 8 nt + c holds the sketch row of n-tile nt, column c above;
  // coordinate k of row n at element 1024 (n >> 3) + 64 (k >> 3) + 8 (n & 7) + (k & 7),
  // i.e. 8-row x 8-coordinate core matrices of 128 bytes, K-adjacent ones 128 bytes
  // apart and 8-row groups 2048 bytes apart.
  uint16_t* bu = st.data() + 4 * m * d;
  for (int nt = 0; nt < m / 8; ++nt)
    for (int c = 0; c < 8; ++c) {
      const int row = 32 * (nt >> 2) + 16 * ((nt >> 1) & 1) + 4 * (c >> 1) + 2 * (nt & 1) + (c & 1);
      for (int kk = 0; kk < d; ++kk) bu[1024 * nt + 64 * (kk >> 3) + 8 * c + (kk & 7)] = s[row * d + kk];
    }
  std::vector<uint16_t> mhi(m * d), mlo(m * d);
  double rownorm = 0.0;
  for (int r = 0; r < m; ++r) {
    std::vector<double> row(d);
    for (int c = 0; c < d; ++c) row[c] = half_bits_to_double(s[r * d + c]);
    for (int len = 1; len < d; len <<= 1)            // row H (H symmetric, unnormalised)
      for (int i = 0; i < d; i += 2 * len)
        for (int k = i; k < i + len; ++k) {
          const double a = row[k], bb = row[k + len];
          row[k] = a + bb;
          row[k + len] = a - bb;
        }
    double nn = 0.0;
    for (int c = 0; c < d; ++c) {
      const double v = row[c] * sk[c] / std::sqrt(static_cast<double>(d));
      mhi[r * d + c] = to_half_bits(v);
      mlo[r * d + c] = to_half_bits(v - half_bits_to_double(mhi[r * d + c]));
      const double kept = half_bits_to_double(mhi[r * d + c]) + half_bits_to_double(mlo[r * d + c]);
      nn += kept * kept;
    }
    rownorm = std::max(rownorm, std::sqrt(nn));
  }
  for (int hl = 0; hl < 2; ++hl) {
    const std::vector<uint16_t>& src = hl ? mlo : mhi;
    uint16_t* frag = st.data() + m * d + hl * m * d;
    for (int w = 0; w < m / 16; ++w)
      for (int ks = 0; ks < d / 16; ++ks)
        for (int lane = 0; lane < 32; ++lane)
          for (int j = 0; j < 4; ++j) {
            const int row = 16 * w + (lane >> 2) + 8 * (j & 1);
            const int col = 16 * ks + 2 * (lane & 3) + 8 * (j >> 1);
            const int o = (((w * (d / 16) + ks) * 32 + lane) * 4 + j) * 2;
            frag[o] = src[row * d + col];
            frag[o + 1] = src[row * d + col + 1];
          }
  }
  ctx->tables.m_rownorm = static_cast<float>(rownorm * (1.0 + 1e-6));
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // Synchronous copies from pageable memory: this is the cold set-up path.
  cudaError_t e = cudaMemcpyAsync(ctx->d_signs, signs.data(), 2 * d * sizeof(float),
                                  cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(ctx->d_sketch_t, st.data(), st.size() * sizeof(uint16_t),
                        cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  ctx->rot_ready = true;
  return TQ_OK;
}

tq_status tq_init_codebooks(tq_ctx* ctx, int key_bits, int value_bits, tq_stream stream) {
  (void)stream;
  if (!ctx) return TQ_ERR_INVALID_ARG;
  if (!valid_key_bits(key_bits) || !valid_bits(value_bits)) return TQ_ERR_UNSUPPORTED;
  tq::Tables t = ctx->tables;
  if (tq_status st = fill_codebook_tables(t, key_bits, value_bits)) return st;
  ctx->tables = t;
  ctx->cb_ready = true;
  return TQ_OK;
}

size_t tq_block_bytes(const tq_ctx* ctx) {
  if (!ctx || !ctx->cb_ready) return 0;
  return block_bytes_for(ctx->tables.key_bits, ctx->tables.value_bits);
}

size_t tq_page_bytes(const tq_ctx* ctx, int n_kv_heads) {
  if (n_kv_heads <= 0) return 0;
  return tq_block_bytes(ctx) * static_cast<size_t>(n_kv_heads);
}

static tq_status check_quantize_args(tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                                     int n_tokens, int n_kv_heads, const void* map, void* cache,
                                     int64_t n_cache_pages) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  if (!ctx->rot_ready || !ctx->cb_ready) return TQ_ERR_NOT_INITIALIZED;
  if (n_tokens < 0 || n_kv_heads <= 0 || n_cache_pages <= 0) return TQ_ERR_INVALID_ARG;
  if (dtype != TQ_F32 && dtype != TQ_BF16 && dtype != TQ_F16) return TQ_ERR_UNSUPPORTED;
  if (n_tokens == 0) return TQ_OK;
  if (!k || !v || !map || !cache) return TQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(cache) % 16) return TQ_ERR_INVALID_ARG;
  const size_t es = dtype == TQ_F32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(k) % (4 * es) || reinterpret_cast<uintptr_t>(v) % (4 * es))
    return TQ_ERR_INVALID_ARG;
  return check_device(ctx);
}

tq_status tq_quantize_append(tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                             int n_tokens, int n_kv_heads, const int64_t* slot_mapping,
                             void* cache, int64_t n_cache_pages, tq_stream stream) {
  if (tq_status st = check_quantize_args(ctx, k, v, dtype, n_tokens, n_kv_heads, slot_mapping,
                                         cache, n_cache_pages))
    return st;
  if (n_tokens == 0) return TQ_OK;
  return from_cuda(tq::launch_quantize_append(ctx->tables, k, v, dtype, n_tokens, n_kv_heads,
                                              slot_mapping, cache, n_cache_pages,
                                              static_cast<cudaStream_t>(stream)));
}

tq_status tq_quantize_prefill(tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                              int n_tokens, int n_kv_heads, const int32_t* block_table,
                              int start_pos, void* cache, int64_t n_cache_pages, tq_stream stream) {
  if (start_pos < 0) return TQ_ERR_INVALID_ARG;
  if (tq_status st = check_quantize_args(ctx, k, v, dtype, n_tokens, n_kv_heads, block_table,
                                         cache, n_cache_pages))
    return st;
  if (n_tokens == 0) return TQ_OK;
  // rows are staged by bulk copies, which need 16-byte aligned sources
  if (reinterpret_cast<uintptr_t>(k) % 16 || reinterpret_cast<uintptr_t>(v) % 16) return TQ_ERR_INVALID_ARG;
  return from_cuda(tq::launch_quantize_prefill(ctx->tables, k, v, dtype, n_tokens, n_kv_heads,
                                               block_table, start_pos, cache, n_cache_pages,
                                               static_cast<cudaStream_t>(stream)));
}

size_t tq_decode_workspace_bytes(const tq_ctx* ctx, int batch, int n_q_heads, int n_kv_heads,
                                 int max_seq_len) {
  if (!ctx || batch <= 0 || n_kv_heads <= 0 || n_q_heads <= 0 || n_q_heads % n_kv_heads ||
      max_seq_len < 0)
    return 0;
  return tq::make_plan(batch, n_q_heads, n_kv_heads, max_seq_len, ctx->sm_count).total;
}

static tq_status check_decode_args(tq_ctx* ctx, const void* q, tq_dtype q_dtype, const void* cache,
                                   int64_t n_cache_pages, const int32_t* block_tables, int max_pages_per_seq,
                                   const int32_t* seq_lens, int batch, int n_q_heads, int n_kv_heads,
                                   int max_seq_len, float scale, const float* out, const void* workspace,
                                   size_t workspace_bytes, tq::DecodePlan* plan, bool need_workspace = true) {
  if (!ctx) return TQ_ERR_INVALID_ARG;
  if (!ctx->rot_ready || !ctx->cb_ready) return TQ_ERR_NOT_INITIALIZED;
  if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads ||
      max_seq_len < 0 || n_cache_pages <= 0 || max_pages_per_seq <= 0)
    return TQ_ERR_INVALID_ARG;
  if (n_q_heads / n_kv_heads > 16) return TQ_ERR_UNSUPPORTED;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16 && q_dtype != TQ_F16) return TQ_ERR_UNSUPPORTED;
  if (!q || !cache || !block_tables || !seq_lens || !out || (need_workspace && !workspace))
    return TQ_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_pages_per_seq) * tq::kPage < max_seq_len) return TQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(cache) % 16) return TQ_ERR_INVALID_ARG;
  const size_t es = q_dtype == TQ_F32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(q) % (4 * es)) return TQ_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
  *plan = tq::make_plan(batch, n_q_heads, n_kv_heads, max_seq_len, ctx->sm_count);
  if (need_workspace && (workspace_bytes < plan->total || reinterpret_cast<uintptr_t>(workspace) % 256))
    return TQ_ERR_WORKSPACE;
  return check_device(ctx);
}

tq_status tq_decode_attention(tq_ctx* ctx, const void* q, tq_dtype q_dtype, const void* cache,
                              int64_t n_cache_pages, const int32_t* block_tables,
                              int max_pages_per_seq, const int32_t* seq_lens, int batch,
                              int n_q_heads, int n_kv_heads, int max_seq_len, float scale,
                              float* out, void* workspace, size_t workspace_bytes,
                              tq_stream stream) {
  tq::DecodePlan plan;
  if (tq_status st = check_decode_args(ctx, q, q_dtype, cache, n_cache_pages, block_tables, max_pages_per_seq,
                                       seq_lens, batch, n_q_heads, n_kv_heads, max_seq_len, scale, out,
                                       workspace, workspace_bytes, &plan))
    return st;
  if (scale == 0.0f) scale = 1.0f / std::sqrt(static_cast<float>(tq::kHeadDim));
  return from_cuda(tq::launch_decode(ctx->tables, plan, q, q_dtype, cache, n_cache_pages,
                                     block_tables, max_pages_per_seq, seq_lens, max_seq_len,
                                     scale, out, workspace, ctx->sparse_tau,
                                     static_cast<cudaStream_t>(stream)));
}

tq_status tq_decode_step(tq_ctx* ctx, const void* k_new, const void* v_new, tq_dtype kv_dtype,
                         const void* q, tq_dtype q_dtype, void* cache, int64_t n_cache_pages,
                         const int32_t* block_tables, int max_pages_per_seq, const int32_t* seq_lens,
                         int batch, int n_q_heads, int n_kv_heads, int max_seq_len, float scale, float* out,
                         void* workspace, size_t workspace_bytes, tq_stream stream) {
  tq::DecodePlan plan;
  if (tq_status st = check_decode_args(ctx, q, q_dtype, cache, n_cache_pages, block_tables, max_pages_per_seq,
                                       seq_lens, batch, n_q_heads, n_kv_heads, max_seq_len, scale, out,
                                       workspace, workspace_bytes, &plan))
    return st;
  if (kv_dtype != TQ_F32 && kv_dtype != TQ_BF16 && kv_dtype != TQ_F16) return TQ_ERR_UNSUPPORTED;
  if (!k_new || !v_new) return TQ_ERR_INVALID_ARG;
  const size_t es = kv_dtype == TQ_F32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(k_new) % (4 * es) || reinterpret_cast<uintptr_t>(v_new) % (4 * es))
    return TQ_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = 1.0f / std::sqrt(static_cast<float>(tq::kHeadDim));
  return from_cuda(tq::launch_decode_step(ctx->tables, plan, k_new, v_new, kv_dtype, q, q_dtype, cache,
                                          n_cache_pages, block_tables, max_pages_per_seq, seq_lens, max_seq_len,
                                          scale, out, workspace, ctx->sparse_tau,
                                     static_cast<cudaStream_t>(stream)));
}

tq_status tq_decode_attention_noalloc(tq_ctx* ctx, const void* q, tq_dtype q_dtype, const void* cache,
                                      int64_t n_cache_pages, const int32_t* block_tables,
                                      int max_pages_per_seq, const int32_t* seq_lens, int batch,
                                      int n_q_heads, int n_kv_heads, int max_seq_len, float scale,
                                      float* out, tq_stream stream) {
  // Arguments first (nothing touches the device before they pass), then the size
  // limit, and only then the scratch address.
  tq::DecodePlan plan;
  if (tq_status st = check_decode_args(ctx, q, q_dtype, cache, n_cache_pages, block_tables, max_pages_per_seq,
                                       seq_lens, batch, n_q_heads, n_kv_heads, max_seq_len, scale, out,
                                       nullptr, 0, &plan, false))
    return st;
  if (plan.total > tq::kNoAllocScratchBytes) return TQ_ERR_WORKSPACE;   // use tq_decode_attention
  // The scratch address is looked up once per device and kept for the process
  // (it does not survive a cudaDeviceReset of that device).
  static std::mutex mu;
  static std::map<int, void*> scratch_of_device;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = scratch_of_device.find(ctx->device);
    if (it != scratch_of_device.end()) {
      scratch = it->second;
    } else {
      if (tq::noalloc_scratch(&scratch) != cudaSuccess || !scratch) return TQ_ERR_CUDA;
      scratch_of_device[ctx->device] = scratch;
    }
  }
  if (scale == 0.0f) scale = 1.0f / std::sqrt(static_cast<float>(tq::kHeadDim));
  return from_cuda(tq::launch_decode(ctx->tables, plan, q, q_dtype, cache, n_cache_pages,
                                     block_tables, max_pages_per_seq, seq_lens, max_seq_len,
                                     scale, out, scratch, ctx->sparse_tau,
                                     static_cast<cudaStream_t>(stream)));
}

tq_status tq_decode_logits(tq_ctx* ctx, const void* q, tq_dtype q_dtype, const void* cache,
                           int64_t n_cache_pages, const int32_t* block_tables, int max_pages_per_seq,
                           const int32_t* seq_lens, int batch, int n_q_heads, int n_kv_heads, int max_seq_len,
                           float scale, float* logits, int64_t logits_stride, tq_stream stream) {
  tq::DecodePlan plan;
  if (tq_status st = check_decode_args(ctx, q, q_dtype, cache, n_cache_pages, block_tables, max_pages_per_seq,
                                       seq_lens, batch, n_q_heads, n_kv_heads, max_seq_len, scale, logits,
                                       nullptr, 0, &plan, false))
    return st;
  if (logits_stride < max_seq_len) return TQ_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = 1.0f / std::sqrt(static_cast<float>(tq::kHeadDim));
  return from_cuda(tq::launch_logits(ctx->tables, plan, q, q_dtype, cache, n_cache_pages, block_tables,
                                     max_pages_per_seq, seq_lens, max_seq_len, scale, logits, logits_stride,
                                     static_cast<cudaStream_t>(stream)));
}

tq_status tq_set_test_flags(tq_ctx* ctx, unsigned flags) {
  if (!ctx || (flags & ~TQ_TEST_WAIT_RUNS_OUT)) return TQ_ERR_INVALID_ARG;
  ctx->tables.test_flags = flags;
  return TQ_OK;
}

tq_status tq_set_sparse_v(tq_ctx* ctx, float tau) {
  if (!ctx || !(tau >= 0.0f) || !(tau <= 1.0f)) return TQ_ERR_INVALID_ARG;
  ctx->sparse_tau = tau;
  return TQ_OK;
}

tq_status tq_get_device_error(tq_ctx* ctx, uint32_t* code, tq_stream stream) {
  if (!ctx || !code) return TQ_ERR_INVALID_ARG;
  if (tq_status st = check_device(ctx)) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  unsigned h = 0;
  cudaError_t e = cudaStreamSynchronize(cs);
  if (e == cudaSuccess) e = cudaMemcpy(&h, ctx->d_err, sizeof h, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(ctx->d_err, 0, sizeof h);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  *code = h;
  return TQ_OK;
}

}  // extern "C"
