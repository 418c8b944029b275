// CUDA kernels (sm_100a) of libtq: quantize/append, query transform and
// split-K decode attention over the packed paged cache.
//
// Method (pages: leviatan.io "Principe de quantification sans calibration";
// wis-web.com llama.cpp-fork post, PolarQuant and QJL paragraphs): each K/V
// vector x is rotated, y = H D x / (sqrt(d) |x|); every coordinate is coded
// with a fixed Lloyd-Max codebook; keys keep one sign bit per row of a seeded
// Gaussian sketch S applied to the residual u = y - c[code], and gamma = |x||u|.
// Decode estimates q.k = |k| <R q, c> + gamma sqrt(pi/2)/m <S R q, sign(S u)>.
//
// Block layout of one (page, KV head), 16 tokens (the same definition is
// written out in the header comment of the Python layout description):
//   [K codes 32 lanes x 8*bk B][sign bits 32 x 8 B][V codes 32 x 8*bv B][norms 96 B]
// Lane chunks are laid out so that lane (g, t) = (lane>>2, lane&3) of a warp
// finds in its own chunk exactly the bits of its mma.sync fragments:
//   keys:   B operand of m16n8k32 (k = coordinate, n = token), token halves th
//   signs:  B operand of m16n8k32 (k = sketch row,  n = token)
//   values: A operand of m16n8k16 (m = coordinate, k = token)

#include "tq.h"
#include "tq_internal.h"

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace tq {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSqrtPiOver2 = 1.2533141373155003f;
constexpr float kInvSqrtD = 0.08838834764831845f;      // 1/sqrt(128)
constexpr float kNegBig = -1.0e30f;                     // finite "minus infinity" for maxima

// --------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s));
  return d;
}

__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
  return v;
}
__device__ __forceinline__ uint32_t warp_or_lanes_mod4(uint32_t v) {
  // OR across the 8 lanes that share lane & 3
  v |= __shfl_xor_sync(kFull, v, 4);
  v |= __shfl_xor_sync(kFull, v, 8);
  v |= __shfl_xor_sync(kFull, v, 16);
  return v;
}

__device__ __forceinline__ void set_error(unsigned* err, unsigned bits) {
  if (err) atomicOr(err, bits);
}

// Four consecutive elements (4*lane .. 4*lane+3) of a 128-wide row.
__device__ __forceinline__ void load_row4(const void* base, size_t row, int dtype, int lane,
                                          float (&x)[4]) {
  if (dtype == TQ_F32) {
    const float4 v = reinterpret_cast<const float4*>(base)[row * 32 + lane];
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else {
    const uint2 raw = reinterpret_cast<const uint2*>(base)[row * 32 + lane];
    if (dtype == TQ_BF16) {
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
      const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
      x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
    } else {
      const __half2 a = *reinterpret_cast<const __half2*>(&raw.x);
      const __half2 b = *reinterpret_cast<const __half2*>(&raw.y);
      const float2 fa = __half22float2(a), fb = __half22float2(b);
      x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
    }
  }
}

// Natural-order Walsh-Hadamard transform of a 128-vector held 4 per lane
// (lane l owns elements 4l..4l+3): two in-lane butterfly stages, then five
// stages across lanes (element stride 4*2^s <-> lane bit s).
__device__ __forceinline__ void fwht128(float (&v)[4], int lane) {
  const float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2; v[1] = a1 + a3; v[2] = a0 - a2; v[3] = a1 - a3;
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const bool upper = (lane >> s) & 1;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(kFull, v[e], 1 << s);
      v[e] = upper ? (o - v[e]) : (v[e] + o);
    }
  }
}

// ============================================================ quantization
// One warp quantizes one 128-vector. Outputs per lane the codes of its four
// coordinates and (keys) the sign bits of sketch rows 4*lane .. 4*lane+3.
struct VecOut {
  int code[4];
  int sgn[4];
  float norm, gamma;
};

__device__ __forceinline__ int encode(float y, const float* thr, int n_thr) {
  int c = 0;
#pragma unroll
  for (int j = 0; j < 15; ++j)
    if (j < n_thr) c += (y > thr[j]) ? 1 : 0;
  return c;
}

// sketch_t: fp16 S^T ([d][m]) staged in shared memory by the calling kernel.
__device__ void quantize_vector(const float (&x)[4], const float* signs, const float* thr,
                                const float* cen, int bits, const __half* sketch_t, bool is_key,
                                int lane, VecOut& o) {
  float v[4];
  float ss = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    ss = fmaf(x[e], x[e], ss);
    v[e] = x[e] * signs[4 * lane + e];
  }
  ss = warp_sum(ss);
  const float n = sqrtf(ss);
  fwht128(v, lane);
  const float inv = n > 0.0f ? 1.0f / (n * 11.313708498984761f) : 0.0f;
  const int n_thr = (1 << bits) - 1;
  float u[4];
  float uu = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float y = v[e] * inv;
    o.code[e] = encode(y, thr, n_thr);
    u[e] = y - cen[o.code[e]];
    uu = fmaf(u[e], u[e], uu);
  }
  o.norm = n;
  o.gamma = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) o.sgn[e] = 0;
  if (!is_key) return;
  uu = warp_sum(uu);
  o.gamma = n * sqrtf(uu);
  // z_r = sum_c S[r][c] u_c for rows r = 4*lane + e; S^T rows are contiguous in r.
  float z[4] = {0.f, 0.f, 0.f, 0.f};
  const uint2* st = reinterpret_cast<const uint2*>(sketch_t);
#pragma unroll 16
  for (int c = 0; c < 128; ++c) {
    const float uc = __shfl_sync(kFull, u[c & 3], c >> 2);
    const uint2 raw = st[c * 32 + lane];
    const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    z[0] = fmaf(s01.x, uc, z[0]);
    z[1] = fmaf(s01.y, uc, z[1]);
    z[2] = fmaf(s23.x, uc, z[2]);
    z[3] = fmaf(s23.y, uc, z[3]);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) o.sgn[e] = z[e] >= 0.0f ? 1 : 0;
}

// Copy S^T (fp16, 32 KB) and the small code tables into shared memory.
__device__ __forceinline__ void stage_tables(const Tables& T, __half* s_sk, float* s_tab) {
  const uint4* src = reinterpret_cast<const uint4*>(T.sketch_t);
  uint4* dst = reinterpret_cast<uint4*>(s_sk);
  for (int i = threadIdx.x; i < kHeadDim * kQjlRows * 2 / 16; i += blockDim.x) dst[i] = __ldg(src + i);
  if (threadIdx.x < 16) {
    s_tab[threadIdx.x] = T.thr_k[threadIdx.x];
    s_tab[16 + threadIdx.x] = T.cen_k[threadIdx.x];
    s_tab[32 + threadIdx.x] = T.thr_v[threadIdx.x];
    s_tab[48 + threadIdx.x] = T.cen_v[threadIdx.x];
  }
  __syncthreads();
}

// Word and bit of code bit p for nibble q of selector j within a group of b words.
__device__ __forceinline__ void code_bit_pos(int b, int j, int q, int p, int& w, int& bit) {
  if (b == 2) {
    w = j >> 2;
    bit = 16 * (j & 1) + 4 * q + 2 * ((j >> 1) & 1) + p;
  } else if (b == 3) {
    if (j < 6) {
      w = j >> 1;
      bit = 16 * (j & 1) + 4 * q + p;
    } else {
      w = p;
      bit = 4 * (4 * (j - 6) + q) + 3;
    }
  } else {
    w = j >> 1;
    bit = 16 * (j & 1) + 4 * q + p;
  }
}

// Store one token's key codes, sign bits and key norms into a block. The key
// and sign words of a token belong to that token alone: plain stores.
__device__ void store_key_token(uint8_t* blk, int tau, int bk, const VecOut& o, int lane) {
  const int j = lane >> 2, t = lane & 3, g = tau & 7, th = tau >> 3;
  uint32_t words[4] = {0u, 0u, 0u, 0u};
  uint32_t sw = 0u;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    for (int p = 0; p < bk; ++p) {
      int w, bit;
      code_bit_pos(bk, j, e, p, w, bit);
      words[w] |= static_cast<uint32_t>((o.code[e] >> p) & 1) << bit;
    }
    sw |= static_cast<uint32_t>(o.sgn[e]) << (8 * e + j);
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) words[w] = warp_or_lanes_mod4(words[w]);
  sw = warp_or_lanes_mod4(sw);
  uint32_t* kw = reinterpret_cast<uint32_t*>(blk);
  if (lane < 4) {                    // lane == t here: writes lane chunk (g, t)
    const int base = (4 * g + t) * 2 * bk + th * bk;
    for (int w = 0; w < bk; ++w) kw[base + w] = words[w];
    uint32_t* sgw = reinterpret_cast<uint32_t*>(blk + 256 * bk);
    sgw[(4 * g + t) * 2 + th] = sw;
  }
}

// Value codes share words between the four tokens 2t, 2t+1, 8+2t, 9+2t of a
// lane chunk: clear-then-set with atomics (global or shared memory).
__device__ void store_value_token(uint8_t* blk, int tau, int bk, int bv, const VecOut& o, int lane) {
  uint32_t* vw = reinterpret_cast<uint32_t*>(blk + 256 * (bk + 1));
  const int tg = tau >> 3, t = (tau >> 1) & 3, et = tau & 1;
  const int mt = lane >> 2, hf = (lane >> 1) & 1;
  const int s = 2 * mt + tg, n = 2 * hf + et;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int r = 4 * (lane & 1) + e;
    const int chunk = 4 * r + t;
    for (int p = 0; p < bv; ++p) {
      int w, bit;
      if (bv == 3) {
        code_bit_pos(3, s & 7, n, p, w, bit);
        w += 3 * (s >> 3);
      } else {
        code_bit_pos(bv, s, n, p, w, bit);
      }
      unsigned* addr = vw + chunk * 2 * bv + w;
      const unsigned m = 1u << bit;
      if ((o.code[e] >> p) & 1) atomicOr(addr, m);
      else atomicAnd(addr, ~m);
    }
  }
}

__device__ __forceinline__ void store_norm(uint8_t* blk, int bk, int bv, int which, int tau, float v) {
  __half* nrm = reinterpret_cast<__half*>(blk + 256 * (bk + bv + 1));
  nrm[16 * which + tau] = __float2half_rn(v);
}

// One warp per (token, KV head): quantize K and V and store them at the slot.
__global__ void __launch_bounds__(256) quantize_append_kernel(Tables T, const void* k, const void* v,
                                                              int dtype, int n_tokens, int n_kv,
                                                              const int64_t* slots, uint8_t* cache,
                                                              int64_t n_pages) {
  extern __shared__ __align__(128) uint8_t smem[];
  __half* s_sk = reinterpret_cast<__half*>(smem);
  __shared__ float s_tab[64];     // thr_k, cen_k, thr_v, cen_v
  stage_tables(T, s_sk, s_tab);
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int wi = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wi < n_tokens * n_kv; wi += warps) {
    const int tok = wi / n_kv, h = wi % n_kv;
    const int64_t slot = slots[tok];
    if (slot < 0 || slot >= n_pages * kPage) {
      if (lane == 0) set_error(T.err, TQ_DEV_BAD_SLOT);
      continue;
    }
    const int64_t page = slot / kPage;
    const int tau = static_cast<int>(slot % kPage);
    uint8_t* blk = cache + (page * n_kv + h) * static_cast<int64_t>(T.block_bytes);
    float x[4];
    VecOut o;
    load_row4(k, static_cast<size_t>(tok) * n_kv + h, dtype, lane, x);
    quantize_vector(x, T.signs_k, s_tab, s_tab + 16, T.key_bits, s_sk, true, lane, o);
    store_key_token(blk, tau, T.key_bits, o, lane);
    if (lane == 0) {
      store_norm(blk, T.key_bits, T.value_bits, 0, tau, o.norm);
      store_norm(blk, T.key_bits, T.value_bits, 1, tau, o.gamma);
    }
    load_row4(v, static_cast<size_t>(tok) * n_kv + h, dtype, lane, x);
    quantize_vector(x, T.signs_v, s_tab + 32, s_tab + 48, T.value_bits, nullptr, false, lane, o);
    store_value_token(blk, tau, T.key_bits, T.value_bits, o, lane);
    if (lane == 0) store_norm(blk, T.key_bits, T.value_bits, 2, tau, o.norm);
  }
}

// One CTA per (page, KV head) of a contiguous run: the block is assembled in
// shared memory (merged with the page's previous contents if the run covers it
// only partly) and written back with 16-byte stores.
__global__ void __launch_bounds__(256) quantize_prefill_kernel(Tables T, const void* k, const void* v,
                                                               int dtype, int n_tokens, int n_kv,
                                                               const int32_t* block_table, int start_pos,
                                                               uint8_t* cache, int64_t n_pages) {
  extern __shared__ __align__(128) uint8_t smem[];
  __half* s_sk = reinterpret_cast<__half*>(smem);
  uint8_t* sblk = smem + kHeadDim * kQjlRows * 2;
  __shared__ float s_tab[64];     // thr_k, cen_k, thr_v, cen_v
  stage_tables(T, s_sk, s_tab);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int first_page = start_pos / kPage;
  const int last_page = (start_pos + n_tokens - 1) / kPage;
  const int n_run_pages = last_page - first_page + 1;
  const int bb = T.block_bytes;
  for (int job = blockIdx.x; job < n_run_pages * n_kv; job += gridDim.x) {
    const int lp = first_page + job / n_kv, h = job % n_kv;
    const int phys = block_table[lp];
    const bool bad = phys < 0 || phys >= n_pages;
    if (bad) {
      if (threadIdx.x == 0) set_error(T.err, TQ_DEV_BAD_SLOT);
      continue;     // uniform across the CTA
    }
    uint8_t* gblk = cache + (static_cast<int64_t>(phys) * n_kv + h) * bb;
    const int t0 = max(start_pos, lp * kPage), t1 = min(start_pos + n_tokens, (lp + 1) * kPage);
    const bool full = (t0 == lp * kPage) && (t1 == (lp + 1) * kPage);
    __syncthreads();
    for (int i = threadIdx.x; i < bb / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(sblk)[i] = full ? make_uint4(0, 0, 0, 0) : reinterpret_cast<const uint4*>(gblk)[i];
    __syncthreads();
    for (int pos = t0 + warp; pos < t1; pos += nwarp) {
      const int tok = pos - start_pos, tau = pos % kPage;
      float x[4];
      VecOut o;
      load_row4(k, static_cast<size_t>(tok) * n_kv + h, dtype, lane, x);
      quantize_vector(x, T.signs_k, s_tab, s_tab + 16, T.key_bits, s_sk, true, lane, o);
      store_key_token(sblk, tau, T.key_bits, o, lane);
      if (lane == 0) {
        store_norm(sblk, T.key_bits, T.value_bits, 0, tau, o.norm);
        store_norm(sblk, T.key_bits, T.value_bits, 1, tau, o.gamma);
      }
      load_row4(v, static_cast<size_t>(tok) * n_kv + h, dtype, lane, x);
      quantize_vector(x, T.signs_v, s_tab + 32, s_tab + 48, T.value_bits, nullptr, false, lane, o);
      store_value_token(sblk, tau, T.key_bits, T.value_bits, o, lane);
      if (lane == 0) store_norm(sblk, T.key_bits, T.value_bits, 2, tau, o.norm);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < bb / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(gblk)[i] = reinterpret_cast<const uint4*>(sblk)[i];
  }
}

// ========================================================= query transform
// Per (sequence, KV head, group of 4 query heads): q~ = H D_K q / sqrt(d) and
// p = S q~, each quantised per head to a 24-bit integer Q = rint(x * 2^e)
// (|Q| < 2^22) split into three int8 limbs Q = 2^16 Q2 + 2^8 Q1 + Q0. They are
// written in the register order of the m16n8k32 A operand whose rows are
//   rows 0-3: Q2 of heads 0-3, rows 4-7: Q0 of heads 0-3,
//   rows 8-11: Q1 of heads 0-3, rows 12-15: zero,
// so that every lane of quad g < 4 sees head g's top and middle limbs, and the
// quad g + 4 (lane + 16) its bottom limb.
//   qfrag[pair][hg][which (q, p)][kt 4][lane 32][reg 4]  (int32 words of 4 int8)
//   qconst[pair][hg][slot 4][4] = {a, b, sum P (int), 0}: in log2 units the logit
//   is l2 = |k| * <Q, C> * a + gamma * (2 <P, s> - sum P) * b.
constexpr int kGroupHeads = 4;

__device__ __forceinline__ int pick_exponent24(float maxabs) {
  if (!(maxabs > 0.0f)) return 0;
  int E;
  frexpf(maxabs, &E);               // maxabs < 2^E
  return 22 - E;                    // maxabs * 2^e < 2^22
}

struct Limbs { uint32_t w2, w1, w0; int sum; };

__device__ __forceinline__ Limbs split3(const float (&x)[4], int e) {
  Limbs r{0u, 0u, 0u, 0};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int Q = __float2int_rn(ldexpf(x[i], e));
    const int q0 = ((Q + 128) & 255) - 128;
    const int r1 = (Q - q0) >> 8;
    const int q1 = ((r1 + 128) & 255) - 128;
    const int q2 = (r1 - q1) >> 8;
    r.w2 |= static_cast<uint32_t>(q2 & 0xFF) << (8 * i);
    r.w1 |= static_cast<uint32_t>(q1 & 0xFF) << (8 * i);
    r.w0 |= static_cast<uint32_t>(q0 & 0xFF) << (8 * i);
    r.sum += Q;
  }
  return r;
}

__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

// grid (n_hg, n_kv, batch), 512 threads: warp w -> head slot w >> 2, sketch
// column quarter w & 3.
__global__ void __launch_bounds__(512) qtransform_kernel(Tables T, const void* q, int dtype, int n_q,
                                                         int n_kv, int group, int n_hg, float scale,
                                                         uint32_t* qfrag, float* qconst,
                                                         unsigned* counters) {
  asm volatile("griddepcontrol.launch_dependents;");
  __shared__ float s_q[kGroupHeads][128];
  __shared__ float s_p[4][kGroupHeads][128];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int hs = w >> 2, cq = w & 3;
  const int hg = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int pair = b * n_kv + hk;
  const int slot = hg * kGroupHeads + hs;
  if (hg == 0 && threadIdx.x == 0) counters[pair] = 0u;
  if (cq == 0) {
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (slot < group) load_row4(q, static_cast<size_t>(b) * n_q + hk * group + slot, dtype, lane, x);
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] *= T.signs_k[4 * lane + e];
    fwht128(x, lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) s_q[hs][4 * lane + e] = x[e] * kInvSqrtD;
  }
  __syncthreads();
  // partial p over the 32 sketch columns of this quarter: rows 4*lane .. 4*lane+3
  {
    const uint2* st = reinterpret_cast<const uint2*>(T.sketch_t);
    uint2 raw[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) raw[j] = __ldg(st + (32 * cq + j) * 32 + lane);
    float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float qc = s_q[hs][32 * cq + j];
      const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&raw[j].x));
      const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&raw[j].y));
      p[0] = fmaf(s01.x, qc, p[0]);
      p[1] = fmaf(s01.y, qc, p[1]);
      p[2] = fmaf(s23.x, qc, p[2]);
      p[3] = fmaf(s23.y, qc, p[3]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) s_p[cq][hs][4 * lane + e] = p[e];
  }
  __syncthreads();
  if (cq != 0) return;
  float x[4], p[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[e] = s_q[hs][4 * lane + e];
    p[e] = s_p[0][hs][4 * lane + e] + s_p[1][hs][4 * lane + e] + s_p[2][hs][4 * lane + e] +
           s_p[3][hs][4 * lane + e];
  }
  const int eq = pick_exponent24(warp_max(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])))));
  const int ep = pick_exponent24(warp_max(fmaxf(fmaxf(fabsf(p[0]), fabsf(p[1])), fmaxf(fabsf(p[2]), fabsf(p[3])))));
  const Limbs lq = split3(x, eq);
  const Limbs lp = split3(p, ep);
  const int psum = warp_isum(lp.sum);              // |sum| < 2^29
  // lane l holds coordinates 4l..4l+3: k-tile kt = l>>3, half sub = (l>>2)&1, t = l&3
  const int kt = lane >> 3, sub = (lane >> 2) & 1, t = lane & 3;
  uint32_t* base = qfrag + (static_cast<size_t>(pair) * n_hg + hg) * 2 * 512;
  const int fl_top = 4 * hs + t;           // quad hs: rows hs (Q2) and hs + 8 (Q1)
  const int fl_bot = 4 * (hs + 4) + t;     // quad hs + 4: rows hs + 4 (Q0) and hs + 12 (zero)
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const Limbs& L = which ? lp : lq;
    uint32_t* f = base + (which * 4 + kt) * 128;
    f[fl_top * 4 + 2 * sub + 0] = L.w2;
    f[fl_top * 4 + 2 * sub + 1] = L.w1;
    f[fl_bot * 4 + 2 * sub + 0] = L.w0;
    f[fl_bot * 4 + 2 * sub + 1] = 0u;
  }
  if (lane == 0) {
    float* qc = qconst + ((static_cast<size_t>(pair) * n_hg + hg) * kGroupHeads + hs) * 4;
    const bool real = slot < group;
    qc[0] = real ? scale * kLog2e * ldexpf(1.0f, -eq - T.k_exp) : 0.0f;
    qc[1] = real ? scale * kLog2e * kSqrtPiOver2 / kQjlRows * ldexpf(1.0f, -ep) : 0.0f;
    qc[2] = __int_as_float(real ? psum : 0);
    qc[3] = 0.0f;
  }
}

// ================================================================== decode
constexpr int kWarps = 4;        // compute warps per CTA
constexpr int kStages = 6;       // TMA stages per warp

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: gives up after ~2^31 clock cycles (about a second).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1ll << 31)) return false;
  }
  return true;
}
__device__ __forceinline__ void tma_load_1d(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- code words -> mma operands --------------------------------------------
// Key selectors: 8 selectors (one per B register of the 4 k-tiles), each four
// code nibbles with bit 3 clear (b <= 3) or raw 4-bit nibbles (b = 4).
template <int B>
__device__ __forceinline__ void key_selectors(const uint32_t* w, uint32_t (&sel)[8]) {
  if constexpr (B == 2) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t e = w[i] & 0x33333333u, o = (w[i] >> 2) & 0x33333333u;
      sel[4 * i + 0] = e;
      sel[4 * i + 1] = e >> 16;
      sel[4 * i + 2] = o;
      sel[4 * i + 3] = o >> 16;
    }
  } else if constexpr (B == 3) {
    const uint32_t a = w[0] & 0x77777777u, b = w[1] & 0x77777777u, c = w[2] & 0x77777777u;
    const uint32_t sp = ((w[0] >> 3) & 0x11111111u) | ((w[1] >> 2) & 0x22222222u) | ((w[2] >> 1) & 0x44444444u);
    sel[0] = a; sel[1] = a >> 16; sel[2] = b; sel[3] = b >> 16;
    sel[4] = c; sel[5] = c >> 16; sel[6] = sp; sel[7] = sp >> 16;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sel[2 * i] = w[i];
      sel[2 * i + 1] = w[i] >> 16;
    }
  }
}

// Byte lookup of 4 codes in a 16-entry byte table (t0..t3) from selector
// nibbles holding 4-bit codes: entries 0-7 via t0/t1, 8-15 via t2/t3, chosen
// per byte by code bit 3.
__device__ __forceinline__ uint32_t lookup16(uint32_t sel, uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3) {
  const uint32_t s7 = sel & 0x7777u;
  const uint32_t m = prmt(0x0000FF00u, 0u, (sel >> 3) & 0x1111u);
  const uint32_t lo = prmt(t0, t1, s7), hi = prmt(t2, t3, s7);
  return (hi & m) | (lo & ~m);
}

template <int B>
__device__ __forceinline__ void key_limbs(uint32_t sel, const uint32_t (&th)[4], const uint32_t (&tl)[4],
                                          uint32_t& hi, uint32_t& lo) {
  if constexpr (B == 4) {
    hi = lookup16(sel, th[0], th[1], th[2], th[3]);
    lo = lookup16(sel, tl[0], tl[1], tl[2], tl[3]);
  } else {
    hi = prmt(th[0], th[1], sel);
    lo = prmt(tl[0], tl[1], sel);
  }
}

// Value selectors: 16 selectors s = 2*mt + tg; nibble n = 2*hf + e.
template <int B>
__device__ __forceinline__ void value_selectors(const uint32_t* w, uint32_t (&sel)[16]) {
  if constexpr (B == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t e = w[i] & 0x33333333u, o = (w[i] >> 2) & 0x33333333u;
      sel[4 * i + 0] = e;
      sel[4 * i + 1] = e >> 16;
      sel[4 * i + 2] = o;
      sel[4 * i + 3] = o >> 16;
    }
  } else if constexpr (B == 3) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const uint32_t* x = w + 3 * g;
      const uint32_t a = x[0] & 0x77777777u, b = x[1] & 0x77777777u, c = x[2] & 0x77777777u;
      const uint32_t sp = ((x[0] >> 3) & 0x11111111u) | ((x[1] >> 2) & 0x22222222u) | ((x[2] >> 1) & 0x44444444u);
      uint32_t* s = sel + 8 * g;
      s[0] = a; s[1] = a >> 16; s[2] = b; s[3] = b >> 16;
      s[4] = c; s[5] = c >> 16; s[6] = sp; s[7] = sp >> 16;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sel[2 * i] = w[i];
      sel[2 * i + 1] = w[i] >> 16;
    }
  }
}

// Four fp16 centroids of one selector as two A registers: r0 = nibbles 0,1
// (hf = 0, tokens e = 0,1), r1 = nibbles 2,3 (hf = 1).
template <int B>
__device__ __forceinline__ void value_regs(uint32_t sel, const uint32_t (&vl)[4], const uint32_t (&vh)[4],
                                           uint32_t& r0, uint32_t& r1) {
  uint32_t lo, hi;
  if constexpr (B == 4) {
    lo = lookup16(sel, vl[0], vl[1], vl[2], vl[3]);
    hi = lookup16(sel, vh[0], vh[1], vh[2], vh[3]);
  } else {
    lo = prmt(vl[0], vl[1], sel);
    hi = prmt(vh[0], vh[1], sel);
  }
  r0 = prmt(lo, hi, 0x5140u);
  r1 = prmt(lo, hi, 0x7362u);
}

struct DecodeArgs {
  const uint8_t* cache;
  int64_t n_pages;
  const int32_t* block_tables;
  int max_pages_per_seq;
  const int32_t* seq_lens;
  int max_seq_len;
  const uint32_t* qfrag;
  const float* qconst;
  float* partial;      // [pair][chunk][hg][4 heads][132]
  unsigned* counters;  // [pair]
  float* out;          // [batch][n_q][128]
  int n_kv, n_q, group, n_hg, chunks, ppc;
};

// Split-K decode attention. grid (chunks, n_kv, batch), kWarps warps per CTA.
// Each warp streams its pages (every kWarps-th page of the chunk) through a
// private ring of kStages shared-memory stages filled by 1-D bulk TMA copies.
template <int BK, int BV, int NH>
__global__ void __launch_bounds__(kWarps * 32) decode_kernel(Tables T, DecodeArgs A) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kBlock = 256 * (BK + BV + 1) + 96;
  constexpr int kSignOff = 256 * BK, kVOff = 256 * (BK + 1), kNormOff = 256 * (BK + BV + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const bool owner = g < kGroupHeads;          // quads 0-3 own heads 0-3 of each group
  const int chunk = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int pair = b * A.n_kv + hk;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kBlock);
  uint32_t* s_qf = reinterpret_cast<uint32_t*>(bars + kWarps * kStages);   // [NH][2][4][128] query fragments
  __shared__ int s_last;
  uint8_t* stage0 = smem + warp * kStages * kBlock;
  uint64_t* mybar = bars + warp * kStages;

  int L = A.seq_lens[b];
  if (L < 0 || L > A.max_seq_len) {
    if (threadIdx.x == 0) set_error(T.err, TQ_DEV_BAD_LENGTH);
    L = L < 0 ? 0 : A.max_seq_len;
  }
  const int seq_pages = (L + kPage - 1) / kPage;
  const int p0 = chunk * A.ppc;
  const int p1 = min(p0 + A.ppc, seq_pages);
  const int nmine = (p1 > p0 + warp) ? (p1 - p0 - warp + kWarps - 1) / kWarps : 0;
  const int32_t* btab = A.block_tables + static_cast<int64_t>(b) * A.max_pages_per_seq;

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(mybar + s, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();

  auto issue = [&](int kth) {
    const int lp = p0 + warp + kth * kWarps;
    int phys = btab[lp];
    const int s = kth % kStages;
    if (phys < 0 || phys >= A.n_pages) {
      set_error(T.err, TQ_DEV_BAD_PAGE);
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mybar + s)) : "memory");
    } else {
      mbar_expect_tx(mybar + s, kBlock);
      tma_load_1d(stage0 + s * kBlock, A.cache + (static_cast<int64_t>(phys) * A.n_kv + hk) * kBlock, kBlock,
                  mybar + s);
    }
  };
  if (lane == 0)
    for (int k = 0; k < min(nmine, kStages); ++k) issue(k);

  // The query fragments come from the preceding kernel.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  {
    const uint4* src = reinterpret_cast<const uint4*>(A.qfrag + static_cast<size_t>(pair) * A.n_hg * 1024);
    for (int i = threadIdx.x; i < NH * 1024 / 4; i += blockDim.x) reinterpret_cast<uint4*>(s_qf)[i] = src[i];
  }
  float ca[NH], cb[NH];
  int csum[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float4 c4 = *reinterpret_cast<const float4*>(
        A.qconst + ((static_cast<size_t>(pair) * A.n_hg + h) * kGroupHeads + (g & 3)) * 4);
    ca[h] = c4.x; cb[h] = c4.y; csum[h] = __float_as_int(c4.z);
  }
  __syncthreads();
  uint32_t kth_[4], ktl_[4], vlo_[4], vhi_[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    kth_[i] = T.kq_hi[i]; ktl_[i] = T.kq_lo[i]; vlo_[i] = T.v_lo[i]; vhi_[i] = T.v_hi[i];
  }

  float acc[NH][8][4];
#pragma unroll
  for (int h = 0; h < NH; ++h)
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[h][mt][c] = 0.0f;
  float m2[NH], lsum[NH], mp2[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) { m2[h] = kNegBig; lsum[h] = 0.0f; mp2[h] = kNegBig; }

  bool alive = true;
  for (int k = 0; k < nmine; ++k) {
    const int s = k % kStages;
    const unsigned parity = (k / kStages) & 1;
    if (!mbar_wait(mybar + s, parity)) {
      if (lane == 0) set_error(T.err, TQ_DEV_TIMEOUT);
      alive = false;
      break;
    }
    const int lp = p0 + warp + k * kWarps;
    const int phys = btab[lp];
    const bool page_ok = phys >= 0 && phys < A.n_pages;
    const uint8_t* blk = stage0 + s * kBlock;

    // ---- this lane's operands from the staged block
    uint32_t kw[2][BK];
#pragma unroll
    for (int th = 0; th < 2; ++th)
#pragma unroll
      for (int i = 0; i < BK; ++i) kw[th][i] = reinterpret_cast<const uint32_t*>(blk)[lane * 2 * BK + th * BK + i];
    const uint2 sw = reinterpret_cast<const uint2*>(blk + kSignOff)[lane];
    uint32_t vw[2 * BV];
#pragma unroll
    for (int i = 0; i < 2 * BV; ++i) vw[i] = reinterpret_cast<const uint32_t*>(blk + kVOff)[lane * 2 * BV + i];
    const uint32_t* nrm = reinterpret_cast<const uint32_t*>(blk + kNormOff);
    float nK[4], gam[4], nV[4];
    {
      const uint32_t r[6] = {nrm[t], nrm[4 + t], nrm[8 + t], nrm[12 + t], nrm[16 + t], nrm[20 + t]};
      float2 f[6];
#pragma unroll
      for (int i = 0; i < 6; ++i) f[i] = __half22float2(*reinterpret_cast<const __half2*>(&r[i]));
      nK[0] = f[0].x; nK[1] = f[0].y; nK[2] = f[1].x; nK[3] = f[1].y;
      gam[0] = f[2].x; gam[1] = f[2].y; gam[2] = f[3].x; gam[3] = f[3].y;
      nV[0] = f[4].x; nV[1] = f[4].y; nV[2] = f[5].x; nV[3] = f[5].y;
    }

    // ---- logits: int8 tensor-core products of query limbs with code limbs
    int dh[NH][2][4], dl[NH][2][4], ds[NH][2][4];
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) dh[h][nt][c] = dl[h][nt][c] = ds[h][nt][c] = 0;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      uint32_t sel[8];
      key_selectors<BK>(kw[nt], sel);
      const uint32_t swn = nt ? sw.y : sw.x;
#pragma unroll
      for (int kt = 0; kt < 4; ++kt) {
        uint32_t h0, l0, h1, l1;
        key_limbs<BK>(sel[2 * kt], kth_, ktl_, h0, l0);
        key_limbs<BK>(sel[2 * kt + 1], kth_, ktl_, h1, l1);
        const uint32_t s0 = (swn >> (2 * kt)) & 0x01010101u, s1 = (swn >> (2 * kt + 1)) & 0x01010101u;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const uint4 fq = reinterpret_cast<const uint4*>(s_qf)[((h * 2 + 0) * 4 + kt) * 32 + lane];
          const uint4 fp = reinterpret_cast<const uint4*>(s_qf)[((h * 2 + 1) * 4 + kt) * 32 + lane];
          const uint32_t aq[4] = {fq.x, fq.y, fq.z, fq.w};
          const uint32_t ap[4] = {fp.x, fp.y, fp.z, fp.w};
          mma_s8(dh[h][nt], aq, h0, h1);
          mma_s8(dl[h][nt], aq, l0, l1);
          mma_s8(ds[h][nt], ap, s0, s1);
        }
      }
    }

    // ---- softmax statistics and split fp16 weights per head group
    const int tok_base = lp * kPage;
    uint32_t pb[NH][2];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float l2[4], lp2[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int idx = 2 * nt + i;
          // bottom-limb partial sums live in quad g + 4 (lane + 16)
          const float x0 = fmaf(256.0f, static_cast<float>(dh[h][nt][i]), static_cast<float>(dl[h][nt][i]));
          const float x0r = __shfl_xor_sync(kFull, x0, 16);
          const int s0r = __shfl_xor_sync(kFull, ds[h][nt][i], 16);
          const int tok = tok_base + 8 * nt + 2 * t + i;
          const float main = fmaf(16777216.0f, static_cast<float>(dh[h][nt][i]),
                                  fmaf(65536.0f, static_cast<float>(dl[h][nt][i] + dh[h][nt][2 + i]),
                                       fmaf(256.0f, static_cast<float>(dl[h][nt][2 + i]), x0r)));
          const int sj = 65536 * ds[h][nt][i] + 256 * ds[h][nt][2 + i] + s0r;
          const float qj = static_cast<float>(2 * sj - csum[h]);
          const float v = fmaf(nK[idx] * main, ca[h], gam[idx] * qj * cb[h]);
          const bool ok = owner && page_ok && tok < L;
          l2[idx] = ok ? v : -INFINITY;
          lp2[idx] = ok ? v + __log2f(nV[idx]) : -INFINITY;
        }
      float pm = fmaxf(fmaxf(l2[0], l2[1]), fmaxf(l2[2], l2[3]));
      float pmp = fmaxf(fmaxf(lp2[0], lp2[1]), fmaxf(lp2[2], lp2[3]));
      pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 1));
      pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 2));
      pmp = fmaxf(pmp, __shfl_xor_sync(kFull, pmp, 1));
      pmp = fmaxf(pmp, __shfl_xor_sync(kFull, pmp, 2));
      if (pm > m2[h] + 8.0f) {
        lsum[h] *= exp2f(m2[h] - pm);
        m2[h] = pm;
      }
      lsum[h] += exp2f(l2[0] - m2[h]) + exp2f(l2[1] - m2[h]) + exp2f(l2[2] - m2[h]) + exp2f(l2[3] - m2[h]);
      const bool need = pmp > mp2[h] + 8.0f;
      const float fac = need ? exp2f(mp2[h] - pmp) : 1.0f;
      if (need) mp2[h] = pmp;
      if (__any_sync(kFull, need)) {
        // acc columns 2t, 2t+1 hold heads (2t)&3, (2t+1)&3 (columns 4-7: low parts)
        const float f0 = __shfl_sync(kFull, fac, 4 * ((2 * t) & 3));
        const float f1 = __shfl_sync(kFull, fac, 4 * ((2 * t + 1) & 3));
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[h][mt][0] *= f0; acc[h][mt][1] *= f1; acc[h][mt][2] *= f0; acc[h][mt][3] *= f1;
        }
      }
      float w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = exp2f(lp2[i] - mp2[h]);
      const __half2 hi01 = __floats2half2_rn(w[0], w[1]), hi23 = __floats2half2_rn(w[2], w[3]);
      const float2 r01 = __half22float2(hi01), r23 = __half22float2(hi23);
      const __half2 lo01 = __floats2half2_rn(w[0] - r01.x, w[1] - r01.y);
      const __half2 lo23 = __floats2half2_rn(w[2] - r23.x, w[3] - r23.y);
      const uint32_t lo01u = *reinterpret_cast<const uint32_t*>(&lo01);
      const uint32_t lo23u = *reinterpret_cast<const uint32_t*>(&lo23);
      const uint32_t plo01 = __shfl_xor_sync(kFull, lo01u, 16), plo23 = __shfl_xor_sync(kFull, lo23u, 16);
      pb[h][0] = owner ? *reinterpret_cast<const uint32_t*>(&hi01) : plo01;
      pb[h][1] = owner ? *reinterpret_cast<const uint32_t*>(&hi23) : plo23;
    }

    // ---- weighted value sum in the rotated domain: fp16 tensor-core products
    uint32_t vs[16];
    value_selectors<BV>(vw, vs);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a0, a1, a2, a3;
      value_regs<BV>(vs[2 * mt], vlo_, vhi_, a0, a1);
      value_regs<BV>(vs[2 * mt + 1], vlo_, vhi_, a2, a3);
#pragma unroll
      for (int h = 0; h < NH; ++h) mma_f16(acc[h][mt], a0, a1, a2, a3, pb[h][0], pb[h][1]);
    }

    // ---- refill this stage with the page kStages ahead (all its reads are consumed)
    __syncwarp();
    if (lane == 0 && k + kStages < nmine) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(k + kStages);
    }
  }
  if (!alive) {
    // A wait ran out: give every transfer this warp still has in flight a
    // bounded chance to land before the shared memory is reused.
    for (int k2 = 0; k2 < nmine; ++k2) mbar_wait(mybar + (k2 % kStages), (k2 / kStages) & 1);
  }
  __syncwarp();
  if (lane == 0)
    for (int s = 0; s < kStages; ++s)
      asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(mybar + s)) : "memory");

  // ---- merge the warps of this CTA (the pipeline buffers are free now)
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    lsum[h] += __shfl_xor_sync(kFull, lsum[h], 1);
    lsum[h] += __shfl_xor_sync(kFull, lsum[h], 2);
  }
  __syncthreads();
  float* s_acc = reinterpret_cast<float*>(smem);                       // [warp][NH][8 columns][128]
  float* s_st = s_acc + kWarps * NH * 8 * 128;                           // [warp][NH][4 heads][3]
#pragma unroll
  for (int h = 0; h < NH; ++h) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int coord = 16 * mt + g + 8 * (c >> 1), col = 2 * t + (c & 1);
        s_acc[((warp * NH + h) * 8 + col) * 128 + coord] = acc[h][mt][c];
      }
    if (t == 0 && owner) {
      float* st = s_st + ((warp * NH + h) * kGroupHeads + g) * 3;
      st[0] = m2[h]; st[1] = lsum[h]; st[2] = mp2[h];
    }
  }
  __syncthreads();
  float* part = A.partial + (static_cast<size_t>(pair) * A.chunks + chunk) * NH * kGroupHeads * 132;
  for (int i = threadIdx.x; i < NH * kGroupHeads * 128; i += blockDim.x) {
    const int hh = i >> 7, coord = i & 127;          // hh = group * 4 + head
    const int h = hh >> 2, h4 = hh & 3;
    float M = kNegBig, Mp = kNegBig;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      M = fmaxf(M, s_st[((w * NH + h) * kGroupHeads + h4) * 3 + 0]);
      Mp = fmaxf(Mp, s_st[((w * NH + h) * kGroupHeads + h4) * 3 + 2]);
    }
    float a = 0.0f, l = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* st = s_st + ((w * NH + h) * kGroupHeads + h4) * 3;
      const float* ac = s_acc + ((w * NH + h) * 8) * 128;
      a += (ac[h4 * 128 + coord] + ac[(h4 + 4) * 128 + coord]) * exp2f(st[2] - Mp);
      l += st[1] * exp2f(st[0] - M);
    }
    part[hh * 132 + coord] = a;
    if (coord == 0) {
      part[hh * 132 + 128] = M;
      part[hh * 132 + 129] = l;
      part[hh * 132 + 130] = Mp;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned ticket = atomicAdd(A.counters + pair, 1u);
    s_last = (ticket == static_cast<unsigned>(A.chunks - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA of this (sequence, KV head): merge chunks, de-rotate, store
  const float* pbase = A.partial + static_cast<size_t>(pair) * A.chunks * NH * kGroupHeads * 132;
  for (int slot = warp; slot < A.group; slot += kWarps) {
    float M = kNegBig, Mp = kNegBig;
    for (int c = lane; c < A.chunks; c += 32) {
      const float* st = pbase + (static_cast<size_t>(c) * NH * kGroupHeads + slot) * 132 + 128;
      M = fmaxf(M, __ldcg(st));
      Mp = fmaxf(Mp, __ldcg(st + 2));
    }
    M = warp_max(M);
    Mp = warp_max(Mp);
    float l = 0.0f;
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c = 0; c < A.chunks; ++c) {
      const float* pc = pbase + (static_cast<size_t>(c) * NH * kGroupHeads + slot) * 132;
      const float wl = exp2f(__ldcg(pc + 128) - M);
      const float wa = exp2f(__ldcg(pc + 130) - Mp);
      l = fmaf(__ldcg(pc + 129), wl, l);
      const float4 v = __ldcg(reinterpret_cast<const float4*>(pc) + lane);
      a[0] = fmaf(v.x, wa, a[0]); a[1] = fmaf(v.y, wa, a[1]);
      a[2] = fmaf(v.z, wa, a[2]); a[3] = fmaf(v.w, wa, a[3]);
    }
    const float f = l > 0.0f ? exp2f(Mp - M) / l : 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) a[e] *= f;
    fwht128(a, lane);
    float4 o;
    o.x = a[0] * T.signs_v[4 * lane + 0] * kInvSqrtD;
    o.y = a[1] * T.signs_v[4 * lane + 1] * kInvSqrtD;
    o.z = a[2] * T.signs_v[4 * lane + 2] * kInvSqrtD;
    o.w = a[3] * T.signs_v[4 * lane + 3] * kInvSqrtD;
    const int qh = hk * A.group + slot;
    reinterpret_cast<float4*>(A.out + (static_cast<size_t>(b) * A.n_q + qh) * 128)[lane] = o;
  }
  if (threadIdx.x == 0) A.counters[pair] = 0u;
}

template <int BK, int BV, int NH>
cudaError_t launch_decode_t(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s) {
  constexpr int kBlock = 256 * (BK + BV + 1) + 96;
  const size_t pipe = static_cast<size_t>(kWarps) * kStages * kBlock + kWarps * kStages * sizeof(uint64_t) +
                      static_cast<size_t>(NH) * 1024 * 4;
  const size_t merge = static_cast<size_t>(kWarps) * NH * 8 * 128 * 4 + kWarps * NH * kGroupHeads * 3 * 4;
  const size_t smem = pipe > merge ? pipe : merge;
  auto fn = decode_kernel<BK, BV, NH>;
  static size_t configured = 0;     // raise the shared-memory limit once per instantiation
  if (configured < smem) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, T, a);
}

template <int BK, int BV>
cudaError_t dispatch_nh(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s) {
  switch (a.n_hg) {
    case 1: return launch_decode_t<BK, BV, 1>(T, a, grid, s);
    case 2: return launch_decode_t<BK, BV, 2>(T, a, grid, s);
    case 3: return launch_decode_t<BK, BV, 3>(T, a, grid, s);
    default: return launch_decode_t<BK, BV, 4>(T, a, grid, s);
  }
}

template <int BK>
cudaError_t dispatch_bv(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s) {
  switch (T.value_bits) {
    case 2: return dispatch_nh<BK, 2>(T, a, grid, s);
    case 3: return dispatch_nh<BK, 3>(T, a, grid, s);
    default: return dispatch_nh<BK, 4>(T, a, grid, s);
  }
}

}  // namespace

cudaError_t launch_quantize_append(const Tables& t, const void* k, const void* v, int dtype, int n_tokens,
                                   int n_kv, const int64_t* slots, void* cache, int64_t n_pages,
                                   cudaStream_t s) {
  const int jobs = n_tokens * n_kv;
  const int warps_per_block = 8;
  int blocks = (jobs + warps_per_block - 1) / warps_per_block;
  if (blocks > 148 * 2) blocks = 148 * 2;
  const size_t smem = kHeadDim * kQjlRows * 2;
  quantize_append_kernel<<<blocks, warps_per_block * 32, smem, s>>>(t, k, v, dtype, n_tokens, n_kv, slots,
                                                                    static_cast<uint8_t*>(cache), n_pages);
  return cudaGetLastError();
}

cudaError_t launch_quantize_prefill(const Tables& t, const void* k, const void* v, int dtype, int n_tokens,
                                    int n_kv, const int32_t* block_table, int start_pos, void* cache,
                                    int64_t n_pages, cudaStream_t s) {
  const int first = start_pos / kPage, last = (start_pos + n_tokens - 1) / kPage;
  const int jobs = (last - first + 1) * n_kv;
  const int blocks = jobs < 148 * 2 ? jobs : 148 * 2;
  const size_t smem = kHeadDim * kQjlRows * 2 + t.block_bytes;
  quantize_prefill_kernel<<<blocks, 256, smem, s>>>(t, k, v, dtype, n_tokens, n_kv, block_table, start_pos,
                                                    static_cast<uint8_t*>(cache), n_pages);
  return cudaGetLastError();
}

cudaError_t launch_decode(const Tables& t, const DecodePlan& plan, const void* q, int q_dtype,
                          const void* cache, int64_t n_pages, const int32_t* block_tables,
                          int max_pages_per_seq, const int32_t* seq_lens, int max_seq_len, float scale,
                          float* out, void* workspace, cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* qfrag = reinterpret_cast<uint32_t*>(ws + plan.off_qfrag);
  float* qconst = reinterpret_cast<float*>(ws + plan.off_qconst);
  float* partial = reinterpret_cast<float*>(ws + plan.off_partial);
  unsigned* counters = reinterpret_cast<unsigned*>(ws + plan.off_counter);
  qtransform_kernel<<<dim3(plan.n_hg, plan.n_kv, plan.batch), 512, 0, s>>>(
      t, q, q_dtype, plan.n_q, plan.n_kv, plan.group, plan.n_hg, scale, qfrag, qconst, counters);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DecodeArgs a;
  a.cache = static_cast<const uint8_t*>(cache);
  a.n_pages = n_pages;
  a.block_tables = block_tables;
  a.max_pages_per_seq = max_pages_per_seq;
  a.seq_lens = seq_lens;
  a.max_seq_len = max_seq_len;
  a.qfrag = qfrag;
  a.qconst = qconst;
  a.partial = partial;
  a.counters = counters;
  a.out = out;
  a.n_kv = plan.n_kv;
  a.n_q = plan.n_q;
  a.group = plan.group;
  a.n_hg = plan.n_hg;
  a.chunks = plan.chunks;
  a.ppc = plan.pages_per_chunk;
  dim3 grid(plan.chunks, plan.n_kv, plan.batch);
  switch (t.key_bits) {
    case 2: return dispatch_bv<2>(t, a, grid, s);
    case 3: return dispatch_bv<3>(t, a, grid, s);
    default: return dispatch_bv<4>(t, a, grid, s);
  }
}

}  // namespace tq
