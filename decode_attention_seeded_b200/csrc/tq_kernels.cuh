// Device code of libtq shared by its translation units: helpers, the
// quantize and decode kernel templates and their launch templates. The
// templates are instantiated per (key bits, value bits) in tq_inst.cu, which
// the build compiles once per pair; tq_kernels.cu holds the rest.
#pragma once

#include "tq.h"
#include "tq_internal.h"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstddef>
#include <cstdint>

namespace tq {

// Tensor map of a run of 16-bit K or V rows [n_tokens][n_kv][128] for the prefill's
// tile loads: four dimensions (64 coordinates, 2 halves, n_kv heads, n_tokens),
// box 64 x 2 x 1 x 16 (one 16-token tile of one head), 128-byte swizzle, zero fill
// outside the run (tq_kernels.cu).
cudaError_t encode_kv_tensor_map(CUtensorMap* map, const void* base, int dtype, int n_tokens, int n_kv);

struct DecodeArgs {
  const void* q;                 // [batch][n_q][128]
  int q_dtype;
  float scale;
  const void* k_new;             // [batch][n_kv][128] (decode step only)
  const void* v_new;
  int kv_dtype;
  uint8_t* cache;
  int64_t n_pages;
  const int32_t* block_tables;
  int max_pages_per_seq;
  const int32_t* seq_lens;
  int max_seq_len;
  float* partial;                // [pair][chunk][hg][4 heads][132]
  unsigned* counters;            // [pair]: finished CTAs; zero between calls
  float* out;                    // [batch][n_q][128]
  int n_kv, n_q, group, n_hg, chunks, ppc, n_pairs;
  int batch;
  int balanced;                  // 0: `chunks` uniform chunks of `ppc` pages per pair; 1: equal shares of all pages
  int seg_w;                     // balanced: fixed cost of one pair, in pages
  int min_share;                 // balanced: least share, in pages (fewer shares for small work)
  int shares;                    // balanced: most shares (the SM count); the grid adds one CTA per pair
  int vs_off;                    // balanced: byte offset of the [batch + 1] prefix array in shared memory
  int sparse;                    // Sparse V on: values of positions below the threshold are skipped
  float sparse_log2;             // log2 of the Sparse V threshold (relative attention weight)
  float* logits;                 // logits-only mode: [batch][n_q][logits_stride] (natural log units)
  int64_t logits_stride;
};

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

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Logical right shift by a constant done on the multiplier (FMA) pipe instead
// of the ALU pipe: the high word of x * 2^(32-k) is x >> k.
template <int K>
__device__ __forceinline__ uint32_t shr(uint32_t x) {
  static_assert(K > 0 && K < 32, "shift");
  return __umulhi(x, 1u << (32 - K));
}

// Hardware base-2 exponential / logarithm (MUFU), subnormals flushed to zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// Section offsets of a (page, KV head) block. TurboQuant keys (b_k = 2..4): key
// codes, sign bits, value codes, norms (|k|, gamma, |v|: 3 x 16 fp16). q8_0 keys
// (b_k = 8): int8 key values (2048 B), 64 fp16 block scales (128 B), value codes,
// value norms (16 fp16).
__host__ __device__ constexpr int sec_scale(int bk) { return bk == 8 ? 2048 : 256 * bk; }
__host__ __device__ constexpr int sec_v(int bk) { return bk == 8 ? 2176 : 256 * (bk + 1); }
__host__ __device__ constexpr int sec_norm(int bk, int bv) { return sec_v(bk) + 256 * bv; }
__host__ __device__ constexpr int block_bytes_of(int bk, int bv) { return sec_norm(bk, bv) + (bk == 8 ? 32 : 96); }
__host__ __device__ constexpr int vnorm_entry0(int bk) { return bk == 8 ? 0 : 32; }   // first |v| entry

// q8_0 key of one token, 4 coordinates (4 lane .. 4 lane + 3) per lane: block
// kt = lane >> 3 has scale d = max|x| / 127 (reduced over its 8 lanes) and values
// rint(x / d). Stores the 4 int8 values as one word of lane chunk 4 (tau & 7) +
// (lane & 3) and, from the block's first lane, the fp16 scale.
__device__ __forceinline__ void store_key_q8(uint8_t* blk, int tau, const float (&x)[4], int lane) {
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 4));
  const float d = amax / 127.0f;
  uint32_t word = 0u;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int qv = d > 0.0f ? __float2int_rn(x[e] / d) : 0;
    word |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * e);
  }
  const int kt = lane >> 3, sub = (lane >> 2) & 1, t = lane & 3, g = tau & 7, th = tau >> 3;
  reinterpret_cast<uint32_t*>(blk)[(64 * (4 * g + t) + 32 * th + 8 * kt + 4 * sub) >> 2] = word;
  if ((lane & 7) == 0)
    reinterpret_cast<__half*>(blk + sec_scale(8))[8 * g + 4 * th + kt] = __float2half_rn(d);
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
  uint32_t* vw = reinterpret_cast<uint32_t*>(blk + sec_v(bk));
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

// Norm arrays keep tokens g and g + 8 in one 32-bit word: entry 2 (tau & 7) + (tau >> 3).
// which: 0 = |k|, 1 = gamma, 2 = |v| (q8_0 keys: |v| only, at entry 0).
__device__ __forceinline__ void store_norm(uint8_t* blk, int bk, int bv, int which, int tau, float v) {
  __half* nrm = reinterpret_cast<__half*>(blk + sec_norm(bk, bv));
  nrm[(bk == 8 ? 0 : 16 * which) + 2 * (tau & 7) + (tau >> 3)] = __float2half_rn(v);
}


// ---- shared-memory barriers and 1-D bulk copies ---------------------------
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
// Bounded wait: gives up after `limit` clock cycles (by default 2^31, about a second).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, long long limit = 1ll << 31) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) return false;
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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------ 5th-generation tensor cores
// Tensor memory (TMEM) is allocated per CTA in columns of 128 lanes x 32 bits; a
// TMEM address holds the lane in bits 31-16 and the column in bits 15-0. Warp w
// may only touch lanes 32 (w % 4) .. 32 (w % 4) + 31.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {   // one full warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {  // the allocating warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 16 lanes x 8 columns, 8 times along the columns: register 4j + i of lane (g, t)
// is (lane g + 8 (i >> 1), column 8j + 2t + (i & 1)) -- the m16n8 accumulator
// order of mma.sync. The store waits for its completion.
__device__ __forceinline__ void tmem_st_16x256b_x8(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n"
      "tcgen05.wait::st.sync.aligned;\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// The matching load; the registers are defined only after its completion wait.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// D (TMEM, fp32) (+)= A (TMEM, fp16, M x 16) B (shared memory, fp16, 16 x N); one thread.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tensor-core operation this thread issued is complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// Shared-memory descriptor of a K-major operand without swizzle: 8-row x 16-byte
// core matrices, K-adjacent ones `lbo` bytes apart, 8-row groups `sbo` apart.
__device__ __forceinline__ uint64_t umma_desc_noswizzle(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Tiled tensor copy of one box of this GPU's memory into this CTA's shared
// memory; the box's bytes complete the transaction count on `bar`.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// ===================================================================== prefill
// Quantize a contiguous run of one sequence, one warp per (page, KV head) tile.
//
// Lane (g, t) holds tokens g and g + 8 of the page at the 32 coordinates of its
// layout chunk, coordinate pf_coord(i, t) = 16 (i >> 2) + 4 t + (i & 3) for
// i = 0..31. Coordinate bits 0, 1, 4, 5, 6 are then bits of i and bits 2, 3 are
// bits of t, so the Walsh-Hadamard transform runs five stages in registers and
// two across the lanes of a quad. The same registers are the m16n8k16 A
// fragments of z = S u (k-step ks = coordinates 16 ks .. 16 ks + 15, tokens on
// the rows), and with S stored in a matching B-fragment order (sketch_qb) the
// accumulator of n-tile nt holds exactly the sketch rows of the lane's sign
// chunk, so codes and sign bits are packed without data exchange. Value codes
// are moved to the value chunks (coordinates x 4 tokens) through a 2 KB
// shared-memory tile per warp.
__device__ __forceinline__ int pf_coord(int i, int t) { return 16 * (i >> 2) + 4 * t + (i & 3); }

// Cell of y in a symmetric b-bit codebook: code = #{j : y > t_j} (a value on a
// threshold may land in either neighbour; such values lie inside the tolerance
// band). thr: the 2^b - 1 thresholds in ascending order; the middle one is 0, so
// a binary search over the positive half and the sign give the cell.
template <int B, typename TA>
__device__ __forceinline__ int cell_code(float y, const TA& thr) {
  constexpr int H = 1 << (B - 1);
  const float a = fabsf(y);
  int k;
  if constexpr (B == 2) {
    k = a > thr[H];
  } else if constexpr (B == 3) {
    const bool p2 = a > thr[H + 1];
    const bool p1 = a > (p2 ? thr[H + 2] : thr[H]);
    k = 2 * p2 + p1;
  } else {
    const bool p4 = a > thr[H + 3];
    const bool p2 = a > (p4 ? thr[H + 5] : thr[H + 1]);
    const bool p1 = a > (p4 ? (p2 ? thr[H + 6] : thr[H + 4]) : (p2 ? thr[H + 2] : thr[H]));
    k = 4 * p4 + 2 * p2 + p1;
  }
  return y > 0.0f ? H + k : H - 1 - k;
}

// Add code `c` of lane-local coordinate i (selector i >> 2, nibble i & 3) to the
// b words of one token half of a key lane chunk.
template <int B>
__device__ __forceinline__ void put_key_code(uint32_t (&w)[4], int i, uint32_t c) {
  const int j = i >> 2, q = i & 3;
  if constexpr (B == 2) {
    w[j >> 2] |= c << (16 * (j & 1) + 4 * q + 2 * ((j >> 1) & 1));
  } else if constexpr (B == 3) {
    if (j < 6) {
      w[j >> 1] |= c << (16 * (j & 1) + 4 * q);
    } else {
      const int bit = 4 * (4 * (j - 6) + q) + 3;
      w[0] |= (c & 1u) << bit;
      w[1] |= ((c >> 1) & 1u) << bit;
      w[2] |= ((c >> 2) & 1u) << bit;
    }
  } else {
    w[j >> 1] |= c << (16 * (j & 1) + 4 * q);
  }
}

// Add the four codes of value coordinate (mt, hf) of a lane chunk to its 2b
// words. x holds one code per byte: byte 2e + tg = token 2t + e + 8 tg.
template <int B>
__device__ __forceinline__ void put_value_codes(uint32_t (&w)[8], int mt, int hf, uint32_t x) {
  if constexpr (B == 2) {
    // selector s = 2 mt + tg -> word mt >> 1, bits 16 tg + 4 (2 hf + e) + 2 (mt & 1)
    const uint32_t y = prmt(x, 0u, 0x3120u);                 // byte e + 2 tg
    const uint32_t z = (y & 0x00030003u) | ((y >> 4) & 0x00300030u);
    w[mt >> 1] |= z << (8 * hf + 2 * (mt & 1));
  } else {
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int tg = 0; tg < 2; ++tg) {
        const uint32_t c = (x >> (8 * (2 * e + tg))) & 0xFFu;
        const int sel = 2 * mt + tg, n = 2 * hf + e;
        if constexpr (B == 4) {
          w[sel >> 1] |= (c & 0xFu) << (16 * (sel & 1) + 4 * n);
        } else {
          const int G = sel >> 3, j = sel & 7;
          if (j < 6) {
            w[3 * G + (j >> 1)] |= (c & 7u) << (16 * (j & 1) + 4 * n);
          } else {
            const int bit = 4 * (4 * (j - 6) + n) + 3;
            w[3 * G + 0] |= (c & 1u) << bit;
            w[3 * G + 1] |= ((c >> 1) & 1u) << bit;
            w[3 * G + 2] |= ((c >> 2) & 1u) << bit;
          }
        }
      }
  }
}

// The lane's 32 coordinates of tokens g, g + 8 from the staged rows (zeros where
// invalid), multiplied by the rotation signs; returns both tokens' squared
// norms over all 128 coordinates. rows: the tile's 16 staged rows of K or V,
// `pitch` bytes apart, elements of `dtype`.
__device__ __forceinline__ void pf_load(const uint8_t* rows, int pitch, int dtype, int g, int t, bool ok0,
                                        bool ok1, uint32_t dmask, float (&v)[2][32], float (&ss)[2]) {
#pragma unroll
  for (int th = 0; th < 2; ++th) {
    const bool ok = th ? ok1 : ok0;
    const uint8_t* row = rows + (g + 8 * th) * pitch;
    float acc = 0.0f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      float x[4];
      if (dtype == TQ_F32) {
        const float4 f = *reinterpret_cast<const float4*>(row + (16 * ks + 4 * t) * 4);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      } else {
        const uint2 raw = *reinterpret_cast<const uint2*>(row + (16 * ks + 4 * t) * 2);
        if (dtype == TQ_BF16) {
          x[0] = __uint_as_float(raw.x << 16); x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
          x[2] = __uint_as_float(raw.y << 16); x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
        } else {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
          x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * ks + e;
        const float xe = ok ? x[e] : 0.0f;
        acc = fmaf(xe, xe, acc);
        v[th][i] = __uint_as_float(__float_as_uint(xe) ^ (((dmask >> i) & 1u) << 31));
      }
    }
    acc += __shfl_xor_sync(kFull, acc, 1);
    acc += __shfl_xor_sync(kFull, acc, 2);
    ss[th] = acc;
  }
}

// In-place natural-order Walsh-Hadamard transform of both tokens (unnormalised).
__device__ __forceinline__ void pf_fwht(float (&v)[2][32], int lane) {
#pragma unroll
  for (int th = 0; th < 2; ++th)
#pragma unroll
    for (int bit = 0; bit < 5; ++bit)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!(i & (1 << bit))) {
          const float a = v[th][i], b = v[th][i | (1 << bit)];
          v[th][i] = a + b;
          v[th][i | (1 << bit)] = a - b;
        }
#pragma unroll
  for (int m = 1; m <= 2; m <<= 1) {
    const float sg = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
    for (int th = 0; th < 2; ++th)
#pragma unroll
      for (int i = 0; i < 32; ++i) v[th][i] = fmaf(v[th][i], sg, __shfl_xor_sync(kFull, v[th][i], m));
  }
}

// Rotation of 16-bit inputs on the tensor cores. The Walsh-Hadamard matrix
// factors over the coordinate bits, H_128 = H_8 (bits 4-6) x H_16 (bits 0-3), so
// each 16-coordinate block ks of the 16-token tile is one m16n8k16 product pair
// X_ks (D_ks H_16) with the rotation signs D_ks folded into the B operand: the
// products are +-x exactly and only the fp32 accumulation rounds. The three
// stages across blocks stay in registers.
//
// The k index kappa of the product is ordered so that the A fragment registers
// are the staged input words as they are (lane (g, t): coordinates 4t .. 4t + 3
// of its two tokens, two per word), and the columns so that the accumulators
// land in the lane layout of pf_coord: kappa -> block coordinate pf_kin(kappa),
// column n of n-tile nt -> block coordinate pf_kout(nt, n).
__host__ __device__ constexpr int pf_kin(int kappa) {
  return 4 * ((kappa & 7) >> 1) + 2 * (kappa >> 3) + (kappa & 1);
}
__host__ __device__ constexpr int pf_kout(int nt, int n) { return 4 * (n >> 1) + 2 * nt + (n & 1); }

// B fragments of all blocks of one sign vector, [ks][lane] uint4 = (b0, b1) of
// n-tile 0, then of n-tile 1; entries +-1 as bf16 (bf16 inputs) or fp16.
__device__ __forceinline__ uint4 pf_rot_frag(const float* signs, int ks, int lane, bool bf16) {
  const int g = lane >> 2, t = lane & 3;
  const uint32_t one = bf16 ? 0x3F80u : 0x3C00u;
  uint32_t w[4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      uint32_t word = 0u;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = pf_kin(2 * t + 8 * r + j), o = pf_kout(nt, g);
        const bool neg = (signs[16 * ks + c] < 0.0f) != ((__popc(c & o) & 1) != 0);
        word |= (one | (neg ? 0x8000u : 0u)) << (16 * j);
      }
      w[2 * nt + r] = word;
    }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// The lane's 32 rotated (unnormalised: H D x) coordinates of tokens g, g + 8 from
// staged 16-bit rows, and both tokens' squared norms |x|^2 = |H D x|^2 / 128.
// Rows of tokens outside the run hold stale data; their results are never stored
// (every product row depends only on its own input row).
__device__ __forceinline__ void pf_rotate16(const uint8_t* rows, int pitch, bool bf16, int g, int t,
                                            const uint4* frag, int lane, float (&v)[2][32], float (&ss)[2]) {
  const uint8_t* r0 = rows + g * pitch + 8 * t;
  const uint8_t* r1 = r0 + 8 * pitch;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint2 x0 = *reinterpret_cast<const uint2*>(r0 + 32 * ks);
    const uint2 x1 = *reinterpret_cast<const uint2*>(r1 + 32 * ks);
    const uint4 b = frag[ks * 32 + lane];
    float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
    if (bf16) {
      mma_bf16(z0, x0.x, x1.x, x0.y, x1.y, b.x, b.y);
      mma_bf16(z1, x0.x, x1.x, x0.y, x1.y, b.z, b.w);
    } else {
      mma_f16(z0, x0.x, x1.x, x0.y, x1.y, b.x, b.y);
      mma_f16(z1, x0.x, x1.x, x0.y, x1.y, b.z, b.w);
    }
    v[0][4 * ks + 0] = z0[0]; v[0][4 * ks + 1] = z0[1]; v[1][4 * ks + 0] = z0[2]; v[1][4 * ks + 1] = z0[3];
    v[0][4 * ks + 2] = z1[0]; v[0][4 * ks + 3] = z1[1]; v[1][4 * ks + 2] = z1[2]; v[1][4 * ks + 3] = z1[3];
  }
#pragma unroll
  for (int th = 0; th < 2; ++th) {
#pragma unroll
    for (int bit = 2; bit < 5; ++bit)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!(i & (1 << bit))) {
          const float a = v[th][i], b = v[th][i | (1 << bit)];
          v[th][i] = a + b;
          v[th][i | (1 << bit)] = a - b;
        }
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) acc = fmaf(v[th][i], v[th][i], acc);
    acc += __shfl_xor_sync(kFull, acc, 1);
    acc += __shfl_xor_sync(kFull, acc, 2);
    ss[th] = acc * (1.0f / 128.0f);
  }
}

constexpr float kPfInvRootD = 0.08838834764831845f;   // 1 / sqrt(128)

// Keys of one tile from the rotated coordinates vv (H D x, both tokens): norms
// |k|, codes (packed into the lane's key words kw), the residual u = y - c^ in
// the rotated unit domain with |u|^2, and u 2^10 as fp16 high and low parts in
// the m16n8k16 A-fragment order of z = S u (tokens on the rows): ah[ks][r],
// r = token half (r & 1), coordinate pair 4ks + 2 (r >> 1).
// cnk10: the key centroids times 2^10 (in shared memory, indexed by the code), so
// that u 2^10 = y 2^10 - c^ 2^10 is one fused operation with a single rounding (the
// same value as (y - c^) 2^10).
template <int BK, typename TA>
__device__ __forceinline__ void pf_key_residual(float (&vv)[2][32], const float (&ss)[2], const TA& thk,
                                                const float* cnk10, uint32_t (&kw)[2][4], float (&nk)[2],
                                                float (&uu)[2], uint32_t (&ah)[8][4], uint32_t (&al)[8][4]) {
#pragma unroll
  for (int th = 0; th < 2; ++th) {
    kw[th][0] = kw[th][1] = kw[th][2] = kw[th][3] = 0u;
    float u2 = 0.0f;
    nk[th] = sqrtf(ss[th]);
    const float inv = nk[th] > 0.0f ? kPfInvRootD / nk[th] : 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float y = vv[th][i] * inv;
      const int c = cell_code<BK>(y, thk);
      const float chat10 = cnk10[c];
      put_key_code<BK>(kw[th], i, static_cast<uint32_t>(c));
      const float u10 = fmaf(y, 1024.0f, -chat10);  // u 2^10: well inside the fp16 range
      u2 = fmaf(u10, u10, u2);
      vv[th][i] = u10;
    }
    u2 += __shfl_xor_sync(kFull, u2, 1);
    u2 += __shfl_xor_sync(kFull, u2, 2);
    uu[th] = u2 * 9.5367431640625e-07f;               // 2^-20: |u|^2
  }
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int th = r & 1, i = 4 * ks + 2 * (r >> 1);
      const float x0 = vv[th][i], x1 = vv[th][i + 1];
      const __half2 hi = __floats2half2_rn(x0, x1);
      const float2 hf = __half22float2(hi);
      ah[ks][r] = *reinterpret_cast<const uint32_t*>(&hi);
      al[ks][r] = pack_half2(x0 - hf.x, x1 - hf.y);
    }
}

// Sign bits of one 8-row block nt of z = S u, in the m16n8 accumulator order
// (z[r]: token half r >> 1, column 2t + (r & 1)), added to the lane's sign words.
__device__ __forceinline__ void pf_sign_bits(uint32_t (&sw)[2], int nt, const float (&z)[4]) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int th = r >> 1, j = 2 * nt + (r & 1);          // lane-local sketch row
    sw[th] |= (z[r] >= 0.0f ? 1u : 0u) << (8 * (j & 3) + (j >> 2));
  }
}

// Store one tile's key words, sign words and the norms |k| and gamma = |k| |u|
// (tokens g, g + 8 of the lane, where inside the run).
template <int BK, int BV>
__device__ __forceinline__ void pf_key_store(uint8_t* blk, int lane, int g, bool ok0, bool ok1,
                                             const uint32_t (&kw)[2][4], const uint32_t (&sw)[2],
                                             const float (&nk)[2], const float (&uu)[2]) {
  uint32_t* kwd = reinterpret_cast<uint32_t*>(blk) + lane * 2 * BK;
  uint32_t* swd = reinterpret_cast<uint32_t*>(blk + sec_scale(BK)) + lane * 2;
#pragma unroll
  for (int th = 0; th < 2; ++th) {
    if (!(th ? ok1 : ok0)) continue;
#pragma unroll
    for (int w = 0; w < BK; ++w) kwd[th * BK + w] = kw[th][w];
    swd[th] = sw[th];
  }
  if ((lane & 3) == 0) {
    __half* nrm = reinterpret_cast<__half*>(blk + sec_norm(BK, BV));
    const float gk0 = nk[0] * sqrtf(uu[0]), gk1 = nk[1] * sqrtf(uu[1]);
    if (ok0) { nrm[2 * g] = __float2half_rn(nk[0]); nrm[16 + 2 * g] = __float2half_rn(gk0); }
    if (ok1) { nrm[2 * g + 1] = __float2half_rn(nk[1]); nrm[16 + 2 * g + 1] = __float2half_rn(gk1); }
  }
}

// Values of one tile from the rotated coordinates: norms, codes, transposed to
// the value chunks (coordinates x 4 tokens) through the warp's 2 KB tile vt, and
// stored (merged under the token mask at the ends of a run).
template <int BK, int BV, typename TA>
__device__ __forceinline__ void pf_values(const float (&vv)[2][32], const float (&ss)[2], const TA& thv,
                                          uint8_t* vt, uint8_t* blk, int lane, int g, int t,
                                          int tau0, int tau1, bool full, bool ok0, bool ok1) {
  float nv[2];
#pragma unroll
  for (int th = 0; th < 2; ++th) nv[th] = sqrtf(ss[th]);
  {
    const float inv0 = nv[0] > 0.0f ? kPfInvRootD / nv[0] : 0.0f;
    const float inv1 = nv[1] > 0.0f ? kPfInvRootD / nv[1] : 0.0f;
    __syncwarp();                                            // the tile's previous readers are done
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int c0 = cell_code<BV>(vv[0][i] * inv0, thv);
      const int c1 = cell_code<BV>(vv[1][i] * inv1, thv);
      // tokens g, g + 8 sit at bytes 2g, 2g + 1 of the coordinate's 16-byte row
      *reinterpret_cast<uint16_t*>(vt + pf_coord(i, t) * 16 + 2 * g) = static_cast<uint16_t>(c0 | (c1 << 8));
    }
    __syncwarp();
  }
  // value chunk of this lane: coordinates g + 8 hf + 16 mt, tokens 2t + e + 8 tg
  uint32_t vw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}, vm[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  const bool tv[4] = {2 * t >= tau0 && 2 * t < tau1, 2 * t + 8 >= tau0 && 2 * t + 8 < tau1,
                      2 * t + 1 >= tau0 && 2 * t + 1 < tau1, 2 * t + 9 >= tau0 && 2 * t + 9 < tau1};
  const uint32_t maskx = (tv[0] ? 0xFFu : 0u) | (tv[1] ? 0xFF00u : 0u) | (tv[2] ? 0xFF0000u : 0u) |
                         (tv[3] ? 0xFF000000u : 0u);
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint32_t x = *reinterpret_cast<const uint32_t*>(vt + (g + 8 * hf + 16 * mt) * 16 + 4 * t);
      put_value_codes<BV>(vw, mt, hf, x & maskx);
      if (!full) put_value_codes<BV>(vm, mt, hf, maskx);
    }
  uint32_t* vwd = reinterpret_cast<uint32_t*>(blk + sec_v(BK)) + lane * 2 * BV;
#pragma unroll
  for (int w = 0; w < 2 * BV; ++w) vwd[w] = full ? vw[w] : ((vwd[w] & ~vm[w]) | vw[w]);
  if (t == 0) {
    __half* nrm = reinterpret_cast<__half*>(blk + sec_norm(BK, BV)) + vnorm_entry0(BK);
    if (ok0) nrm[2 * g] = __float2half_rn(nv[0]);
    if (ok1) nrm[2 * g + 1] = __float2half_rn(nv[1]);
  }
}

// pf_rotate16 on a tile loaded by the tensor map above: 16 tokens x 2 halves of
// 128-byte lines (line l = 2 token + half), 16-byte chunk c of line l stored at
// chunk c ^ (l % 8) (the 128-byte swizzle; the tile is 1024-byte aligned). Tokens
// g and g + 8 are 16 lines apart, so both use the same chunk permutation, and the
// eight rows a quarter-warp reads fall in distinct chunks.
__device__ __forceinline__ void pf_rotate16_sw(const uint8_t* tile, bool bf16, int g, int t, const uint4* frag,
                                               int lane, float (&v)[2][32], float (&ss)[2]) {
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int half = ks >> 2, l0 = 2 * g + half;
    const int chunk = (2 * (ks & 3) + (t >> 1)) ^ (l0 & 7);
    const uint8_t* p = tile + l0 * 128 + chunk * 16 + 8 * (t & 1);
    const uint2 x0 = *reinterpret_cast<const uint2*>(p);
    const uint2 x1 = *reinterpret_cast<const uint2*>(p + 16 * 128);
    const uint4 b = frag[ks * 32 + lane];
    float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
    if (bf16) {
      mma_bf16(z0, x0.x, x1.x, x0.y, x1.y, b.x, b.y);
      mma_bf16(z1, x0.x, x1.x, x0.y, x1.y, b.z, b.w);
    } else {
      mma_f16(z0, x0.x, x1.x, x0.y, x1.y, b.x, b.y);
      mma_f16(z1, x0.x, x1.x, x0.y, x1.y, b.z, b.w);
    }
    v[0][4 * ks + 0] = z0[0]; v[0][4 * ks + 1] = z0[1]; v[1][4 * ks + 0] = z0[2]; v[1][4 * ks + 1] = z0[3];
    v[0][4 * ks + 2] = z1[0]; v[0][4 * ks + 3] = z1[1]; v[1][4 * ks + 2] = z1[2]; v[1][4 * ks + 3] = z1[3];
  }
#pragma unroll
  for (int th = 0; th < 2; ++th) {
#pragma unroll
    for (int bit = 2; bit < 5; ++bit)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!(i & (1 << bit))) {
          const float a = v[th][i], b = v[th][i | (1 << bit)];
          v[th][i] = a + b;
          v[th][i | (1 << bit)] = a - b;
        }
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) acc = fmaf(v[th][i], v[th][i], acc);
    acc += __shfl_xor_sync(kFull, acc, 1);
    acc += __shfl_xor_sync(kFull, acc, 2);
    ss[th] = acc * (1.0f / 128.0f);
  }
}

// Shared memory of the prefill kernel, per CTA of W warps: W value-transpose
// tiles (2 KB), W x 2 half-stages (16 staged K rows, 16 staged V rows, pf_pitch
// bytes apart), the rotation B fragments of D_K and D_V (8 KB), W x 2 barriers.
// A half-stage is refilled with the next tile's rows as soon as its rows have
// been read, so copies overlap the arithmetic.
__host__ __device__ constexpr int pf_pitch(int elem) { return 128 * elem + 32; }
constexpr int kPfRotBytes = 2 * 8 * 32 * 16;
__host__ __device__ constexpr size_t pf_smem(int warps, int elem) {
  return size_t(warps) * 2048 + size_t(warps) * 32 * pf_pitch(elem) + kPfRotBytes + size_t(warps) * 2 * 8;
}

template <int BK, int BV>
__global__ void __launch_bounds__(256, 2) quantize_prefill_kernel(Tables T, const void* k, const void* v,
                                                                  int dtype, int n_tokens, int n_kv,
                                                                  const int32_t* block_table, int start_pos,
                                                                  uint8_t* cache, int64_t n_pages) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int W = blockDim.x >> 5;
  const int elem = dtype == TQ_F32 ? 4 : 2;
  const int pitch = pf_pitch(elem), rb = 128 * elem;
  const uint2* qb = reinterpret_cast<const uint2*>(T.sketch_qb);            // [8 ks][16 nt][32 lane]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* vt = smem + warp * 2048;                                          // value transpose tile
  uint8_t* stage0 = smem + W * 2048 + warp * 32 * pitch;                     // K rows, then V rows
  uint4* rot = reinterpret_cast<uint4*>(smem + W * 2048 + W * 32 * pitch);  // [kv][ks][lane]
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + W * 2048 + W * 32 * pitch + kPfRotBytes) + warp * 2;
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (elem == 2)
    for (int e = threadIdx.x; e < 2 * 8 * 32; e += blockDim.x)
      rot[e] = pf_rot_frag(e < 256 ? T.signs_k : T.signs_v, (e >> 5) & 7, e & 31, dtype == TQ_BF16);
  __syncthreads();
  uint32_t dmk = 0u, dmv = 0u;                  // rotation sign bits of the lane's coordinates
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    dmk |= (T.signs_k[pf_coord(i, t)] < 0.0f ? 1u : 0u) << i;
    dmv |= (T.signs_v[pf_coord(i, t)] < 0.0f ? 1u : 0u) << i;
  }
  float thk[16], thv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    thk[i] = T.thr_k[i];
    thv[i] = T.thr_v[i];
  }
  __shared__ float cnk10[16];                   // key centroids x 2^10, by code
  if (threadIdx.x < 16) cnk10[threadIdx.x] = T.cen_k[threadIdx.x] * 1024.0f;
  __syncthreads();
  __syncwarp();
  const int first_page = start_pos / kPage;
  const int n_tiles = ((start_pos + n_tokens - 1) / kPage - first_page + 1) * n_kv;
  const int bb = T.block_bytes;
  const int stride = gridDim.x * W;

  // Stage the 16 rows of K (kv = 0) or V (kv = 1) of `tile`: lane tau copies token
  // tau's row when the token is in the run and the tile's page id is in range.
  auto stage_rows = [&](int tile, int kv) {
    const int lp = first_page + tile / n_kv, h = tile % n_kv;
    const int phys = block_table[lp];
    const bool good = phys >= 0 && phys < n_pages;
    const int tau0 = max(start_pos - lp * kPage, 0), tau1 = min(start_pos + n_tokens - lp * kPage, kPage);
    if (lane == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");    // earlier reads of these rows
      mbar_expect_tx(bar + kv, good ? static_cast<unsigned>((tau1 - tau0) * rb) : 0u);
    }
    __syncwarp();
    if (good && lane >= tau0 && lane < tau1) {
      const int64_t row = static_cast<int64_t>(lp * kPage + lane - start_pos) * n_kv + h;
      const uint8_t* src = static_cast<const uint8_t*>(kv ? v : k) + row * rb;
      tma_load_1d(stage0 + (kv * 16 + lane) * pitch, src, rb, bar + kv);
    }
  };

  int tile = blockIdx.x * W + warp;
  if (tile < n_tiles) {
    stage_rows(tile, 0);
    stage_rows(tile, 1);
  }
  unsigned ph = 0;
  bool alive = true;
  for (; tile < n_tiles && alive; tile += stride, ph ^= 1u) {
    const int next = tile + stride;
    const int lp = first_page + tile / n_kv, h = tile % n_kv;
    const int phys = block_table[lp];
    const bool good = phys >= 0 && phys < n_pages;
    if (!good && lane == 0) set_error(T.err, TQ_DEV_BAD_SLOT);
    uint8_t* blk = cache + (static_cast<int64_t>(good ? phys : 0) * n_kv + h) * bb;
    const int tau0 = max(start_pos - lp * kPage, 0), tau1 = min(start_pos + n_tokens - lp * kPage, kPage);
    const bool full = tau0 == 0 && tau1 == kPage;
    const bool ok0 = g >= tau0 && g < tau1, ok1 = g + 8 >= tau0 && g + 8 < tau1;

#pragma unroll 1
    for (int kv = 0; kv < 2; ++kv) {               // 0: keys, 1: values (one copy of the rotation code)
    // the outcome is made warp-uniform: the code below shuffles across the warp
    if (!__all_sync(kFull, mbar_wait(bar + kv, ph))) {
      if (lane == 0) set_error(T.err, TQ_DEV_TIMEOUT);
      // bounded: let the copies still in flight land before the rows are reused
      // (kv = 0: this tile's K and V rows; kv = 1: its V rows and the next tile's K rows)
      mbar_wait(bar + kv, ph);
      if (kv == 0) mbar_wait(bar + 1, ph);
      else if (next < n_tiles) mbar_wait(bar, ph ^ 1u);
      alive = false;
      break;
    }
    float vv[2][32], ss[2];
    // 16-bit inputs are rotated on the tensor cores as they are read; fp32 inputs
    // and q8_0 keys (not rotated) are read into registers
    const bool mma_rot = elem == 2 && !(BK == 8 && kv == 0);
    if (mma_rot)
      pf_rotate16(stage0 + kv * 16 * pitch, pitch, dtype == TQ_BF16, g, t, rot + kv * 256, lane, vv, ss);
    else
      pf_load(stage0 + kv * 16 * pitch, pitch, dtype, g, t, ok0, ok1, kv ? dmv : (BK == 8 ? 0u : dmk), vv, ss);
    __syncwarp();                                  // the rows are read: refill with the next tile's
    if (next < n_tiles) stage_rows(next, kv);
    if (!good) continue;
    if (BK == 8 && kv == 0) {
    // ---------------- q8_0 keys: the lane's coordinates i = 0..31 of token half th
    // are bytes 32 th + i of its lane chunk; block kt = i >> 3 spans the quad
      uint32_t w8[2][8];
      float dsc[2][4];
#pragma unroll
      for (int th = 0; th < 2; ++th)
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
          float amax = 0.0f;
#pragma unroll
          for (int i = 8 * kt; i < 8 * kt + 8; ++i) amax = fmaxf(amax, fabsf(vv[th][i]));
          amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
          const float d = amax / 127.0f;
          dsc[th][kt] = d;
#pragma unroll
          for (int w = 2 * kt; w < 2 * kt + 2; ++w) {
            uint32_t word = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int qv = d > 0.0f ? __float2int_rn(vv[th][4 * w + e] / d) : 0;
              word |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * e);
            }
            w8[th][w] = word;
          }
        }
      uint4* kd = reinterpret_cast<uint4*>(blk + lane * 64);
      __half* sd = reinterpret_cast<__half*>(blk + sec_scale(8)) + 8 * g;
#pragma unroll
      for (int th = 0; th < 2; ++th) {
        if (!(th ? ok1 : ok0)) continue;
        kd[2 * th] = make_uint4(w8[th][0], w8[th][1], w8[th][2], w8[th][3]);
        kd[2 * th + 1] = make_uint4(w8[th][4], w8[th][5], w8[th][6], w8[th][7]);
        if (t == 0) {
          const __half2 s01 = __floats2half2_rn(dsc[th][0], dsc[th][1]);
          const __half2 s23 = __floats2half2_rn(dsc[th][2], dsc[th][3]);
          reinterpret_cast<uint2*>(sd + 4 * th)[0] =
              make_uint2(*reinterpret_cast<const uint32_t*>(&s01), *reinterpret_cast<const uint32_t*>(&s23));
        }
      }
      continue;
    }
    if (!mma_rot) pf_fwht(vv, lane);
    if (kv == 0) {
      if constexpr (BK != 8) {
        // ---------------- keys: norm, codes, residual, z = S u, signs
        float nk[2], uu[2];
        uint32_t kw[2][4], sw[2] = {0u, 0u};
        uint32_t ah[8][4], al[8][4];
        pf_key_residual<BK>(vv, ss, thk, cnk10, kw, nk, uu, ah, al);
#pragma unroll 1
        for (int nt = 0; nt < 16; nt += 2) {             // two independent accumulator chains
          float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint2 b0 = __ldg(qb + (ks * 16 + nt) * 32 + lane), b1 = __ldg(qb + (ks * 16 + nt + 1) * 32 + lane);
            mma_f16(z0, ah[ks][0], ah[ks][1], ah[ks][2], ah[ks][3], b0.x, b0.y);
            mma_f16(z1, ah[ks][0], ah[ks][1], ah[ks][2], ah[ks][3], b1.x, b1.y);
            mma_f16(z0, al[ks][0], al[ks][1], al[ks][2], al[ks][3], b0.x, b0.y);
            mma_f16(z1, al[ks][0], al[ks][1], al[ks][2], al[ks][3], b1.x, b1.y);
          }
          pf_sign_bits(sw, nt, z0);
          pf_sign_bits(sw, nt + 1, z1);
        }
        pf_key_store<BK, BV>(blk, lane, g, ok0, ok1, kw, sw, nk, uu);
      }
    } else {
      pf_values<BK, BV>(vv, ss, thv, vt, blk, lane, g, t, tau0, tau1, full, ok0, ok1);
    }
    }
  }
  __syncwarp();
  if (lane == 0) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar + 1)) : "memory");
  }
}

// ------------------------------------------------------------------------
// Prefill with z = S u on the 5th-generation tensor cores (16-bit K/V inputs,
// TurboQuant keys). One CTA of 16 warps per SM; each half of the CTA (8 warps)
// quantizes 8 tiles at a time, one per warp, and forms the sketch product of
// their 128 tokens in one 128 x 128 x 128 tensor-core pass:
//   - each warp writes its 16 residual rows (u 2^10 as fp16 high and low parts)
//     to its lanes of the group's A tiles in tensor memory and arrives on the
//     group's barrier;
//   - one thread issues 2 x 8 MMAs (K = 16 each; high parts, then low parts into
//     the same fp32 accumulators) with S in shared memory as the B operand, and
//     commits them to the group's product barrier;
//   - meanwhile the warps quantize their tiles' values; then each reads its 16
//     rows of z back and packs the sign bits.
// Tensor-memory rows: warp w owns lanes 32 (w % 4) + 16 ((w / 4) % 2) + 0..15.
// Columns of group c: A high parts 256c + 0..63, low parts + 64..127 (two fp16
// coordinates per column, natural order), accumulators + 128..255 (column n =
// the B operand's row n, arranged so that column block nt holds the sketch rows
// of the mma.sync n-tile nt, whose sign-packing order is kept).
// S (fp16, 32 KB) is one bulk copy of Tables::sketch_umma: row n = 8 nt + c,
// coordinate k at byte 2048 (n >> 3) + 128 (k >> 3) + 16 (n & 7) + 2 (k & 7).
// Each warp's K and V tiles come in by one tensor copy each (encode_kv_tensor_map),
// into 4 KB 128-byte-swizzled buffers read by pf_rotate16_sw; the next round's
// tiles are requested as soon as a tile has been read.
constexpr int kTcWarps = 16;
constexpr int kTcTileBytes = 16 * 256;                      // one 16-token tile of K or V rows
constexpr size_t kTcOffS = size_t(kTcWarps) * 2 * kTcTileBytes;   // after the (1024-aligned) stages
constexpr size_t kTcOffRot = kTcOffS + 32768;
constexpr size_t kTcOffVt = kTcOffRot + kPfRotBytes;
constexpr size_t kTcOffBar = kTcOffVt + kTcWarps * 2048;
constexpr int kTcBars = 2 * kTcWarps + 1 + 2 + 2;          // staging, S copy, A ready x 2, z ready x 2
constexpr size_t kTcSmem = 1024 + kTcOffBar + kTcBars * 8 + 16;   // + alignment of the stages
constexpr uint32_t kTcCols = 512;

template <int BK, int BV>
__global__ void __launch_bounds__(kTcWarps * 32, 1) quantize_prefill_tc_kernel(
    Tables T, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv, int dtype,
    int n_tokens, int n_kv, const int32_t* block_table, int start_pos, uint8_t* cache, int64_t n_pages) {
  static_assert(BK >= 2 && BK <= 4, "TurboQuant keys only");
  extern __shared__ __align__(128) uint8_t smem_raw[];
  constexpr int W = kTcWarps;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int grp = warp >> 3, wg = warp & 7;
  // the swizzled tiles need 1024-byte alignment
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stage0 = smem + warp * 2 * kTcTileBytes;              // K tile, then V tile
  uint8_t* sk = smem + kTcOffS;                                  // S, tensor-core B layout
  uint4* rot = reinterpret_cast<uint4*>(smem + kTcOffRot);       // rotation B fragments [kv][ks][lane]
  uint8_t* vt = smem + kTcOffVt + warp * 2048;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTcOffBar);
  uint64_t* bar = bars + 2 * warp;                               // this warp's K and V rows landed
  uint64_t* bar_sk = bars + 2 * W;                               // S landed
  uint64_t* bar_a = bars + 2 * W + 1 + grp;                      // the group's A rows are written
  uint64_t* bar_z = bars + 2 * W + 3 + grp;                      // the group's products are complete
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + kTcBars);
  __shared__ int s_abort;

  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
  }
  if (threadIdx.x == 0) {
    mbar_init(bar_sk, 1);
    for (int c = 0; c < 2; ++c) {
      mbar_init(bars + 2 * W + 1 + c, 8);
      mbar_init(bars + 2 * W + 3 + c, 1);
    }
    s_abort = 0;
  }
  if (lane == 0) asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  for (int e = threadIdx.x; e < 2 * 8 * 32; e += blockDim.x)
    rot[e] = pf_rot_frag(e < 256 ? T.signs_k : T.signs_v, (e >> 5) & 7, e & 31, dtype == TQ_BF16);
  if (warp == 0) tmem_alloc(s_tmem, kTcCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *s_tmem;
  if (threadIdx.x == 0) {
    mbar_expect_tx(bar_sk, 32768u);
    tma_load_1d(sk, T.sketch_umma, 32768u, bar_sk);
  }
  float thk[16], thv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    thk[i] = T.thr_k[i];
    thv[i] = T.thr_v[i];
  }
  __shared__ float cnk10[16];                   // key centroids x 2^10, by code
  if (threadIdx.x < 16) cnk10[threadIdx.x] = T.cen_k[threadIdx.x] * 1024.0f;
  __syncthreads();
  const bool bf16 = dtype == TQ_BF16;
  const int first_page = start_pos / kPage;
  const int n_tiles = ((start_pos + n_tokens - 1) / kPage - first_page + 1) * n_kv;
  const int bb = T.block_bytes;
  const int gstride = gridDim.x * 2 * 8;                       // tiles per round over the grid

  // Stage the K (kv = 0) or V (kv = 1) tile of `tile`: one tensor copy of the
  // page's 16 tokens of head h (tokens outside the run read as zeros).
  auto stage_rows = [&](int tile, int kv) {
    if (lane == 0) {
      const int lp = first_page + tile / n_kv, h = tile % n_kv;
      const int phys = block_table[lp];
      const bool good = phys >= 0 && phys < n_pages;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");    // earlier reads of this tile
      mbar_expect_tx(bar + kv, good ? static_cast<unsigned>(kTcTileBytes) : 0u);
      if (good) tma_load_4d(stage0 + kv * kTcTileBytes, kv ? &tmv : &tmk, 0, 0, h, lp * kPage - start_pos, bar + kv);
    }
    __syncwarp();
  };

  const uint32_t lanes = static_cast<uint32_t>(32 * (warp & 3) + 16 * ((warp >> 2) & 1)) << 16;
  const uint32_t col0 = 256u * grp;
  // f32 accumulators, f16 A and B, both K-major, N = 128 (bits 17-22: N / 8), M = 128 (bits 24-28: M / 16)
  constexpr uint32_t kIdesc = (1u << 4) | (16u << 17) | (8u << 24);
  const uint32_t sk_addr = smem_u32(sk);

  int tile = (blockIdx.x * 2 + grp) * 8 + wg;
  if (tile < n_tiles) {
    stage_rows(tile, 0);
    stage_rows(tile, 1);
  }
  // staging barriers: phase of the next wait, and whether a copy is in flight
  unsigned kph = 0, vph = 0;
  bool kpend = tile < n_tiles, vpend = tile < n_tiles;
  bool dead = false;               // a staging wait ran out: no more copies, no more work
  auto aborted = [&]() { return __any_sync(kFull, *reinterpret_cast<volatile int*>(&s_abort) != 0); };
  for (int r = 0;; ++r, tile += gstride) {
    if (tile - wg >= n_tiles) break;                              // the group is done (group-uniform)
    if (aborted()) break;
    const int next = tile + gstride;
    bool work = tile < n_tiles && !dead;
    int lp = 0, h = 0, tau0 = 0, tau1 = 0;
    bool good = false;
    if (work) {
      lp = first_page + tile / n_kv;
      h = tile % n_kv;
      const int phys = block_table[lp];
      good = phys >= 0 && phys < n_pages;
      if (!good && lane == 0) set_error(T.err, TQ_DEV_BAD_SLOT);
      tau0 = max(start_pos - lp * kPage, 0);
      tau1 = min(start_pos + n_tokens - lp * kPage, kPage);
    }
    uint8_t* blk = cache + (static_cast<int64_t>(good ? block_table[lp] : 0) * n_kv + h) * bb;
    const bool full = tau0 == 0 && tau1 == kPage;
    const bool ok0 = g >= tau0 && g < tau1, ok1 = g + 8 >= tau0 && g + 8 < tau1;

    // ---- keys: rotation, codes, residual rows into tensor memory
    float nk[2] = {0.f, 0.f}, uu[2] = {0.f, 0.f};
    uint32_t kw[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
    if (work && !__all_sync(kFull, mbar_wait(bar, kph))) {
      if (lane == 0) set_error(T.err, TQ_DEV_TIMEOUT);
      dead = true;
      work = false;
    }
    if (work) {
      kpend = false;
      kph ^= 1u;
      float vv[2][32], ss[2];
      pf_rotate16_sw(stage0, bf16, g, t, rot, lane, vv, ss);
      __syncwarp();                                               // the K rows are read
      if (next < n_tiles) {
        stage_rows(next, 0);
        kpend = true;
      }
      uint32_t ah[8][4], al[8][4];
      pf_key_residual<BK>(vv, ss, thk, cnk10, kw, nk, uu, ah, al);
      uint32_t ra[32];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        ra[4 * ks + 0] = ah[ks][0]; ra[4 * ks + 1] = ah[ks][2]; ra[4 * ks + 2] = ah[ks][1]; ra[4 * ks + 3] = ah[ks][3];
      }
      tmem_st_16x256b_x8(tmem + lanes + col0, ra);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        ra[4 * ks + 0] = al[ks][0]; ra[4 * ks + 1] = al[ks][2]; ra[4 * ks + 2] = al[ks][1]; ra[4 * ks + 3] = al[ks][3];
      }
      tmem_st_16x256b_x8(tmem + lanes + col0 + 64, ra);
    }
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_a);

    // ---- one thread of the group: z = S u for the group's 128 rows
    if (wg == 0 && lane == 0) {
      const bool ready = (r > 0 || mbar_wait(bar_sk, 0)) && mbar_wait(bar_a, r & 1);
      if (ready) {
        tc_fence_after_sync();
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            umma_f16_ts(tmem + col0 + 128, tmem + col0 + 64 * hl + 8 * ks,
                        umma_desc_noswizzle(sk_addr + 256 * ks, 128, 2048), kIdesc, (hl | ks) ? 1u : 0u);
        umma_commit(bar_z);
      } else {
        set_error(T.err, TQ_DEV_TIMEOUT);
        s_abort = 1;
        mbar_arrive(bar_z);                                       // release the group; nothing is read
      }
    }

    // ---- values, while the product runs
    if (work && !__all_sync(kFull, mbar_wait(bar + 1, vph))) {
      if (lane == 0) set_error(T.err, TQ_DEV_TIMEOUT);
      dead = true;
      work = false;
    }
    if (work) {
      vpend = false;
      vph ^= 1u;
      float vv[2][32], ss[2];
      pf_rotate16_sw(stage0 + kTcTileBytes, bf16, g, t, rot + 256, lane, vv, ss);
      __syncwarp();                                               // the V rows are read
      if (next < n_tiles) {
        stage_rows(next, 1);
        vpend = true;
      }
      if (good) pf_values<BK, BV>(vv, ss, thv, vt, blk, lane, g, t, tau0, tau1, full, ok0, ok1);
    }

    // ---- this warp's rows of z: sign bits, then the key words
    if (!__all_sync(kFull, mbar_wait(bar_z, r & 1))) {
      if (lane == 0) {
        set_error(T.err, TQ_DEV_TIMEOUT);
        s_abort = 1;
      }
      break;
    }
    tc_fence_after_sync();
    if (aborted()) break;
    if (work && good) {
      uint32_t sw[2] = {0u, 0u};
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t zr[32];
        tmem_ld_16x256b_x8(tmem + lanes + col0 + 128 + 64 * hf, zr);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float z[4] = {__uint_as_float(zr[4 * j]), __uint_as_float(zr[4 * j + 1]),
                              __uint_as_float(zr[4 * j + 2]), __uint_as_float(zr[4 * j + 3])};
          pf_sign_bits(sw, 8 * hf + j, z);
        }
      }
      pf_key_store<BK, BV>(blk, lane, g, ok0, ok1, kw, sw, nk, uu);
    }
    tc_fence_before_sync();
  }
  // bounded: let this warp's copies still in flight (after a wait ran out or an
  // abort) land before the CTA exits
  if (kpend) mbar_wait(bar, kph);
  if (vpend) mbar_wait(bar + 1, vph);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTcCols);
  }
  if (lane == 0) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar + 1)) : "memory");
  }
}

// ========================================================= query transform
// Per (sequence, KV head, group of 4 query heads), computed in the prologue of
// the decode kernel: q~ = H D_K q / sqrt(d) and p = S q~, each quantised per
// head to a 24-bit integer Q = rint(x * 2^e) (|Q| < 2^22) split into three int8
// limbs Q = 2^16 Q2 + 2^8 Q1 + Q0. They form the B operand (k = coordinate or
// sketch row, n = column) of m16n8k32 products whose A operand is a 16-token
// tile of codes or sign bits:
//   n-tile 0: column 2h = Q2 of head h, column 2h + 1 = Q1 of head h,
//   n-tile 1: column 2h = Q0 of head h, column 2h + 1 = 0,
// so that lane (g, t) of the accumulator sees all three limbs of head t. With
// two or more groups (code keys), two groups share n-tile 1: column 2h + 1 then
// holds Q0 of head h of the second group (put_frag_paired), which saves one
// product in five per k-step for every second group. With 4-bit keys and two or
// more groups the key term instead runs on fp16 tensor cores: the centroids are
// fp16 values, looked up in pairs from a byte-indexed table, and q~ 2^sig is split
// into fp16 high and low parts (columns 2h, 2h + 1 of one n-tile), two m16n8k16
// products per k-tile and group; the sign term keeps its int8 limbs. In
// log2 units the logit is l2 = |k| <Q, C> a + gamma (2 <P, s> - sum P) b with
// a = scale log2(e) 2^(-e_q - k_exp), b = scale log2(e) sqrt(pi/2)/m 2^(-e_p).
constexpr int kGroupHeads = 4;

// Powers of two built from the IEEE-754 exponent field (exact).
// pow2i(n) = 2^n for -149 <= n <= 127 (n is clamped to that range).
__device__ __forceinline__ float pow2i(int n) {
  n = min(max(n, -149), 127);
  return n >= -126 ? __uint_as_float(static_cast<unsigned>(n + 127) << 23)
                   : __uint_as_float(static_cast<unsigned>(n + 127 + 64) << 23) * 5.421010862427522e-20f;  // 2^-64
}
// E with x < 2^E for finite x > 0 (the exponent frexp returns, for normal x).
__device__ __forceinline__ int exp_above(float x) {
  return static_cast<int>((__float_as_uint(x) >> 23) & 0xFFu) - 126;
}

__device__ __forceinline__ int pick_exponent24(float maxabs) {
  if (!(maxabs > 0.0f)) return 0;
  return min(22 - exp_above(maxabs), 127);   // maxabs * 2^e < 2^22
}

struct Limbs { uint32_t w2, w1, w0; int sum; };

__device__ __forceinline__ Limbs split3(const float (&x)[4], int e) {
  Limbs r{0u, 0u, 0u, 0};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int Q = __float2int_rn(x[i] * pow2i(e));
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

// ================================================================== decode
// Warps per decode CTA, one CTA per SM. Uniform split: 16 for one group of 4
// query heads (the kernel then fits 128 registers), 12 for two or three groups
// (168 registers; with three groups a few hundred bytes spill, and the extra
// warps still hide more latency than the spills cost). The balanced split,
// whose loop over segments needs more registers: 12 for one or three groups, 8
// for two (12 were slower there).
template <int NH, bool BAL = false>
struct DecodeWarps {
  static constexpr int value = BAL ? (NH == 2 ? 8 : 12) : NH == 1 ? 16 : 12;
};
// TMA stages per warp: six when they fit in 160 KB of shared memory, else four.
constexpr int kAccPitch = 132;      // floats per accumulator column in the CTA merge

__host__ __device__ constexpr int decode_stages(int warps, int block) {
  return warps * 6 * block <= 160 * 1024 ? 6 : warps * 4 * block <= 160 * 1024 ? 4 : 3;
}


// ---- code words -> mma operands --------------------------------------------
// Key selectors: 8 selectors (one per B register of the 4 k-tiles), each four
// code nibbles with bit 3 clear (b <= 3) or raw 4-bit nibbles (b = 4).
template <int B>
__device__ __forceinline__ void key_selectors(const uint32_t* w, uint32_t (&sel)[8]) {
  if constexpr (B == 2) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t e = w[i] & 0x33333333u, o = shr<2>(w[i]) & 0x33333333u;
      sel[4 * i + 0] = e;
      sel[4 * i + 1] = shr<16>(e);
      sel[4 * i + 2] = o;
      sel[4 * i + 3] = shr<16>(o);
    }
  } else if constexpr (B == 3) {
    const uint32_t a = w[0] & 0x77777777u, b = w[1] & 0x77777777u, c = w[2] & 0x77777777u;
    const uint32_t sp = (shr<3>(w[0]) & 0x11111111u) | (shr<2>(w[1]) & 0x22222222u) | (shr<1>(w[2]) & 0x44444444u);
    sel[0] = a; sel[1] = shr<16>(a); sel[2] = b; sel[3] = shr<16>(b);
    sel[4] = c; sel[5] = shr<16>(c); sel[6] = sp; sel[7] = shr<16>(sp);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sel[2 * i] = w[i];
      sel[2 * i + 1] = shr<16>(w[i]);
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

// Value selectors (2- and 3-bit values; 4-bit values use a byte-indexed table):
// 16 selectors s = 2*mt + tg; nibble n = 2*hf + e.
template <int B>
__device__ __forceinline__ void value_selectors(const uint32_t* w, uint32_t (&sel)[16]) {
  static_assert(B == 2 || B == 3, "value selectors: 2 or 3 bits");
  if constexpr (B == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t e = w[i] & 0x33333333u, o = shr<2>(w[i]) & 0x33333333u;
      sel[4 * i + 0] = e;
      sel[4 * i + 1] = shr<16>(e);
      sel[4 * i + 2] = o;
      sel[4 * i + 3] = shr<16>(o);
    }
  } else if constexpr (B == 3) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const uint32_t* x = w + 3 * g;
      const uint32_t a = x[0] & 0x77777777u, b = x[1] & 0x77777777u, c = x[2] & 0x77777777u;
      const uint32_t sp = (shr<3>(x[0]) & 0x11111111u) | (shr<2>(x[1]) & 0x22222222u) | (shr<1>(x[2]) & 0x44444444u);
      uint32_t* s = sel + 8 * g;
      s[0] = a; s[1] = shr<16>(a); s[2] = b; s[3] = shr<16>(b);
      s[4] = c; s[5] = shr<16>(c); s[6] = sp; s[7] = shr<16>(sp);
    }
  }
}

// Four fp16 centroids of one selector as two A registers: r0 = nibbles 0,1
// (hf = 0, tokens e = 0,1), r1 = nibbles 2,3 (hf = 1).
template <int B>
__device__ __forceinline__ void value_regs(uint32_t sel, const uint32_t (&vl)[4], const uint32_t (&vh)[4],
                                           uint32_t& r0, uint32_t& r1) {
  const uint32_t lo = prmt(vl[0], vl[1], sel), hi = prmt(vh[0], vh[1], sel);
  r0 = prmt(lo, hi, 0x5140u);
  r1 = prmt(lo, hi, 0x7362u);
}

// Load N 32-bit words from 8-byte-aligned shared memory with the widest accesses.
template <int N>
__device__ __forceinline__ void lds_words(const uint32_t* src, uint32_t (&dst)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(src)[i];
      dst[4 * i] = v.x; dst[4 * i + 1] = v.y; dst[4 * i + 2] = v.z; dst[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const uint2 v = reinterpret_cast<const uint2*>(src)[i];
      dst[2 * i] = v.x; dst[2 * i + 1] = v.y;
    }
  }
}

// (DecodeArgs is declared above the anonymous namespace.)

// Shared-memory scratch of the prologue (after the stages and barriers).
// Every member starts on a 16-byte boundary (vector loads read qt and u).
constexpr int kQrawPitch = 136;     // floats per raw query row: the sketch's B loads avoid bank conflicts

template <int NH>
struct alignas(16) Prologue {
  alignas(16) float qraw[NH * kGroupHeads][kQrawPitch];   // queries as given (fp32)
  alignas(16) uint4 qb[NH][2][4][32];              // B fragments [group][q~ / p][k-tile][lane] (see put_frag;
                                                   // with fp16 key products, q~ as fp16 pairs for both k-halves)
  alignas(16) float cst[NH * kGroupHeads][4];      // a, b, sum P (int bits)
  alignas(16) float qn[NH * kGroupHeads];          // |q|
  alignas(16) float u[128];                        // appended key: R_K^T u (original domain)
  alignas(16) float z[128];                        // S u
  alignas(16) float tab[64];                       // key / value thresholds and centroids
  alignas(16) VecOut key[32];                      // appended key: codes and norms per lane
  alignas(16) int sig[NH * kGroupHeads + 1];       // fp16 scaling exponents (last: appended key residual)
};
static_assert(offsetof(Prologue<1>, u) % 16 == 0 && offsetof(Prologue<3>, u) % 16 == 0, "alignment");

// Store the three int8 limb words (Q2, Q1, Q0) of limb word `w` (coordinates or
// sketch rows 4w .. 4w + 3) of head `hj` (0..3) of a group straight into the
// B-fragment order the main loop reads: frag[k-tile][lane] holds, for lane (g, t),
// the words (n-tile 0: k rows 4t.., 16 + 4t..; n-tile 1: the same rows) of column g,
// where column 2 hj carries Q2 (n-tile 0) and Q0 (n-tile 1) and column 2 hj + 1
// carries Q1 (n-tile 0) and zero (n-tile 1). Word w sits in k-tile w >> 3, at row
// offset 16 ((w >> 2) & 1) + 4 (w & 3), i.e. lane t = w & 3, register (w >> 2) & 1.
__device__ __forceinline__ void put_frag(uint4 (&frag)[4][32], int hj, int w, uint32_t q2, uint32_t q1,
                                         uint32_t q0) {
  const int kt = w >> 3, sub = (w >> 2) & 1, tt = w & 3;
  uint32_t* even = reinterpret_cast<uint32_t*>(&frag[kt][4 * (2 * hj) + tt]);
  uint32_t* odd = reinterpret_cast<uint32_t*>(&frag[kt][4 * (2 * hj + 1) + tt]);
  even[sub] = q2;
  odd[sub] = q1;
  even[2 + sub] = q0;
  odd[2 + sub] = 0u;
}

// The same for group h of NH when groups are paired (two or more groups, code
// keys): n-tile 1 of the even group of a pair carries the lowest limb of both,
// column 2 hj for head hj of the even group and column 2 hj + 1 for head hj of
// the odd one, so that one product serves both and lane (g, t) still finds the
// lowest limbs of its own heads t and 4 + t in its accumulator. The odd group's
// own n-tile 1 is never read; an unpaired last group keeps a zero column.
template <int NH>
__device__ __forceinline__ void put_frag_paired(uint4 (&frags)[NH][2][4][32], int which, int h, int hj, int w,
                                                uint32_t q2, uint32_t q1, uint32_t q0) {
  const int kt = w >> 3, sub = (w >> 2) & 1, tt = w & 3;
  uint32_t* even = reinterpret_cast<uint32_t*>(&frags[h][which][kt][4 * (2 * hj) + tt]);
  uint32_t* odd = reinterpret_cast<uint32_t*>(&frags[h][which][kt][4 * (2 * hj + 1) + tt]);
  even[sub] = q2;
  odd[sub] = q1;
  if (h & 1) {
    reinterpret_cast<uint32_t*>(&frags[h - 1][which][kt][4 * (2 * hj + 1) + tt])[2 + sub] = q0;
  } else {
    even[2 + sub] = q0;
    if (h + 1 >= NH) odd[2 + sub] = 0u;
  }
}

// Rotate and code one vector held 4 per lane; returns codes in o, n and (keys) gamma,
// and the residual u = y - c[code] per lane.
__device__ __forceinline__ void rotate_and_code(const float (&x)[4], const float4 sg, const float* thr,
                                                const float* cen, int bits, int lane, VecOut& o, float (&u)[4]) {
  float v[4];
  float ss = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    ss = fmaf(x[e], x[e], ss);
    v[e] = x[e] * (&sg.x)[e];
  }
  ss = warp_sum(ss);
  const float n = sqrtf(ss);
  fwht128(v, lane);
  const float inv = n > 0.0f ? 1.0f / (n * 11.313708498984761f) : 0.0f;
  const int n_thr = (1 << bits) - 1;
  float uu = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float y = v[e] * inv;
    o.code[e] = encode(y, thr, n_thr);
    u[e] = y - cen[o.code[e]];
    uu = fmaf(u[e], u[e], uu);
    o.sgn[e] = 0;
  }
  o.norm = n;
  o.gamma = n * sqrtf(warp_sum(uu));
}

// Split-K decode attention, one launch per call; this is the body for one
// segment: a run of consecutive pages of one (sequence, KV head) pair (the
// kernel below says which segments a CTA serves). W warps per CTA, one CTA per
// SM. Each warp streams the segment's pages through a private ring of S
// shared-memory stages filled by 1-D bulk TMA copies. The first S pages of
// every warp, one per stage, are fixed (page p0 + warp + W k) and their copies
// go out as soon as the lengths and block table are read, before any barrier;
// all later pages are claimed one at a time from a shared counter, so warps
// that the scheduler favours take more pages and the warps of a CTA finish
// together. The prologue (query transform, and with APPEND the quantization of
// the new token) runs while the first copies are in flight.
//
// Per 16-token page a warp computes, with tokens on the rows of the products:
//   logits  int8 m16n8k32: A = key-code limbs (hi, lo) or 0/1 sign bytes of
//           tokens g and g+8, B = query limbs -> lane (g, t) gets head t of
//           tokens g and g + 8 with all limbs in its own registers;
//   values  fp16 m16n8k16: A = value centroids (coordinates x tokens),
//           B = softmax weights split into fp16 high parts (columns 0-3) and
//           low parts (columns 4-7), transposed into place with shuffles.
// APPEND: the CTA whose segment holds a sequence's last page first quantizes
// (k_new, v_new) of that sequence into position seq_len - 1; a warp that is
// given that page before then holds its copy back until the token is written.
//
// One piece of work of a CTA: logical pages [p0, p0 + len) of one (sequence, KV
// head) pair (clipped to the sequence), whose merged record goes to slot `slot`;
// the pair's records are slots first_slot .. first_slot + n_segs - 1.
struct Segment {
  int pair, p0, len;
  int slot, first_slot, n_segs;
  bool last;                     // the CTA's last segment
};

// LOOP: the CTA serves several segments one after the other (balanced split).
template <int BK, int BV, int NH, int MODE, bool LOOP>
__device__ __forceinline__ void decode_segment(const Tables& T, const DecodeArgs& A, const Segment& sg) {
  constexpr bool APPEND = MODE == 1;        // append the new token first (decode step)
  constexpr bool LOGITS = MODE == 2;        // write the logits; no softmax, no value sum
  constexpr bool KQ8 = BK == 8;              // q8_0 keys (raw query, block scales, no QJL)
  constexpr bool KF16 = BK == 4 && NH >= 2;  // 4-bit keys, two or more head groups: fp16 key products
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int W = DecodeWarps<NH, LOOP>::value;
  constexpr int kBlock = block_bytes_of(BK, BV);
  constexpr int S = decode_stages(W, kBlock);
  constexpr int kStatic = S;                   // pages per warp assigned before the claim counter
  constexpr int kSignOff = sec_scale(BK), kVOff = sec_v(BK), kNormOff = sec_norm(BK, BV);
  constexpr int kNormBytes = KQ8 ? 32 : 96;
  constexpr int kHeads = NH * kGroupHeads;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int pair = sg.pair;
  const int b = pair / A.n_kv, hk = pair % A.n_kv;
  // When one CTA serves several segments, the table pointers are made opaque per
  // segment, so that the loads through them are not hoisted out of the segment
  // loop (that would keep their registers live across every main loop).
  const uint16_t* tab_m = T.sketch_m;
  const float* tab_sk = T.signs_k;
  const float* tab_sv = T.signs_v;
  if constexpr (LOOP) asm volatile("" : "+l"(tab_m), "+l"(tab_sk), "+l"(tab_sv));

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + W * S * kBlock);
  static_assert((W * S * kBlock + W * S * 8) % 16 == 0, "prologue alignment");
  Prologue<NH>& P = *reinterpret_cast<Prologue<NH>*>(bars + W * S);
  int* s_btab = reinterpret_cast<int*>(&P + 1);   // physical ids of the chunk's claimable pages
  __shared__ int s_last, s_claim;
  __shared__ int s_lp[W * S];                     // logical page of each stage (-1: bad page id)
  __shared__ int s_def[W];                        // physical id of a copy held back for the append
  __shared__ uint64_t s_never;                    // test hook: a barrier nothing completes
  uint8_t* stage0 = smem + warp * S * kBlock;
  uint64_t* mybar = bars + warp * S;
  int* mylp = s_lp + warp * S;

  // The ring barriers first: they touch only this CTA's shared memory, and their
  // initialisation fences wait for this thread's earlier memory operations, so
  // they go ahead of every global load (a previous segment of this CTA may have
  // written the stage bytes through the generic proxy; bulk copies write them next).
  if (lane == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    for (int s = 0; s < S; ++s) mbar_init(mybar + s, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  // The prologue's own loads go out next, ahead of the page stream, so that they
  // do not queue behind it: the last eight warps' rows of M = S R_K (fp16 high
  // and low parts as m16n8k16 A fragments) and the inputs of this warp's jobs
  // (query heads warp, warp + W, ...; with APPEND the new key or value).
  constexpr int kSkW = W - kQjlRows / 16;          // warps kSkW.. own sketch rows 16 (warp - kSkW) + 0..15
  const int skw = warp - kSkW;
  uint4 amh[8], aml[8];
  if (!KQ8 && skw >= 0) {
    const uint4* F = reinterpret_cast<const uint4*>(tab_m) + skw * 8 * 32 + lane;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      amh[ks] = __ldg(F + ks * 32);
      aml[ks] = __ldg(F + kQjlRows / 16 * 8 * 32 + ks * 32);
    }
  }
  const float4 sgk = __ldg(reinterpret_cast<const float4*>(tab_sk) + lane);
  const float4 sgv = __ldg(reinterpret_cast<const float4*>(tab_sv) + lane);
  if (threadIdx.x < 16) {
    P.tab[threadIdx.x] = T.thr_k[threadIdx.x];
    P.tab[16 + threadIdx.x] = T.cen_k[threadIdx.x];
    P.tab[32 + threadIdx.x] = T.thr_v[threadIdx.x];
    P.tab[48 + threadIdx.x] = T.cen_v[threadIdx.x];
  }
  // 4-bit values: the fp16 A-operand registers of the value product come from a
  // byte-indexed table in shared memory, entry b = fp16x2 (c(b & 15), c(b >> 4))
  // with the first code in the low half, one load per two codes instead of the
  // 16-entry byte-permute lookup (whose bit-3 select costs more than the load).
  // For 2-bit values the 8-byte entries a byte would need collide on the banks,
  // and for 4-bit keys the limb pairs need two more byte-permutes per load: both
  // stay on the byte-permute lookups.
  __shared__ uint32_t s_vtab[BV == 4 && !LOGITS ? 256 : 1];
  // 4-bit keys: entry b = fp16x2 (c(b & 15), c(b >> 4)) of the key centroids (fp16
  // values), the A-operand pairs of the fp16 key products
  __shared__ uint32_t s_ktab[KF16 ? 256 : 1];
  if constexpr (KF16) {
    for (int e = threadIdx.x; e < 256; e += blockDim.x)
      s_ktab[e] = pack_half2(T.cen_k[e & 15], T.cen_k[e >> 4]);
  }
  if constexpr (BV == 4 && !LOGITS) {
    auto byte_of = [](const uint32_t (&tb)[4], int c) -> uint32_t { return (tb[c >> 2] >> (8 * (c & 3))) & 0xFFu; };
    for (int e = threadIdx.x; e < 256; e += blockDim.x)
      s_vtab[e] = byte_of(T.v_lo, e & 15) | (byte_of(T.v_hi, e & 15) << 8) | (byte_of(T.v_lo, e >> 4) << 16) |
                  (byte_of(T.v_hi, e >> 4) << 24);
  }
  // Everything above reads only the context's own tables, which no kernel writes.
  // Launched as a programmatic dependent of the previous kernel in the stream:
  // its memory operations are complete and visible once this wait returns, so
  // nothing it may have written (queries, lengths, block tables, the cache) is
  // read before it. (With LOOP, the kernel has already waited.) Before the wait,
  // only L2 prefetch hints go out for the lines read first after it: they move
  // no data into the SM, so they cannot observe anything stale.
  if constexpr (!LOOP) {
    const int n_bt = (min(sg.len, A.max_pages_per_seq - sg.p0) * 4 + 127) >> 7;   // block-table lines
    const int n_q = (A.group * 128 * (A.q_dtype == TQ_F32 ? 4 : 2) + 127) >> 7;   // query lines
    const int i = threadIdx.x;
    const char* addr = nullptr;
    if (i == 0) addr = reinterpret_cast<const char*>(A.seq_lens + b);
    else if (i <= n_bt)
      addr = reinterpret_cast<const char*>(A.block_tables + static_cast<int64_t>(b) * A.max_pages_per_seq + sg.p0) +
             128 * (i - 1);
    else if (i <= n_bt + n_q)
      addr = static_cast<const char*>(A.q) +
             (static_cast<size_t>(b) * A.n_q + hk * A.group) * 128 * (A.q_dtype == TQ_F32 ? 4 : 2) +
             128 * (i - 1 - n_bt);
    if (addr) asm volatile("prefetch.global.L2 [%0];" ::"l"(addr));
    asm volatile("griddepcontrol.wait;" ::: "memory");
  }
  const size_t kv_row = static_cast<size_t>(b) * A.n_kv + hk;
  constexpr int kQJobs = (kHeads + W - 1) / W;     // query heads per warp (at most)
  float xq[kQJobs][4];
#pragma unroll
  for (int i = 0; i < kQJobs; ++i) {
    const int j = warp + W * i;
    xq[i][0] = xq[i][1] = xq[i][2] = xq[i][3] = 0.0f;
    if (j < A.group) load_row4(A.q, static_cast<size_t>(b) * A.n_q + hk * A.group + j, A.q_dtype, lane, xq[i]);
  }
  // the append jobs: key (job kHeads) and value (kHeads + 1), on warps kHeads % W, (kHeads + 1) % W
  const int ajob = warp == kHeads % W ? kHeads : (warp == (kHeads + 1) % W ? kHeads + 1 : -1);
  float xa[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (APPEND && ajob >= 0) load_row4(ajob == kHeads ? A.k_new : A.v_new, kv_row, A.kv_dtype, lane, xa);
  // this warp's static pages (lane k holds page p0 + warp + W k), fetched before
  // the length is known (bounded by the table width; pages past the sequence are
  // discarded below)
  const int32_t* btab = A.block_tables + static_cast<int64_t>(b) * A.max_pages_per_seq;
  const int p0 = sg.p0;
  const int first_j = p0 + warp + lane * W;
  const int spec_phys = (lane < kStatic && first_j < A.max_pages_per_seq) ? __ldg(btab + first_j) : -1;
  // the first kSpecWin entries of the chunk's claimable window, also fetched now
  // (entries past the table width are skipped; past the sequence, never claimed)
  constexpr int kSpecPer = 2, kSpecWin = kSpecPer * W * 32;
  const int win_lim = min(sg.len, A.max_pages_per_seq - p0) - W * kStatic;
  int spec_win[kSpecPer];
#pragma unroll
  for (int r = 0; r < kSpecPer; ++r) {
    const int i = threadIdx.x + r * W * 32;
    spec_win[r] = i < win_lim ? __ldg(btab + p0 + W * kStatic + i) : -1;
  }

  int L = A.seq_lens[b];
  if (L < 0 || L > A.max_seq_len) {
    if (threadIdx.x == 0) set_error(T.err, TQ_DEV_BAD_LENGTH);
    L = L < 0 ? 0 : A.max_seq_len;
  }
  const int seq_pages = (L + kPage - 1) / kPage;
  const int p1 = min(p0 + sg.len, seq_pages);
  const int n_static = p1 > p0 + warp ? min(kStatic, (p1 - p0 - warp + W - 1) / W) : 0;
  const int n_dyn = max(0, p1 - p0 - W * kStatic);      // pages handed out by the claim counter
  // the CTA holding the last page appends the new token before that page is fetched
  const bool appender = APPEND && L > 0 && p0 <= seq_pages - 1 && seq_pages - 1 < p0 + sg.len;
  const int held = appender ? seq_pages - 1 : -1;

  // lane 0 only: start the transfer of logical page lp (physical `phys`) into stage s
  auto issue = [&](int phys, int lp, int s) {
    const bool ok = phys >= 0 && phys < A.n_pages;
    mylp[s] = ok ? lp : -1;
    if (!ok) {
      set_error(T.err, TQ_DEV_BAD_PAGE);
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mybar + s)) : "memory");
    } else if constexpr (LOGITS) {          // key codes and signs, then the norms; no value codes
      const uint8_t* src = A.cache + (static_cast<int64_t>(phys) * A.n_kv + hk) * kBlock;
      mbar_expect_tx(mybar + s, kVOff + kNormBytes);
      tma_load_1d(stage0 + s * kBlock, src, kVOff, mybar + s);
      tma_load_1d(stage0 + s * kBlock + kNormOff, src + kNormOff, kNormBytes, mybar + s);
    } else {
      mbar_expect_tx(mybar + s, kBlock);
      tma_load_1d(stage0 + s * kBlock, A.cache + (static_cast<int64_t>(phys) * A.n_kv + hk) * kBlock, kBlock,
                  mybar + s);
    }
  };
  // Ring bookkeeping (warp-uniform): stages [0, filled) are taken in ring order;
  // stage def_stage (if >= 0) holds the page being appended, issued after the
  // append. Lane k issues stage k of the static pages.
  int filled = n_static, def_stage = -1;
  {
    const int lp = p0 + warp + W * lane;
    const bool mine = lane < n_static, defer = mine && lp == held;
    if (defer) {
      s_def[warp] = spec_phys;
      mylp[lane] = lp;
    } else if (mine) {
      issue(spec_phys, lp, lane);
    }
    const unsigned dm = __ballot_sync(kFull, defer);
    if (dm) def_stage = __ffs(dm) - 1;
  }

  // ---- prologue, while the first pages are in flight
  // Raw queries for the sketch product, with their fp16 scaling exponents and
  // norms; the QJL limb sums start at zero.
  if constexpr (!KQ8) {
#pragma unroll
    for (int i = 0; i < kQJobs; ++i) {
      const int j = warp + W * i;
      if (j >= kHeads) continue;                   // warp-uniform
      const float* x = xq[i];
      const float mx = warp_max(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))));
      const float ss = warp_sum(fmaf(x[0], x[0], fmaf(x[1], x[1], fmaf(x[2], x[2], x[3] * x[3]))));
      reinterpret_cast<float4*>(&P.qraw[j][0])[lane] = make_float4(x[0], x[1], x[2], x[3]);
      if (lane == 0) {
        int E = 0;
        if (mx > 0.0f) E = max(exp_above(mx), -115);   // 2^(10-E) stays a normal float
        P.sig[j] = 10 - E;                             // fp16 high/low split near 2^10
        P.qn[j] = sqrtf(ss);
        P.cst[j][2] = __int_as_float(0);
      }
    }
  }
  if (threadIdx.x == 0) s_claim = W * kStatic;
#pragma unroll
  for (int r = 0; r < kSpecPer; ++r) {
    const int i = threadIdx.x + r * W * 32;
    if (i < n_dyn) s_btab[i] = spec_win[r];
  }
  for (int i = kSpecWin + threadIdx.x; i < n_dyn; i += W * 32) s_btab[i] = btab[p0 + W * kStatic + i];
  __syncthreads();
  // Fill the rest of the ring from the claim counter (lane k takes stage
  // filled + k), and claim one more page to keep pending for the first refill.
  int pend;                               // next claimed logical page (-1: none); lane 0 updates it
  {
    const int want = S - filled + 1;
    int base = 0;
    if (lane == 0) base = atomicAdd(&s_claim, want);
    base = __shfl_sync(kFull, base, 0);
    const int nvalid = min(max(p1 - p0 - base, 0), want);   // claims that fall inside the chunk
    const int nfill = min(nvalid, want - 1);
    const int lp = p0 + base + lane;
    const bool mine = lane < nfill, defer = mine && lp == held;
    if (mine) {
      const int phys = s_btab[lp - p0 - W * kStatic];
      if (defer) {
        s_def[warp] = phys;
        mylp[filled + lane] = lp;
      } else {
        issue(phys, lp, filled + lane);
      }
    }
    const unsigned dm = __ballot_sync(kFull, defer);
    if (dm) def_stage = filled + __ffs(dm) - 1;
    pend = nvalid == want ? p0 + base + want - 1 : -1;
    filled += nfill;
  }
  const int pos = L - 1;
  uint8_t* ablk = nullptr;                // block receiving the appended token
  if (appender) {
    const int phys = btab[pos / kPage];
    if (phys >= 0 && phys < A.n_pages) ablk = A.cache + (static_cast<int64_t>(phys) * A.n_kv + hk) * kBlock;
    else if (threadIdx.x == 0) set_error(T.err, TQ_DEV_BAD_SLOT);
  }
  // Jobs: the query limbs, and (appender) the quantization of the new key and
  // value. The sketch warps meanwhile form p = M q = S q~ for every query head.
#pragma unroll
  for (int i = 0; i < kQJobs; ++i) {
    const int j = warp + W * i;
    if (j >= kHeads) continue;                     // warp-uniform
    float x[4] = {xq[i][0], xq[i][1], xq[i][2], xq[i][3]};
    if constexpr (!KQ8) {                          // q~ = H D_K q / sqrt(d); q8_0 keys use q itself
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] *= (&sgk.x)[e];
      fwht128(x, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] *= kInvSqrtD;
    }
    const float qmax = warp_max(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))));
    int eq;
    if constexpr (KF16) {
      // q~ 2^sig as fp16 high and low parts (|q~ 2^sig| < 2^10) in the B order of the
      // fp16 key products: k-tile kt, half jh = coordinates 32 kt + 16 jh + 4 t' + 0..3
      // at lane (g', t'), column g' = 2 (head) + part; this lane holds the four
      // coordinates 4 lane .. 4 lane + 3, i.e. kt = lane >> 3, jh = (lane >> 2) & 1, t' = lane & 3
      const int E = qmax > 0.0f ? max(exp_above(qmax), -100) : 0;
      eq = 10 - E;
      const float sc = pow2i(eq);
      float hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v = x[e] * sc;
        hi[e] = __half2float(__float2half_rn(v));
        lo[e] = v - hi[e];
      }
      const int kt = lane >> 3, jh = (lane >> 2) & 1, tt = lane & 3, hj = j & 3;
      uint32_t* ph = reinterpret_cast<uint32_t*>(&P.qb[j >> 2][0][kt][4 * (2 * hj) + tt]);
      uint32_t* pl = reinterpret_cast<uint32_t*>(&P.qb[j >> 2][0][kt][4 * (2 * hj + 1) + tt]);
      ph[2 * jh] = pack_half2(hi[0], hi[1]);
      ph[2 * jh + 1] = pack_half2(hi[2], hi[3]);
      pl[2 * jh] = pack_half2(lo[0], lo[1]);
      pl[2 * jh + 1] = pack_half2(lo[2], lo[3]);
    } else {
      eq = pick_exponent24(qmax);
      const Limbs lq = split3(x, eq);
      if constexpr (!KQ8 && NH >= 2) put_frag_paired<NH>(P.qb, 0, j >> 2, j & 3, lane, lq.w2, lq.w1, lq.w0);
      else put_frag(P.qb[j >> 2][0], j & 3, lane, lq.w2, lq.w1, lq.w0);   // lane l: coordinates 4l .. 4l + 3
    }
    if (lane == 0) {
      const bool real = j < A.group;
      P.cst[j][0] = real ? A.scale * kLog2e * pow2i(-eq - (KQ8 || KF16 ? 0 : T.k_exp)) : 0.0f;
      if (KQ8) {
        P.cst[j][1] = 0.0f;
        P.cst[j][2] = __int_as_float(0);
      }
    }
  }
  if (ablk && ajob == kHeads) {                    // the appended key
    if constexpr (KQ8) {
      store_key_q8(ablk, pos % kPage, xa, lane);
    } else {
      float u[4];
      VecOut o;
      rotate_and_code(xa, sgk, P.tab, P.tab + 16, BK, lane, o, u);
      // S u = M R_K^T u with R_K^T u = D_K H u / sqrt(d)
      fwht128(u, lane);
      float mx = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        u[e] *= (&sgk.x)[e] * kInvSqrtD;
        P.u[4 * lane + e] = u[e];
        mx = fmaxf(mx, fabsf(u[e]));
      }
      mx = warp_max(mx);
      int E = 0;
      if (mx > 0.0f) E = max(exp_above(mx), -115);
      if (lane == 0) P.sig[kHeads] = 10 - E;
      P.key[lane] = o;
    }
  } else if (ablk && ajob == kHeads + 1) {         // the appended value
    float u[4];
    VecOut o;
    rotate_and_code(xa, sgv, P.tab + 32, P.tab + 48, BV, lane, o, u);
    store_value_token(ablk, pos % kPage, BK, BV, o, lane);
    if (lane == 0) store_norm(ablk, BK, BV, 2, pos % kPage, o.norm);
  }
  // Sketch products on the tensor cores: warp kSkW + w owns rows 16w .. 16w+15 of
  // M = S R_K, as fp16 high and low parts. The B columns are (source s, fp16 high
  // part) and (source s, fp16 low part) of x_s * 2^sig_s. On return, lane (g, t)
  // holds rows 16w + g (c[0] + c[1]) and 16w + g + 8 (c[2] + c[3]) of source t,
  // still scaled by 2^sig_t.
  auto sketch_m = [&](const float* vec, int pitch, const int* sig, int sources, float (&c)[4]) {
    const int src = g >> 1;
    const bool has = src < sources;
    const float sc = has ? pow2i(sig[src]) : 0.0f;
    const bool lo_col = g & 1;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    c[0] = c[1] = c[2] = c[3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      float2 u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
      if (has) {
        u0 = *reinterpret_cast<const float2*>(vec + src * pitch + 16 * ks + 2 * t);
        u1 = *reinterpret_cast<const float2*>(vec + src * pitch + 16 * ks + 2 * t + 8);
      }
      const float2 v0 = make_float2(u0.x * sc, u0.y * sc), v1 = make_float2(u1.x * sc, u1.y * sc);
      const __half2 h0 = __floats2half2_rn(v0.x, v0.y), h1 = __floats2half2_rn(v1.x, v1.y);
      __half2 b0 = h0, b1 = h1;
      if (lo_col) {
        const float2 r0 = __half22float2(h0), r1 = __half22float2(h1);
        b0 = __floats2half2_rn(v0.x - r0.x, v0.y - r0.y);
        b1 = __floats2half2_rn(v1.x - r1.x, v1.y - r1.y);
      }
      const uint32_t ub0 = *reinterpret_cast<uint32_t*>(&b0), ub1 = *reinterpret_cast<uint32_t*>(&b1);
      mma_f16(c, amh[ks].x, amh[ks].y, amh[ks].z, amh[ks].w, ub0, ub1);
      mma_f16(d, aml[ks].x, aml[ks].y, aml[ks].z, aml[ks].w, ub0, ub1);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] += d[e];
  };
  if (!KQ8 && skw >= 0) {
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float c[4];
      sketch_m(&P.qraw[4 * h][0], kQrawPitch, &P.sig[4 * h], 4, c);
      // int8 limbs of P = p 2^ep for head j = 4h + t, rows 16 skw + g (+8). The
      // exponent comes from the bound |p_r| <= |M_r| |q|, the same in every warp.
      const int j = 4 * h + t;
      const float inv = pow2i(-P.sig[j]);
      const float p0 = (c[0] + c[1]) * inv, p1 = (c[2] + c[3]) * inv;
      const int ep = pick_exponent24(T.m_rownorm * P.qn[j] * 1.0001f);
      const float f = pow2i(ep);
      const int Q0 = __float2int_rn(p0 * f), Q1 = __float2int_rn(p1 * f);
      // limbs of row 16 skw + g go to byte g & 3 of word 4 skw + (g >> 2); row +8 to word + 2
      const int sh = 8 * (g & 3);
      uint32_t w[6];
      {
        const int a0 = ((Q0 + 128) & 255) - 128, r0 = (Q0 - a0) >> 8, a1 = ((r0 + 128) & 255) - 128;
        const int b0 = ((Q1 + 128) & 255) - 128, r1 = (Q1 - b0) >> 8, b1 = ((r1 + 128) & 255) - 128;
        w[0] = static_cast<uint32_t>(a0 & 0xFF) << sh;
        w[1] = static_cast<uint32_t>(a1 & 0xFF) << sh;
        w[2] = static_cast<uint32_t>(((r0 - a1) >> 8) & 0xFF) << sh;
        w[3] = static_cast<uint32_t>(b0 & 0xFF) << sh;
        w[4] = static_cast<uint32_t>(b1 & 0xFF) << sh;
        w[5] = static_cast<uint32_t>(((r1 - b1) >> 8) & 0xFF) << sh;
      }
#pragma unroll
      for (int k = 0; k < 6; ++k) {
        w[k] |= __shfl_xor_sync(kFull, w[k], 4);
        w[k] |= __shfl_xor_sync(kFull, w[k], 8);
      }
      int ps = Q0 + Q1;
      ps += __shfl_xor_sync(kFull, ps, 4);
      ps += __shfl_xor_sync(kFull, ps, 8);
      ps += __shfl_xor_sync(kFull, ps, 16);
      if ((g & 3) == 0) {
        const int wd = 4 * skw + (g >> 2);
        if constexpr (NH >= 2) {
          put_frag_paired<NH>(P.qb, 1, h, t, wd, w[2], w[1], w[0]);
          put_frag_paired<NH>(P.qb, 1, h, t, wd + 2, w[5], w[4], w[3]);
        } else {
          put_frag(P.qb[h][1], t, wd, w[2], w[1], w[0]);
          put_frag(P.qb[h][1], t, wd + 2, w[5], w[4], w[3]);
        }
      }
      if (g == 0) {
        atomicAdd(reinterpret_cast<int*>(&P.cst[j][2]), j < A.group ? ps : 0);
        if (skw == 0)
          P.cst[j][1] = j < A.group ? A.scale * kLog2e * kSqrtPiOver2 / kQjlRows * pow2i(-ep) : 0.0f;
      }
    }
  }
  __syncthreads();
  if (!KQ8 && ablk) {                              // CTA-uniform: the appended key's sign bits
    if (skw >= 0) {
      float c[4];
      sketch_m(P.u, 128, &P.sig[kHeads], 1, c);
      if (t == 0) {
        const float inv = pow2i(-P.sig[kHeads]);
        P.z[16 * skw + g] = (c[0] + c[1]) * inv;
        P.z[16 * skw + g + 8] = (c[2] + c[3]) * inv;
      }
    }
    __syncthreads();
    if (ajob == kHeads) {
      VecOut o = P.key[lane];
#pragma unroll
      for (int e = 0; e < 4; ++e) o.sgn[e] = P.z[4 * lane + e] >= 0.0f ? 1 : 0;
      store_key_token(ablk, pos % kPage, BK, o, lane);
      if (lane == 0) {
        store_norm(ablk, BK, BV, 0, pos % kPage, o.norm);
        store_norm(ablk, BK, BV, 1, pos % kPage, o.gamma);
      }
    }
  }
  if (ablk) {                                      // CTA-uniform
    asm volatile("fence.proxy.async.global;" ::: "memory");   // the page is next read by the TMA unit
    __syncthreads();
  }
  if (lane == 0 && def_stage >= 0) issue(s_def[warp], held, def_stage);   // the appended page
  __syncwarp();
  __syncwarp();                           // lane 0's stage records are visible to the warp

  // B fragments (query limbs): P.qb[group][q~ / p][k-tile][lane], one uint4 per lane
  // and k-tile, read with one vector load per use (see put_frag).
  float ca[NH], cb[NH];
  int csum[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    ca[h] = P.cst[4 * h + t][0];
    cb[h] = P.cst[4 * h + t][1];
    csum[h] = __float_as_int(P.cst[4 * h + t][2]);
  }
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
  float lsum[NH], mp2[NH], smx[NH];           // smx: running maximum of l2 (Sparse V only)
#pragma unroll
  for (int h = 0; h < NH; ++h) { lsum[h] = 0.0f; mp2[h] = kNegBig; smx[h] = kNegBig; }

  // transpose sources for the value-product B operand (see below)
  const int h4 = g & 3;
  const int src0 = 4 * (2 * t) + h4, src1 = 4 * (2 * t + 1) + h4;
  const bool hi_col = g < 4;

  bool alive = true;
  int s = 0;
  unsigned parity = 0;
  int inflight = filled;                  // stages holding a page not yet consumed (warp-uniform)
  // Test hook (TQ_TEST_WAIT_RUNS_OUT): warp 0 of block 0 first waits, with a short
  // limit, on a barrier that nothing completes, so that its wait runs out.
  bool runout = (T.test_flags & 1u) && blockIdx.x == 0 && warp == 0;
  if (runout) {
    if (lane == 0) {
      mbar_init(&s_never, 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
  }
  // ---- one page's logits (row a4, first half): returns, for tokens g and g + 8 of
  // the page in stage st and each head group, l2 + log2|v| (l2 = the logit in log2
  // units; -inf outside the sequence), the token's 1 / |v| and log2|v|, and the
  // page's value-code words.
  struct PageLogits {
    float lp2[NH][2];
    float rnv[2], lgv[2];
    uint32_t vw[2 * BV];
  };
  auto page_logits = [&](int st, PageLogits& o) {
    const int lp = mylp[st];
    const bool page_ok = lp >= 0;
    const uint8_t* blk = stage0 + st * kBlock;

    // ---- this lane's operands from the staged block (tokens g and g + 8)
    // (q8_0 keys: 16 words of int8 key values, the same count as 2 * 8 code words)
    uint32_t kw[2 * BK];
    lds_words<2 * BK>(reinterpret_cast<const uint32_t*>(blk) + lane * 2 * BK, kw);
    uint2 sw = make_uint2(0u, 0u);
    uint4 sc4 = make_uint4(0u, 0u, 0u, 0u);   // q8_0: fp16 block scales 4 th + kt of tokens g, g + 8
    if constexpr (KQ8) sc4 = *reinterpret_cast<const uint4*>(blk + kSignOff + 16 * g);
    else sw = reinterpret_cast<const uint2*>(blk + kSignOff)[lane];
    if constexpr (!LOGITS) lds_words<2 * BV>(reinterpret_cast<const uint32_t*>(blk + kVOff) + lane * 2 * BV, o.vw);
    const uint32_t* nrm = reinterpret_cast<const uint32_t*>(blk + kNormOff);
    float2 nK = make_float2(0.0f, 0.0f), gm = make_float2(0.0f, 0.0f), nV;
    if constexpr (KQ8) {
      const uint32_t rv = nrm[g];
      nV = __half22float2(*reinterpret_cast<const __half2*>(&rv));
    } else {
      const uint32_t rk = nrm[g], rg = nrm[8 + g], rv = nrm[16 + g];
      nK = __half22float2(*reinterpret_cast<const __half2*>(&rk));
      gm = __half22float2(*reinterpret_cast<const __half2*>(&rg));
      nV = __half22float2(*reinterpret_cast<const __half2*>(&rv));
    }

    // ---- logits: int8 tensor-core products, tokens on the rows
    int dh[NH][2][4], dl[NH][2][4], ds[NH][2][4];
    float dk[NH][4];                          // 4-bit keys: fp16 products (columns: head t high, low part)
#pragma unroll
    for (int h = 0; h < NH; ++h) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) dh[h][nt][c] = dl[h][nt][c] = ds[h][nt][c] = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) dk[h][c] = 0.0f;
    }
    float lq8[NH][2];                        // q8_0: sum over blocks of d_b <Q_b, k8_b>
    if constexpr (KQ8) {
      float dsc[2][4];
      {
        const uint32_t sw4[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&sw4[i]));
          dsc[i >> 1][2 * (i & 1)] = f.x;
          dsc[i >> 1][2 * (i & 1) + 1] = f.y;
        }
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) lq8[h][0] = lq8[h][1] = 0.0f;
#pragma unroll
      for (int kt = 0; kt < 4; ++kt) {
        // A fragment of block kt: tokens g, g + 8 (rows), coordinates 4t.. and 16+4t.. (columns)
        const uint32_t ak[4] = {kw[2 * kt], kw[8 + 2 * kt], kw[2 * kt + 1], kw[8 + 2 * kt + 1]};
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
          const uint4 fq = P.qb[h][0][kt][lane];
          mma_s8(d0, ak, fq.x, fq.y);
          mma_s8(d1, ak, fq.z, fq.w);
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            // columns: (Q2, Q1) of head t in d0, Q0 in d1; |Q2 . k| 2^16 can pass 2^31, so in fp32
            const float m = fmaf(65536.0f, static_cast<float>(d0[2 * r]),
                                 fmaf(256.0f, static_cast<float>(d0[2 * r + 1]), static_cast<float>(d1[2 * r])));
            lq8[h][r] = fmaf(dsc[r][kt], m, lq8[h][r]);
          }
        }
      }
    } else {
      uint32_t sel0[8], sel1[8];
      if constexpr (!KF16) {
        key_selectors<BK>(kw, sel0);
        key_selectors<BK>(kw + BK, sel1);
      }
      const uint8_t* kt8 = reinterpret_cast<const uint8_t*>(s_ktab);
#pragma unroll
      for (int kt = 0; kt < 4; ++kt) {
        uint32_t ah[4], al[4], as[4];
        if constexpr (KF16) {
          // word kt of token g (g + 8): byte 0 = coordinates 4t, 4t + 1 and byte 1 = 4t + 2, 4t + 3
          // (the A pairs of the first k-half), bytes 2, 3 = coordinates 16 + 4t .. 16 + 4t + 3
          // (the second k-half); the B fragments use the same coordinate order
          const uint32_t w0 = kw[kt], w1 = kw[4 + kt];
          uint32_t a[8];
          a[0] = *reinterpret_cast<const uint32_t*>(kt8 + ((w0 << 2) & 0x3FCu));
          a[1] = *reinterpret_cast<const uint32_t*>(kt8 + ((w1 << 2) & 0x3FCu));
          a[2] = *reinterpret_cast<const uint32_t*>(kt8 + (shr<6>(w0) & 0x3FCu));
          a[3] = *reinterpret_cast<const uint32_t*>(kt8 + (shr<6>(w1) & 0x3FCu));
          a[4] = *reinterpret_cast<const uint32_t*>(kt8 + (shr<14>(w0) & 0x3FCu));
          a[5] = *reinterpret_cast<const uint32_t*>(kt8 + (shr<14>(w1) & 0x3FCu));
          a[6] = *reinterpret_cast<const uint32_t*>(kt8 + (shr<22>(w0) & 0x3FCu));
          a[7] = *reinterpret_cast<const uint32_t*>(kt8 + (shr<22>(w1) & 0x3FCu));
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            const uint4 fq = P.qb[h][0][kt][lane];
            mma_f16(dk[h], a[0], a[1], a[2], a[3], fq.x, fq.y);
            mma_f16(dk[h], a[4], a[5], a[6], a[7], fq.z, fq.w);
          }
        } else {
          key_limbs<BK>(sel0[2 * kt], kth_, ktl_, ah[0], al[0]);          // token g,     k 4t..
          key_limbs<BK>(sel1[2 * kt], kth_, ktl_, ah[1], al[1]);          // token g + 8, k 4t..
          key_limbs<BK>(sel0[2 * kt + 1], kth_, ktl_, ah[2], al[2]);      // token g,     k 16+4t..
          key_limbs<BK>(sel1[2 * kt + 1], kth_, ktl_, ah[3], al[3]);      // token g + 8, k 16+4t..
        }
        as[0] = (kt == 0 ? sw.x : __umulhi(sw.x, 1u << (32 - 2 * kt))) & 0x01010101u;
        as[1] = (kt == 0 ? sw.y : __umulhi(sw.y, 1u << (32 - 2 * kt))) & 0x01010101u;
        as[2] = __umulhi(sw.x, 1u << (31 - 2 * kt)) & 0x01010101u;
        as[3] = __umulhi(sw.y, 1u << (31 - 2 * kt)) & 0x01010101u;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const uint4 fq = P.qb[h][0][kt][lane];
          const uint4 fp = P.qb[h][1][kt][lane];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            if constexpr (NH >= 2) {
              if (nt == 1 && (h & 1)) continue;              // the pair's even group serves n-tile 1
            }
            const uint32_t q0 = nt ? fq.z : fq.x, q1 = nt ? fq.w : fq.y;
            const uint32_t r0 = nt ? fp.z : fp.x, r1 = nt ? fp.w : fp.y;
            if constexpr (!KF16) {
              mma_s8(dh[h][nt], ah, q0, q1);
              if (nt == 0) mma_s8(dl[h][nt], al, q0, q1);   // Q0 x C_lo (below 2^-22 of the sum) is left out
            }
            mma_s8(ds[h][nt], as, r0, r1);
          }
        }
      }
    }

    // One running maximum of l2 + log2|v| per head (see the softmax below). Norms
    // are floored at 2^-24 so that a zero value vector still counts in the denominator.
    const int n_valid = page_ok ? L - lp * kPage : 0;     // tokens of this page inside the sequence
    o.lgv[0] = lg2(fmaxf(nV.x, 5.9604645e-8f));
    o.lgv[1] = lg2(fmaxf(nV.y, 5.9604645e-8f));
    o.rnv[0] = ex2(-o.lgv[0]);
    o.rnv[1] = ex2(-o.lgv[1]);
#pragma unroll
    for (int h = 0; h < NH; ++h) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        // accumulator columns: n-tile 0 -> (Q2, Q1) of head t, n-tile 1 -> (Q0, 0)
        //   <Q,C> = 2^16 (256 Q2.Chi + Q2.Clo + Q1.Chi) + 256 (Q1.Clo + Q0.Chi) [+ Q0.Clo, left out]
        float l2;
        if constexpr (KQ8) {
          l2 = ca[h] * lq8[h][r];
        } else {
          int hiw, low, sj;
          if constexpr (NH == 1) {
            hiw = 256 * dh[h][0][2 * r] + dl[h][0][2 * r] + dh[h][0][2 * r + 1];
            low = 256 * (dl[h][0][2 * r + 1] + dh[h][1][2 * r]);
            sj = 65536 * ds[h][0][2 * r] + 256 * ds[h][0][2 * r + 1] + ds[h][1][2 * r];
          } else {
            // the lowest limbs: n-tile 1 of this group, or (the odd group of a pair)
            // column 2t + 1 of the even group's
            const int q0t = (h & 1) ? dh[h & ~1][1][2 * r + 1] : dh[h][1][2 * r];
            const int p0t = (h & 1) ? ds[h & ~1][1][2 * r + 1] : ds[h][1][2 * r];
            hiw = 256 * dh[h][0][2 * r] + dl[h][0][2 * r] + dh[h][0][2 * r + 1];
            low = 256 * (dl[h][0][2 * r + 1] + q0t);
            sj = 65536 * ds[h][0][2 * r] + 256 * ds[h][0][2 * r + 1] + p0t;
          }
          const float main = KF16 ? dk[h][2 * r] + dk[h][2 * r + 1]
                                  : fmaf(65536.0f, static_cast<float>(hiw), static_cast<float>(low));
          const float nk = r ? nK.y : nK.x, gg = r ? gm.y : gm.x;
          l2 = fmaf(nk * ca[h], main, gg * cb[h] * static_cast<float>(2 * sj - csum[h]));
        }
        if constexpr (LOGITS) {               // natural-log logit of (token g + 8r, head 4h + t)
          const int qi = 4 * h + t;
          if ((g + 8 * r) < n_valid && qi < A.group)
            A.logits[(static_cast<int64_t>(b) * A.n_q + hk * A.group + qi) * A.logits_stride + lp * kPage + g +
                     8 * r] = l2 * 0.6931471805599453f;
        }
        o.lp2[h][r] = (g + 8 * r) < n_valid ? l2 + o.lgv[r] : -INFINITY;
      }
    }
  };

  // ---- softmax over one or two pages (row a4, second half): one running maximum
  // of l2 + log2|v| per head. The fp16 weight of token t is
  // w_t = 2^(l2_t + log2|v_t| - m) <= 2^8 (the maximum is only moved when it grows
  // by more than 8), and the softmax denominator gathers w_t / |v_t| = 2^(l2_t - m).
  // Returns each page's value-product B operand (weights as fp16 high and low
  // parts, transposed into place) and whether its values may be skipped (Sparse V).
  auto softmax = [&](int npg, PageLogits* pg, uint32_t (*pb)[NH][2], bool* skip) {
    bool kept[2] = {false, false};        // Sparse V: this lane keeps a (token, head) value
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float pm = fmaxf(pg[0].lp2[h][0], pg[0].lp2[h][1]);
      if (npg == 2) pm = fmaxf(pm, fmaxf(pg[1].lp2[h][0], pg[1].lp2[h][1]));
      // The head's maximum over its 8 lanes is only needed when it moves: when no
      // lane's own values exceed the margin, no head's maximum does either.
      if (__any_sync(kFull, pm > mp2[h] + 8.0f)) {
        pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 4));
        pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 8));
        pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, 16));
        const bool need = pm > mp2[h] + 8.0f;
        const float fac = need ? ex2(mp2[h] - pm) : 1.0f;
        if (need) mp2[h] = pm;
        lsum[h] *= fac;
        // value accumulator columns 2t, 2t+1 hold heads (2t)&3, (2t+1)&3 (columns 4-7: low parts)
        const float f0 = __shfl_sync(kFull, fac, (2 * t) & 3);
        const float f1 = __shfl_sync(kFull, fac, (2 * t + 1) & 3);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[h][mt][0] *= f0; acc[h][mt][1] *= f1; acc[h][mt][2] *= f0; acc[h][mt][3] *= f1;
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (q == 1 && npg == 1) break;
        const PageLogits& o = pg[q];
        float w0 = ex2(o.lp2[h][0] - mp2[h]), w1 = ex2(o.lp2[h][1] - mp2[h]);
        lsum[h] = fmaf(w0, o.rnv[0], fmaf(w1, o.rnv[1], lsum[h]));
        if (A.sparse) {
          // Sparse V: a value is skipped when its attention weight is below the
          // threshold times the largest weight seen so far by this warp (never more
          // than the largest overall); the denominator above still counts it.
          const float l20 = o.lp2[h][0] - o.lgv[0], l21 = o.lp2[h][1] - o.lgv[1];
          float ps = fmaxf(l20, l21);
          ps = fmaxf(ps, __shfl_xor_sync(kFull, ps, 4));
          ps = fmaxf(ps, __shfl_xor_sync(kFull, ps, 8));
          ps = fmaxf(ps, __shfl_xor_sync(kFull, ps, 16));
          smx[h] = fmaxf(smx[h], ps);
          const float cut = smx[h] + A.sparse_log2;
          const bool k0 = l20 >= cut, k1 = l21 >= cut;
          w0 = k0 ? w0 : 0.0f;
          w1 = k1 ? w1 : 0.0f;
          kept[q] = kept[q] || k0 || k1;
        }
        // weights of (token g, head t) and (token g+8, head t): high fp16 parts and residuals
        const __half2 whi = __floats2half2_rn(w0, w1);
        const float2 wr = __half22float2(whi);
        const __half2 wlo = __floats2half2_rn(w0 - wr.x, w1 - wr.y);
        const uint32_t uhi = *reinterpret_cast<const uint32_t*>(&whi);
        const uint32_t ulo = *reinterpret_cast<const uint32_t*>(&wlo);
        // value-product B operand: lane (g', t') needs column g' (head g'&3, high part
        // if g' < 4) at tokens 2t', 2t'+1 (-> b0) and 2t'+8, 2t'+9 (-> b1); tokens 2t'
        // and 2t'+8 of a head live in lane 4*(2t') + head, tokens 2t'+1, 2t'+9 in the next quad.
        const uint32_t x0h = __shfl_sync(kFull, uhi, src0), x0l = __shfl_sync(kFull, ulo, src0);
        const uint32_t x1h = __shfl_sync(kFull, uhi, src1), x1l = __shfl_sync(kFull, ulo, src1);
        const uint32_t x0 = hi_col ? x0h : x0l, x1 = hi_col ? x1h : x1l;
        pb[q][h][0] = prmt(x0, x1, 0x5410u);
        pb[q][h][1] = prmt(x0, x1, 0x7632u);
      }
    }
    skip[0] = A.sparse && !__any_sync(kFull, kept[0]);
    skip[1] = A.sparse && !__any_sync(kFull, kept[1]);
  };

  // ---- weighted value sum in the rotated domain: fp16 tensor-core products
  auto value_product = [&](const uint32_t (&vw)[2 * BV], const uint32_t (&pbq)[NH][2]) {
    if constexpr (BV == 4) {
      // m-tile mt: word mt, whose bytes 0 .. 3 give A registers 0 .. 3
      const uint8_t* vt8 = reinterpret_cast<const uint8_t*>(s_vtab);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const uint32_t w = vw[mt];
        const uint32_t a0 = *reinterpret_cast<const uint32_t*>(vt8 + ((w << 2) & 0x3FCu));
        const uint32_t a1 = *reinterpret_cast<const uint32_t*>(vt8 + (shr<6>(w) & 0x3FCu));
        const uint32_t a2 = *reinterpret_cast<const uint32_t*>(vt8 + (shr<14>(w) & 0x3FCu));
        const uint32_t a3 = *reinterpret_cast<const uint32_t*>(vt8 + (shr<22>(w) & 0x3FCu));
#pragma unroll
        for (int h = 0; h < NH; ++h) mma_f16(acc[h][mt], a0, a1, a2, a3, pbq[h][0], pbq[h][1]);
      }
    } else {
      uint32_t vs[16];
      value_selectors<BV>(vw, vs);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a0, a1, a2, a3;
        value_regs<BV>(vs[2 * mt], vlo_, vhi_, a0, a1);
        value_regs<BV>(vs[2 * mt + 1], vlo_, vhi_, a2, a3);
#pragma unroll
        for (int h = 0; h < NH; ++h) mma_f16(acc[h][mt], a0, a1, a2, a3, pbq[h][0], pbq[h][1]);
      }
    }
  };

  // ---- refill stage st with the pending claim (all its reads are consumed), and
  // claim the next page; that claim is only used at the next refill
  auto refill_stage = [&](int st) {
    const bool refill = __shfl_sync(kFull, pend, 0) >= 0;
    __syncwarp();
    if (lane == 0 && refill) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(s_btab[pend - p0 - W * kStatic], pend, st);
      const int next = p0 + atomicAdd(&s_claim, 1);
      pend = next < p1 ? next : -1;
    }
    __syncwarp();
    if (!refill) --inflight;
  };

  while (inflight > 0) {
    // Two pages per iteration while two are in flight (one group of 4 query
    // heads, uniform split): their key work is independent and interleaves, and
    // the softmax reduction is shared. With more head groups the second page's
    // registers would spill, and the balanced split spends them on more warps;
    // one page at a time is faster there.
    const int npg = (NH == 1 && !LOOP && inflight >= 2) ? 2 : 1;
    const int s2 = s + 1 == S ? 0 : s + 1;
    const unsigned parity2 = s + 1 == S ? parity ^ 1u : parity;
    // warp-uniform outcome: the page body runs warp-wide shuffles and mma.sync
    bool landed;
    if (runout) {
      landed = __all_sync(kFull, mbar_wait(&s_never, 0u, 1ll << 16));
      runout = false;
    } else {
      landed = __all_sync(kFull, mbar_wait(mybar + s, parity));
    }
    if (landed && npg == 2) landed = __all_sync(kFull, mbar_wait(mybar + s2, parity2));
    if (!landed) {
      if (lane == 0) set_error(T.err, TQ_DEV_TIMEOUT);
      alive = false;
      break;
    }
    PageLogits pg[2];
    page_logits(s, pg[0]);
    if (npg == 2) page_logits(s2, pg[1]);
    if constexpr (!LOGITS) {
      uint32_t pb[2][NH][2];
      bool skip[2];
      softmax(npg, pg, pb, skip);
      if (!skip[0]) value_product(pg[0].vw, pb[0]);
      if (npg == 2 && !skip[1]) value_product(pg[1].vw, pb[1]);
    }
    refill_stage(s);
    if (npg == 2) refill_stage(s2);
    s += npg;
    if (s >= S) {
      s -= S;
      parity ^= 1u;
    }
  }
  if (!alive) {
    // A wait ran out: give every transfer this warp still has in flight a
    // bounded chance to land before the shared memory is reused.
    for (int i = 0; i < inflight; ++i) mbar_wait(mybar + (s + i) % S, s + i >= S ? parity ^ 1u : parity);
  }
  __syncwarp();
  if (lane == 0) {
    for (int s2 = 0; s2 < S; ++s2)
      asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(mybar + s2)) : "memory");
    if ((T.test_flags & 1u) && blockIdx.x == 0 && warp == 0)
      asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(&s_never)) : "memory");
  }
  // the page stream is done: the next kernel in the stream may be scheduled on SMs
  // this grid frees (it waits for this grid's completion before touching memory)
  if (sg.last) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if constexpr (LOGITS) return;                   // logits are written; nothing to merge

  // ---- merge the warps of this CTA
  constexpr int kSlots = NH * kGroupHeads;
  __shared__ float s_mx[W * kSlots];                    // each warp's running maxima (not in the stages)
#pragma unroll
  for (int h = 0; h < NH; ++h) {                        // each head's denominator over its 8 lanes
    lsum[h] += __shfl_xor_sync(kFull, lsum[h], 4);
    lsum[h] += __shfl_xor_sync(kFull, lsum[h], 8);
    lsum[h] += __shfl_xor_sync(kFull, lsum[h], 16);
    if (g == 0) s_mx[warp * kSlots + 4 * h + t] = mp2[h];
  }
  __syncthreads();                                      // every warp is out of its page loop: stages free
  // s_acc [W][kSlots][kAccPitch]: each warp's head sums (lanes t < 2 store the even
  // m-tiles, t >= 2 the odd ones: with a pitch of 132 floats one store touches 32
  // banks); s_l, s_f [W][kSlots]: denominator and the factor 2^(m_w - M) towards
  // the CTA's maximum M (s_M [kSlots]); the maxima m_w are in s_mx.
  float* s_acc = reinterpret_cast<float*>(smem);
  float* s_m = s_acc + W * kSlots * kAccPitch;
  float* s_l = s_m + W * kSlots;
  float* s_f = s_l + W * kSlots;
  float* s_M = s_f + W * kSlots;
  // Value-accumulator columns 2t, 2t + 1 of lane (g, t) hold heads 2 (t & 1) and
  // 2 (t & 1) + 1 of each group: the high weight parts for t < 2, the low parts
  // for t >= 2. Lanes t and t ^ 2 add them, so that both hold the head sums.
#pragma unroll
  for (int h = 0; h < NH; ++h) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float sum = acc[h][mt][c] + __shfl_xor_sync(kFull, acc[h][mt][c], 2);
        const int slot = 4 * h + 2 * (t & 1) + (c & 1), coord = 16 * mt + g + 8 * (c >> 1);
        if ((mt & 1) == (t >> 1)) s_acc[(warp * kSlots + slot) * kAccPitch + coord] = sum;
      }
    }
    if (g == 0) s_l[warp * kSlots + 4 * h + t] = lsum[h];
  }
  if (threadIdx.x < W * kSlots) {                       // one thread per (warp, head slot)
    const int w = threadIdx.x / kSlots, slot = threadIdx.x % kSlots;
    float M = kNegBig;
#pragma unroll
    for (int v = 0; v < W; ++v) M = fmaxf(M, s_mx[v * kSlots + slot]);
    s_f[w * kSlots + slot] = ex2(s_mx[w * kSlots + slot] - M);
    if (w == 0) s_M[slot] = M;
  }
  __syncthreads();
  constexpr int kRec = 132;                             // floats per (segment, head slot) record
  float* part = A.partial + static_cast<size_t>(sg.slot) * kSlots * kRec;
  for (int i = threadIdx.x; i < kSlots * 128; i += blockDim.x) {
    const int slot = i >> 7, coord = i & 127;
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) a = fmaf(s_acc[(w * kSlots + slot) * kAccPitch + coord], s_f[w * kSlots + slot], a);
    part[slot * kRec + coord] = a;
    if (coord == 0) {
      float l = 0.0f;
#pragma unroll
      for (int w = 0; w < W; ++w) l = fmaf(s_l[w * kSlots + slot], s_f[w * kSlots + slot], l);
      part[slot * kRec + 128] = s_M[slot];
      part[slot * kRec + 129] = l;
    }
  }
  // Publish the record: the barrier orders every thread's stores before thread 0's
  // acquire-release increment at GPU scope (release is cumulative over what
  // happens before it), and the CTA that takes the last ticket acquires all records.
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned ticket;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(ticket) : "l"(A.counters + pair) : "memory");
    s_last = (ticket == static_cast<unsigned>(sg.n_segs - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  if (threadIdx.x == 0) A.counters[pair] = 0u;    // every CTA has counted: ready for the next call

  // ---- last CTA of this (sequence, KV head): merge the records of all the pair's
  // segments, de-rotate, store. kParts warps share a head slot, each taking every
  // kParts-th record; lane l holds coordinates 4l .. 4l + 3 (the layout of the
  // inverse rotation). Records come straight from L2 (ld.global.cg), all of a
  // warp's loads in flight at once, in one pass: each part keeps its own running
  // maximum, and the parts meet in shared memory with their maxima.
  constexpr int kParts = W >= kSlots ? W / kSlots : 1;
  const float* pbase = A.partial + static_cast<size_t>(sg.first_slot) * kSlots * kRec;
  const int n_rec = sg.n_segs;
  float* s_v = reinterpret_cast<float*>(smem);           // [kParts][kSlots][kRec]: sums, l, max
  for (int sl0 = 0; sl0 < kSlots; sl0 += (kParts > 1 ? kSlots : W)) {
    const int slot = sl0 + (kParts > 1 ? warp % kSlots : warp);
    const int prt = kParts > 1 ? warp / kSlots : 0;
    if (slot < kSlots && prt < kParts) {                  // warp-uniform
      float M = kNegBig, v[4] = {0.f, 0.f, 0.f, 0.f}, lt = 0.0f;
      for (int c0 = prt; c0 < n_rec; c0 += 8 * kParts) {
        float4 x[8];
        float2 ml[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {                     // issue every load of the batch first
          const int c = c0 + k * kParts;
          const float* rec = pbase + (static_cast<size_t>(c < n_rec ? c : prt) * kSlots + slot) * kRec;
          x[k] = __ldcg(reinterpret_cast<const float4*>(rec) + lane);
          ml[k] = __ldcg(reinterpret_cast<const float2*>(rec + 128));
        }
        float bm = M;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (c0 + k * kParts < n_rec) bm = fmaxf(bm, ml[k].x);
        if (bm > M) {                                     // rescale what this part has so far
          const float r = ex2(M - bm);
          lt *= r;
          v[0] *= r; v[1] *= r; v[2] *= r; v[3] *= r;
          M = bm;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float f = c0 + k * kParts < n_rec ? ex2(ml[k].x - M) : 0.0f;
          lt = fmaf(ml[k].y, f, lt);
          v[0] = fmaf(x[k].x, f, v[0]); v[1] = fmaf(x[k].y, f, v[1]);
          v[2] = fmaf(x[k].z, f, v[2]); v[3] = fmaf(x[k].w, f, v[3]);
        }
      }
      float* mine = s_v + (prt * kSlots + slot) * kRec;
      reinterpret_cast<float4*>(mine)[lane] = make_float4(v[0], v[1], v[2], v[3]);
      if (lane == 0) {
        mine[128] = lt;
        mine[129] = M;
      }
    }
  }
  __syncthreads();
  const float4 sv = __ldg(reinterpret_cast<const float4*>(tab_sv) + lane);
  for (int slot = warp; slot < A.group; slot += W) {
    float v[4] = {0.f, 0.f, 0.f, 0.f}, lt = 0.0f, M = kNegBig;
#pragma unroll
    for (int q = 0; q < kParts; ++q) M = fmaxf(M, s_v[(q * kSlots + slot) * kRec + 129]);
#pragma unroll
    for (int q = 0; q < kParts; ++q) {
      const float* r = s_v + (q * kSlots + slot) * kRec;
      const float4 x = reinterpret_cast<const float4*>(r)[lane];
      const float f = ex2(r[129] - M);
      lt = fmaf(r[128], f, lt);
      v[0] = fmaf(x.x, f, v[0]); v[1] = fmaf(x.y, f, v[1]); v[2] = fmaf(x.z, f, v[2]); v[3] = fmaf(x.w, f, v[3]);
    }
    const float inv = lt > 0.0f ? 1.0f / lt : 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] *= inv;
    fwht128(v, lane);
    float4 o;
    o.x = v[0] * sv.x * kInvSqrtD;
    o.y = v[1] * sv.y * kInvSqrtD;
    o.z = v[2] * sv.z * kInvSqrtD;
    o.w = v[3] * sv.w * kInvSqrtD;
    const int qh = hk * A.group + slot;
    reinterpret_cast<float4*>(A.out + (static_cast<size_t>(b) * A.n_q + qh) * 128)[lane] = o;
  }
}

// The decode launch.
// Uniform mode: CTA i serves chunk i / n_pairs of pair i % n_pairs (chunks of ppc pages).
// Balanced mode (12 or 8 warps, see DecodeWarps): the pairs' pages are laid end to end, each
// non-empty pair preceded by seg_w "virtual" pages standing for its fixed cost
// (prologue, merge), and the line is cut into G equal shares, one per CTA (share of
// position y: ceil((y + 1) G / N) - 1). A CTA serves one segment per pair its share
// overlaps, one after the other.
template <int BK, int BV, int NH, int MODE, bool BAL>
__global__ void __launch_bounds__(DecodeWarps<NH, BAL>::value * 32, 1) decode_kernel(Tables T, DecodeArgs A) {
  // Launched as a programmatic dependent of the previous kernel in the stream: its
  // memory operations are complete and visible once the grid-dependency wait
  // returns. The uniform split waits inside the segment body, after loading the
  // context's constant tables; the balanced split reads the lengths first.
  if constexpr (BAL) asm volatile("griddepcontrol.wait;" ::: "memory");
  if constexpr (!BAL) {
    Segment sg;
    sg.pair = static_cast<int>(blockIdx.x % static_cast<unsigned>(A.n_pairs));
    const int chunk = static_cast<int>(blockIdx.x / static_cast<unsigned>(A.n_pairs));
    sg.p0 = chunk * A.ppc;
    sg.len = A.ppc;
    sg.slot = sg.pair * A.chunks + chunk;
    sg.first_slot = sg.pair * A.chunks;
    sg.n_segs = A.chunks;
    sg.last = true;
    decode_segment<BK, BV, NH, MODE, false>(T, A, sg);
  } else {
    extern __shared__ __align__(128) uint8_t smem[];
    int* s_vs = reinterpret_cast<int*>(smem + A.vs_off);     // [batch + 1]: virtual pages before sequence b
    int* s_ne = s_vs + A.batch + 1;                         // [batch + 1]: non-empty sequences before b
    __shared__ Segment s_sg;
    __shared__ long long s_n, s_g, s_x, s_hi;
    __shared__ int s_wsum[32], s_carry, s_more;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    // block-wide exclusive prefix of v over [0, n) into dst[0..n], blockDim values at a time
    auto block_scan = [&](int n, auto value, int* dst) {
      if (threadIdx.x == 0) s_carry = 0;
      __syncthreads();
      for (int base = 0; base < n; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const int v = i < n ? value(i) : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFull, x, o);
          if (lane >= o) x += y;
        }
        if (lane == 31) s_wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
          int w = lane < nw ? s_wsum[lane] : 0;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, w, o);
            if (lane >= o) w += y;
          }
          if (lane < nw) s_wsum[lane] = w;              // inclusive over warps
        }
        __syncthreads();
        const int incl = x + (warp > 0 ? s_wsum[warp - 1] : 0);
        if (i < n) dst[i] = s_carry + incl - v;
        __syncthreads();
        if (threadIdx.x == 0) s_carry += s_wsum[nw - 1];
        __syncthreads();
      }
      if (threadIdx.x == 0) dst[n] = s_carry;
      __syncthreads();
    };
    // virtual length of sequence b: its pages plus seg_w, or 0 when empty
    block_scan(A.batch, [&](int bb) {
      const int L = min(max(A.seq_lens[bb], 0), A.max_seq_len);
      const int pg = (L + kPage - 1) / kPage;
      return pg > 0 ? pg + A.seg_w : 0;
    }, s_vs);
    block_scan(A.batch, [&](int bb) { return s_vs[bb + 1] > s_vs[bb] ? 1 : 0; }, s_ne);
    if (threadIdx.x == 0) {
      const long long n = static_cast<long long>(A.n_kv) * s_vs[A.batch];
      s_n = n;
      s_g = min(static_cast<long long>(A.shares), max(1LL, (n + A.min_share - 1) / A.min_share));
    }
    __syncthreads();
    // pairs of empty sequences: zero outputs (nothing attends; logits are left alone)
    if (MODE != 2) {
      for (int p = blockIdx.x; p < A.n_pairs; p += gridDim.x) {
        const int bb = p / A.n_kv, hk = p % A.n_kv;
        if (s_vs[bb + 1] != s_vs[bb]) continue;
        for (int i = threadIdx.x; i < A.group * 128; i += blockDim.x)
          A.out[(static_cast<size_t>(bb) * A.n_q + hk * A.group) * 128 + i] = 0.0f;
      }
    }
    const long long n = s_n, gg = s_g;
    if (n == 0) return;
    // the pair holding virtual position y: its ordinal among the pairs of non-empty
    // sequences (consecutive along the line), first virtual page, virtual length
    struct At { int p, vl; long long vp; };
    auto pair_at = [&](long long y) {
      int bl = 0, bh = A.batch;                       // n_kv s_vs[bl] <= y < n_kv s_vs[bh]
      while (bh - bl > 1) {
        const int mid = (bl + bh) >> 1;
        if (static_cast<long long>(A.n_kv) * s_vs[mid] <= y) bl = mid; else bh = mid;
      }
      At r;
      r.vl = s_vs[bl + 1] - s_vs[bl];                 // > 0: the largest such bl is a non-empty sequence
      const long long vb = static_cast<long long>(A.n_kv) * s_vs[bl];
      const int hk = static_cast<int>((y - vb) / r.vl);
      r.p = s_ne[bl] * A.n_kv + hk;
      r.vp = vb + static_cast<long long>(hk) * r.vl;
      return r;
    };
    auto share_lo = [&](long long i) { return i * n / gg; };
    if (static_cast<long long>(blockIdx.x) >= gg) return;
    // This CTA serves share blockIdx.x: every pair it overlaps, one segment each,
    // in order. The segment of share i in the pair of ordinal o writes record
    // i + o, unique because consecutive pairs share at most one share; a pair's
    // records run from (its first share) + o over its shares.
    if (threadIdx.x == 0) {
      s_x = share_lo(blockIdx.x);
      s_hi = share_lo(blockIdx.x + 1);
    }
    auto next_segment = [&]() {                     // thread 0
      auto cta_of = [&](long long y) { return static_cast<int>(((y + 1) * gg + n - 1) / n) - 1; };
      s_more = 0;
      long long x = s_x;
      const long long hi = s_hi;
      while (x < hi) {
        const At a = pair_at(x);
        const long long r0 = a.vp + A.seg_w, s0 = max(x, r0), s1 = min(hi, a.vp + a.vl);
        x = a.vp + a.vl;
        if (s1 > s0) {
          const int t = a.p / A.n_kv, hk = a.p % A.n_kv;
          int bl = 0, bh = A.batch;                   // the t-th non-empty sequence: largest bl, s_ne[bl] <= t
          while (bh - bl > 1) {
            const int mid = (bl + bh) >> 1;
            if (s_ne[mid] <= t) bl = mid; else bh = mid;
          }
          Segment sg;
          sg.pair = bl * A.n_kv + hk;
          sg.p0 = static_cast<int>(s0 - r0);
          sg.len = static_cast<int>(s1 - s0);
          const int f = cta_of(r0), l = cta_of(r0 + (a.vl - A.seg_w) - 1);
          sg.slot = static_cast<int>(blockIdx.x) + a.p;
          sg.first_slot = f + a.p;
          sg.n_segs = l - f + 1;
          sg.last = x >= hi;
          if (sg.len > A.ppc) {                       // the block-table window is sized by the host
            set_error(T.err, TQ_DEV_BAD_LENGTH);
            sg.len = A.ppc;
          }
          s_sg = sg;
          s_more = 1;
          break;
        }
      }
      s_x = x;
    };
    if (threadIdx.x == 0) next_segment();
    __syncthreads();
    while (s_more) {
      decode_segment<BK, BV, NH, MODE, true>(T, A, s_sg);
      __syncthreads();
      if (threadIdx.x == 0) next_segment();
      __syncthreads();
    }
  }
}

template <int BK, int BV, int NH, int MODE, bool BAL>
cudaError_t launch_decode_tb(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s) {
  constexpr int W = DecodeWarps<NH, BAL>::value;
  constexpr int kBlock = block_bytes_of(BK, BV);
  constexpr int S = decode_stages(W, kBlock);
  // main loop: stages, barriers, prologue scratch, the chunk's block-table window
  const size_t pipe = static_cast<size_t>(W) * S * kBlock + W * S * sizeof(uint64_t) + sizeof(Prologue<NH>) +
                      ((static_cast<size_t>(a.ppc) * 4 + 15) & ~static_cast<size_t>(15));
  // CTA merge: every warp's head sums [W][slots][kAccPitch] and softmax state
  // [3][W][slots] + [slots]; the final merge reuses the same space for at most
  // max(W, slots) records of 132 floats
  constexpr size_t kSlotsL = static_cast<size_t>(NH) * kGroupHeads;
  const size_t merge = (W * kSlotsL * kAccPitch + 3 * W * kSlotsL + kSlotsL) * 4;
  static_assert((W > static_cast<int>(kSlotsL) ? W : kSlotsL) * 132 <= W * kSlotsL * kAccPitch, "final merge space");
  const size_t base = ((pipe > merge ? pipe : merge) + 15) & ~static_cast<size_t>(15);
  // balanced mode: two [batch + 1] prefixes of the split, after everything else
  const size_t smem = base + (BAL ? (2 * static_cast<size_t>(a.batch) + 2) * 4 : 0);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  DecodeArgs args = a;
  args.vs_off = static_cast<int>(base);
  auto fn = decode_kernel<BK, BV, NH, MODE, BAL>;
  static size_t configured = 0;     // raise the shared-memory limit once per instantiation
  if (configured < smem) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the launch with the previous kernel's tail
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, T, args);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int BK, int BV>
cudaError_t launch_prefill_t(const Tables& t, const void* k, const void* v, int dtype, int n_tokens, int n_kv,
                             const int32_t* block_table, int start_pos, void* cache, int64_t n_pages,
                             cudaStream_t s) {
  const int first = start_pos / kPage, last = (start_pos + n_tokens - 1) / kPage;
  const int tiles = (last - first + 1) * n_kv;
  const int elem = dtype == TQ_F32 ? 4 : 2;
  if constexpr (BK != 8) {
    if (elem == 2) {                      // TurboQuant keys from 16-bit inputs: z = S u on tcgen05
      auto fn = quantize_prefill_tc_kernel<BK, BV>;
      static int max_blocks = 0;
      if (max_blocks == 0) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kTcSmem));
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        max_blocks = sms;                 // one CTA per SM (its shared memory and all tensor memory)
      }
      int blocks = (tiles + kTcWarps - 1) / kTcWarps;
      if (blocks > max_blocks) blocks = max_blocks;
      CUtensorMap tmk, tmv;
      cudaError_t e = encode_kv_tensor_map(&tmk, k, dtype, n_tokens, n_kv);
      if (e == cudaSuccess) e = encode_kv_tensor_map(&tmv, v, dtype, n_tokens, n_kv);
      if (e != cudaSuccess) return e;
      fn<<<blocks, kTcWarps * 32, kTcSmem, s>>>(t, tmk, tmv, dtype, n_tokens, n_kv, block_table, start_pos,
                                                static_cast<uint8_t*>(cache), n_pages);
      return cudaGetLastError();
    }
  }
  const int warps = 8;
  int blocks = (tiles + warps - 1) / warps;
  const size_t smem = pf_smem(warps, elem);
  auto fn = quantize_prefill_kernel<BK, BV>;
  // grid limit = resident CTAs, worked out once per instantiation and shared-memory size
  static size_t configured = 0;
  static int max_blocks = 0;
  if (configured != smem) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, warps * 32, smem) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    max_blocks = sms * per_sm;
    configured = smem;
  }
  if (blocks > max_blocks) blocks = max_blocks;
  fn<<<blocks, warps * 32, smem, s>>>(t, k, v, dtype, n_tokens, n_kv, block_table, start_pos,
                                      static_cast<uint8_t*>(cache), n_pages);
  return cudaGetLastError();
}

}  // namespace

// One instantiation unit per (key bits, value bits): decode launches of every
// group size, mode and split, and the prefill launch.
#define TQ_FOR_EACH_BITS(X) X(2, 2) X(2, 3) X(2, 4) X(3, 2) X(3, 3) X(3, 4) \
                               X(4, 2) X(4, 3) X(4, 4) X(8, 2) X(8, 3) X(8, 4)
#define TQ_DECLARE_BITS(BK, BV)                                                                      \
  cudaError_t decode_bits_##BK##_##BV(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s,    \
                                      int mode);                                                           \
  cudaError_t prefill_bits_##BK##_##BV(const Tables& t, const void* k, const void* v, int dtype,            \
                                       int n_tokens, int n_kv, const int32_t* block_table, int start_pos,   \
                                       void* cache, int64_t n_pages, cudaStream_t s);
TQ_FOR_EACH_BITS(TQ_DECLARE_BITS)

}  // namespace tq
