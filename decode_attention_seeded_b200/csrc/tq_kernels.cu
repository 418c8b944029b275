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
// written out independently by the oracle's layout module):
//   [K codes 32 lanes x 8*bk B][sign bits 32 x 8 B][V codes 32 x 8*bv B][norms 96 B]
// or, with q8_0 keys (bk = 8):
//   [int8 K values 32 lanes x 64 B][fp16 block scales 128 B][V codes 32 x 8*bv B][V norms 32 B]
// Lane chunks are laid out so that lane (g, t) = (lane>>2, lane&3) of a warp
// finds in its own chunk exactly the bits of its mma.sync fragments:
//   keys:   A operand of m16n8k32 (m = token: g and g + 8, k = coordinate)
//   signs:  A operand of m16n8k32 (m = token, k = sketch row)
//   values: A operand of m16n8k16 (m = coordinate, k = token)

#include "tq_kernels.cuh"

namespace tq {
namespace {

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
    if (T.key_bits == 8) {
      store_key_q8(blk, tau, x, lane);
    } else {
      quantize_vector(x, T.signs_k, s_tab, s_tab + 16, T.key_bits, s_sk, true, lane, o);
      store_key_token(blk, tau, T.key_bits, o, lane);
      if (lane == 0) {
        store_norm(blk, T.key_bits, T.value_bits, 0, tau, o.norm);
        store_norm(blk, T.key_bits, T.value_bits, 1, tau, o.gamma);
      }
    }
    load_row4(v, static_cast<size_t>(tok) * n_kv + h, dtype, lane, x);
    quantize_vector(x, T.signs_v, s_tab + 32, s_tab + 48, T.value_bits, nullptr, false, lane, o);
    store_value_token(blk, tau, T.key_bits, T.value_bits, o, lane);
    if (lane == 0) store_norm(blk, T.key_bits, T.value_bits, 2, tau, o.norm);
  }
}

// ---- fixed scratch for callers that cannot allocate device memory ----------
// Split-K records and completion counters of tq_decode_attention_noalloc. One
// copy per device, zero when the module is loaded; every decode that runs to the
// end leaves the counters at zero again.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

DecodeArgs decode_args(const DecodePlan& plan, const void* q, int q_dtype, float scale, const void* cache,
                       int64_t n_pages, const int32_t* block_tables, int max_pages_per_seq, const int32_t* seq_lens,
                       int max_seq_len, float* out, void* workspace, float sparse_tau) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeArgs a{};
  a.q = q;
  a.q_dtype = q_dtype;
  a.scale = scale;
  a.cache = static_cast<uint8_t*>(const_cast<void*>(cache));
  a.n_pages = n_pages;
  a.block_tables = block_tables;
  a.max_pages_per_seq = max_pages_per_seq;
  a.seq_lens = seq_lens;
  a.max_seq_len = max_seq_len;
  a.partial = ws ? reinterpret_cast<float*>(ws + plan.off_partial) : nullptr;
  a.counters = ws ? reinterpret_cast<unsigned*>(ws + plan.off_counter) : nullptr;
  a.out = out;
  a.n_kv = plan.n_kv;
  a.n_q = plan.n_q;
  a.group = plan.group;
  a.n_hg = plan.n_hg;
  a.chunks = plan.chunks;
  a.ppc = plan.pages_per_chunk;
  a.n_pairs = plan.n_pairs;
  a.batch = plan.batch;
  a.balanced = plan.balanced;
  a.seg_w = plan.seg_w;
  a.min_share = plan.min_share;
  a.shares = plan.shares;
  a.sparse = sparse_tau > 0.0f ? 1 : 0;
  a.sparse_log2 = sparse_tau > 0.0f ? log2f(sparse_tau) : 0.0f;
  return a;
}


// Decode dispatch over the (key bits, value bits) instantiation units.
cudaError_t dispatch_bits(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s, int mode) {
#define TQ_CASE(BK, BV) \
  if (T.key_bits == BK && T.value_bits == BV) return decode_bits_##BK##_##BV(T, a, grid, s, mode);
  TQ_FOR_EACH_BITS(TQ_CASE)
#undef TQ_CASE
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t noalloc_scratch(void** ptr) { return cudaGetSymbolAddress(ptr, g_noalloc_scratch); }

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
#define TQ_CASE(BK, BV)                                                                                       \
  if (t.key_bits == BK && t.value_bits == BV)                                                                 \
    return prefill_bits_##BK##_##BV(t, k, v, dtype, n_tokens, n_kv, block_table, start_pos, cache, n_pages, s);
  TQ_FOR_EACH_BITS(TQ_CASE)
#undef TQ_CASE
  return cudaErrorNotSupported;
}

cudaError_t launch_decode(const Tables& t, const DecodePlan& plan, const void* q, int q_dtype,
                          const void* cache, int64_t n_pages, const int32_t* block_tables,
                          int max_pages_per_seq, const int32_t* seq_lens, int max_seq_len, float scale,
                          float* out, void* workspace, float sparse_tau, cudaStream_t s) {
  const DecodeArgs a = decode_args(plan, q, q_dtype, scale, cache, n_pages, block_tables, max_pages_per_seq,
                                   seq_lens, max_seq_len, out, workspace, sparse_tau);
  return dispatch_bits(t, a, dim3(plan.grid), s, 0);
}

cudaError_t launch_logits(const Tables& t, const DecodePlan& plan, const void* q, int q_dtype, const void* cache,
                          int64_t n_pages, const int32_t* block_tables, int max_pages_per_seq,
                          const int32_t* seq_lens, int max_seq_len, float scale, float* logits,
                          int64_t logits_stride, cudaStream_t s) {
  DecodeArgs a = decode_args(plan, q, q_dtype, scale, cache, n_pages, block_tables, max_pages_per_seq, seq_lens,
                             max_seq_len, nullptr, nullptr, 0.0f);
  a.logits = logits;
  a.logits_stride = logits_stride;
  return dispatch_bits(t, a, dim3(plan.grid), s, 2);
}

cudaError_t encode_kv_tensor_map(CUtensorMap* map, const void* base, int dtype, int n_tokens, int n_kv) {
  using Encode = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static const Encode encode = []() -> Encode {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<Encode>(fn);
  }();
  if (!encode) return cudaErrorNotSupported;
  if (n_tokens < 1 || n_kv < 1 || (reinterpret_cast<uintptr_t>(base) & 15u)) return cudaErrorInvalidValue;
  const cuuint64_t dims[4] = {64, 2, static_cast<cuuint64_t>(n_kv), static_cast<cuuint64_t>(n_tokens)};
  const cuuint64_t strides[3] = {128, 256, 256ull * static_cast<cuuint64_t>(n_kv)};   // bytes, dims 1..3
  const cuuint32_t box[4] = {64, 2, 1, 16};
  const cuuint32_t step[4] = {1, 1, 1, 1};
  const CUresult r = encode(map, dtype == TQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                            4, const_cast<void*>(base), dims, strides, box, step, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_decode_step(const Tables& t, const DecodePlan& plan, const void* k_new, const void* v_new,
                               int kv_dtype, const void* q, int q_dtype, void* cache, int64_t n_pages,
                               const int32_t* block_tables, int max_pages_per_seq, const int32_t* seq_lens,
                               int max_seq_len, float scale, float* out, void* workspace, float sparse_tau,
                               cudaStream_t s) {
  DecodeArgs a = decode_args(plan, q, q_dtype, scale, cache, n_pages, block_tables, max_pages_per_seq, seq_lens,
                             max_seq_len, out, workspace, sparse_tau);
  a.k_new = k_new;
  a.v_new = v_new;
  a.kv_dtype = kv_dtype;
  return dispatch_bits(t, a, dim3(plan.grid), s, 1);
}

}  // namespace tq
