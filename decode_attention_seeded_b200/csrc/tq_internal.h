// Internal interface between the host library (tq_host.cpp) and the CUDA
// kernels (tq_kernels.cu). Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace tq {

constexpr int kHeadDim = 128;
constexpr int kQjlRows = 128;
constexpr int kPage = 16;

// Everything a kernel needs to know about the codebooks and seeded tables.
// Passed by value as a kernel parameter (lives in the constant bank).
struct Tables {
  int key_bits = 0, value_bits = 0;
  int block_bytes = 0;          // bytes of one (page, KV head) block
  int k_exp = 0;                // key centroids * 2^k_exp are exact int16 values
  float thr_k[16];              // 2^b - 1 thresholds (rest unused)
  float thr_v[16];
  float cen_k[16];              // fp16 centroids widened to fp32
  float cen_v[16];
  uint32_t kq_hi[4];            // key centroid int16 split hi*256 + lo, hi bytes (16 entries)
  uint32_t kq_lo[4];            //   ... lo bytes (signed, in [-128, 127])
  uint32_t v_lo[4];             // value centroid fp16 low bytes (16 entries)
  uint32_t v_hi[4];             //   ... high bytes
  const float* signs_k = nullptr;     // device [128], +-1
  const float* signs_v = nullptr;     // device [128], +-1
  const uint16_t* sketch_t = nullptr; // device fp16 bits of S^T, [128 (d)][128 (m)]
  const uint16_t* sketch_m = nullptr;  // device fp16 bits of M = S R_K, high then low parts, as m16n8k16 A
                                       //   fragments [2][8 w][8 ks][32 lane][4 reg][2]
  float m_rownorm = 0.0f;             // max over rows r of |M_r| (bounds |p_r| <= |M_r| |q|)
  const uint16_t* sketch_qb = nullptr;  // device fp16 bits of S as prefill B fragments [8 ks][16 nt][32 lane][2 reg][2]
  const uint16_t* sketch_umma = nullptr;  // device fp16 bits of S as the prefill's tensor-core B operand (32 KB)
  unsigned* err = nullptr;            // device error word
  unsigned test_flags = 0;            // TQ_TEST_* bits (tq_set_test_flags)
};

// Workspace carve-up for one decode call; all offsets in bytes, 256-aligned.
// Decode grid: one CTA per (chunk, sequence x KV head pair), CTA index =
// chunk * n_pairs + pair, one resident CTA per SM.
constexpr int kMinChunkPages = 16;
constexpr int kMaxChunkPages = 8192;
constexpr int kMinShare = 48;          // balanced mode: least pages per CTA share
constexpr int kMaxBalancedBatch = 4096;  // balanced mode keeps a [batch + 1] prefix in shared memory
struct DecodePlan {
  int batch, n_q, n_kv, group, n_hg;  // n_hg = ceil(group / 4) groups of 4 query heads
  int n_pairs;                         // batch * n_kv
  int max_pages, pages_per_chunk, chunks;
  // Balanced mode (chosen when uniform chunks per pair would leave SMs idle): `grid`
  // CTAs take equal shares of all pages, each pair counted with seg_w extra pages for
  // its fixed cost; pages_per_chunk then bounds one CTA's share (its block-table window).
  int balanced, grid, seg_w, min_share, shares;
  size_t off_partial, off_counter, total;
};

DecodePlan make_plan(int batch, int n_q, int n_kv, int max_seq_len, int sm_count);

cudaError_t launch_quantize_append(const Tables& t, const void* k, const void* v, int dtype,
                                   int n_tokens, int n_kv, const int64_t* slots, void* cache,
                                   int64_t n_pages, cudaStream_t s);
cudaError_t launch_quantize_prefill(const Tables& t, const void* k, const void* v, int dtype,
                                    int n_tokens, int n_kv, const int32_t* block_table,
                                    int start_pos, void* cache, int64_t n_pages, cudaStream_t s);
cudaError_t launch_decode(const Tables& t, const DecodePlan& plan, const void* q, int q_dtype,
                          const void* cache, int64_t n_pages, const int32_t* block_tables,
                          int max_pages_per_seq, const int32_t* seq_lens, int max_seq_len,
                          float scale, float* out, void* workspace, float sparse_tau, cudaStream_t s);

cudaError_t launch_logits(const Tables& t, const DecodePlan& plan, const void* q, int q_dtype, const void* cache,
                          int64_t n_pages, const int32_t* block_tables, int max_pages_per_seq,
                          const int32_t* seq_lens, int max_seq_len, float scale, float* logits,
                          int64_t logits_stride, cudaStream_t s);

cudaError_t launch_decode_step(const Tables& t, const DecodePlan& plan, const void* k_new, const void* v_new,
                               int kv_dtype, const void* q, int q_dtype, void* cache, int64_t n_pages,
                               const int32_t* block_tables, int max_pages_per_seq, const int32_t* seq_lens,
                               int max_seq_len, float scale, float* out, void* workspace, float sparse_tau,
                               cudaStream_t s);

// Device address (current device) of the fixed decode scratch used by
// tq_decode_attention_noalloc; kNoAllocScratchBytes bytes, 256-byte aligned.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
cudaError_t noalloc_scratch(void** ptr);

}  // namespace tq
