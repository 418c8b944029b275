/*
 * tq.h -- C ABI of the B200 (sm_100a) compressed-KV cache library (libtq.so).
 *
 * TurboQuant-style KV-cache compression and decode attention, as described on
 * the pages "TurboQuant : 6x moins de cache, jusqu'a 8x plus rapide"
 * (leviatan.io: "Principe de quantification sans calibration", "Benchmarks de
 * memoire") and the wis-web.com llama.cpp-fork post (paragraphs on PolarQuant
 * and on QJL): each K/V vector is rotated by a seeded random Walsh-Hadamard
 * transform, its L2 norm is kept, every rotated coordinate is coded with a fixed
 * b-bit Lloyd-Max codebook of the known post-rotation law (no per-block scales),
 * and keys add one QJL sign bit per row of a seeded Gaussian sketch plus the
 * residual norm. Decode attention reads the packed cache directly.
 *
 * Conventions for every call:
 *   - Pointers marked (device) are CUDA device pointers; (host) are host memory.
 *     The caller owns every buffer it passes; the library owns only the context
 *     and the small device tables it allocates in tq_create / tq_init_*.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream). Nothing throws across the ABI.
 *   - Arguments the host can check are checked before any launch; a bad one
 *     returns TQ_ERR_INVALID_ARG / TQ_ERR_UNSUPPORTED and enqueues nothing.
 *   - Decode calls (tq_decode_attention, tq_decode_step, tq_decode_logits,
 *     tq_decode_attention_noalloc) launch as programmatic dependents of the
 *     previous work in the stream: their kernel waits for it to complete before
 *     touching memory, so stream order holds as usual. They also allow the next
 *     kernel to launch early, once their page stream is done. A caller kernel
 *     launched with programmatic stream serialization must therefore wait for its
 *     grid dependency (cudaGridDependencySynchronize) before it reads their
 *     outputs, as programmatic dependent launch requires anyway. Kernels launched
 *     without that attribute see ordinary stream order.
 *   - Faults detected on the device (a page id or slot out of range, a wait
 *     that ran out) are not traps: the kernel skips the access, records a code
 *     in the context's device error word and finishes. tq_get_device_error
 *     reads (and clears) it.
 *   - Fixed geometry in this version: head_dim d = 128, QJL rows m = 128,
 *     16 tokens per page, key/value code widths 2, 3 or 4 bits.
 *   - Asymmetric cache (key_bits = 8): keys are kept in q8_0 blocks instead of
 *     TurboQuant codes (wis-web.com llama.cpp-fork post, first finding: values
 *     tolerate 2-3 bits when keys stay in q8_0). Each key is cut into 4 blocks of
 *     32 coordinates; a block stores d = max|x| / 127 as fp16 and rint(x / d) as
 *     int8 (0 for an all-zero block); no rotation and no QJL bits. Values are
 *     TurboQuant codes as above. Decode uses the raw query against the int8
 *     values, scaled per block.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,      /* null pointer, bad size, inconsistent shapes      */
  TQ_ERR_UNSUPPORTED = 2,      /* geometry or bit width this build does not serve  */
  TQ_ERR_WORKSPACE = 3,        /* workspace too small or misaligned                 */
  TQ_ERR_CUDA = 4,             /* a CUDA runtime call failed                         */
  TQ_ERR_DEVICE = 5,           /* device error word was set (see TQ_DEV_* bits)      */
  TQ_ERR_NOT_INITIALIZED = 6   /* tq_init_rotation / tq_init_codebooks not called    */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* Bits of the device error word. */
#define TQ_DEV_BAD_SLOT     0x1u   /* quantize: slot id outside the page pool           */
#define TQ_DEV_BAD_PAGE     0x2u   /* decode: block-table entry outside the page pool    */
#define TQ_DEV_TIMEOUT      0x4u   /* a bounded wait on a TMA transfer ran out          */
#define TQ_DEV_BAD_LENGTH   0x8u   /* decode: seq_len above max_seq_len or negative     */

typedef struct tq_ctx tq_ctx;   /* opaque; owned by the library */
typedef void* tq_stream;        /* cudaStream_t */

/* Library version (major*10000 + minor*100 + patch) and status text. */
int tq_version(void);
const char* tq_status_string(tq_status s);

/*
 * Create a context on CUDA device `device`. head_dim, qjl_rows and page_size
 * must be 128, 128 and 16. Allocates a few tens of KB of device tables and the
 * device error word. *out receives the context (NULL on error).
 */
tq_status tq_create(tq_ctx** out, int head_dim, int qjl_rows, int page_size, int device);
void tq_destroy(tq_ctx* ctx);

/*
 * Seeded rotation and sketch (pages: PolarQuant paragraph -- random
 * Walsh-Hadamard rotation; QJL paragraph -- random projection signs).
 * D_K, D_V in {+1,-1}^d: entry i is -1 iff the top bit of SplitMix64 output i
 * of seed_k / seed_v is set. S (m x d): entry r*d+c is the cosine branch of
 * Box-Muller on SplitMix64 outputs 2(r*d+c), 2(r*d+c)+1 of seed_s, rounded to
 * fp16. Computed on the host, copied to the device on `stream`.
 */
tq_status tq_init_rotation(tq_ctx* ctx, uint64_t seed_k, uint64_t seed_v, uint64_t seed_s,
                           tq_stream stream);

/*
 * Lloyd-Max codebooks (pages: the coordinate law after the rotation is known in
 * advance, so no quantisation constants are stored; turbo2/3/4 = 2/3/4 bits).
 * Law: one coordinate of a uniform point on the unit sphere, density
 * proportional to (1-t^2)^((d-3)/2). Centroids are rounded to fp16; thresholds
 * are midpoints of adjacent stored centroids. key_bits in {2,3,4,8} (8: q8_0
 * keys, no key codebook), value_bits in {2,3,4}.
 */
tq_status tq_init_codebooks(tq_ctx* ctx, int key_bits, int value_bits, tq_stream stream);

/* Bytes of one (page, KV head) block and of one physical page (all KV heads):
 * block = 16 * (16*key_bits + 16 + 4 + 16*value_bits + 2); with q8_0 keys
 * block = 16 * (128 + 8 + 16*value_bits + 2). 0 if not initialised. */
size_t tq_block_bytes(const tq_ctx* ctx);
size_t tq_page_bytes(const tq_ctx* ctx, int n_kv_heads);

/*
 * Quantize and append tokens into the paged cache.
 *   k, v          (device) [n_tokens, n_kv_heads, 128] contiguous, dtype fp32 / bf16 / fp16.
 *   slot_mapping  (device) int64 [n_tokens]: physical_page * 16 + offset of each token.
 *                 Slots must be distinct within one call; any order is allowed.
 *   cache         (device) n_cache_pages physical pages of tq_page_bytes() bytes each,
 *                 page-major then KV-head-major; 16-byte aligned.
 * For each (token, head): n = |x|, y = R x / n, codes = cell(y); keys also
 * u = y - c[code], gamma = n |u|, sign bits [S u >= 0]; stored per the block layout.
 * Slot ids outside [0, 16*n_cache_pages) set TQ_DEV_BAD_SLOT and are skipped.
 */
tq_status tq_quantize_append(tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                             int n_tokens, int n_kv_heads, const int64_t* slot_mapping,
                             void* cache, int64_t n_cache_pages, tq_stream stream);

/*
 * Quantize a contiguous run of one sequence's tokens (a prefill or a chunk of
 * one): logical positions [start_pos, start_pos + n_tokens) go to the pages
 * named by block_table (device int32 [>= ceil((start_pos+n_tokens)/16)]).
 * Same arithmetic as tq_quantize_append; whole pages are written with full-width
 * stores, partial pages are merged with what they already hold. k and v must be
 * 16-byte aligned (their rows are staged in shared memory by bulk copies);
 * otherwise TQ_ERR_INVALID_ARG.
 */
tq_status tq_quantize_prefill(tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                              int n_tokens, int n_kv_heads, const int32_t* block_table,
                              int start_pos, void* cache, int64_t n_cache_pages, tq_stream stream);

/*
 * Workspace for tq_decode_attention / tq_decode_step (caller-allocated device
 * memory, 256-byte aligned). It holds split-K partials and one completion
 * counter per (sequence, KV head). Zero-fill it once before its first use
 * (e.g. cudaMemsetAsync); every call leaves the counters at zero again. Calls
 * that share a workspace must not run concurrently.
 */
size_t tq_decode_workspace_bytes(const tq_ctx* ctx, int batch, int n_q_heads, int n_kv_heads,
                                 int max_seq_len);

/*
 * Decode attention over the compressed paged GQA cache.
 *   q             (device) [batch, n_q_heads, 128], dtype fp32 / bf16 / fp16.
 *   cache         (device) as written by tq_quantize_*.
 *   block_tables  (device) int32 [batch, max_pages_per_seq]: physical page of each logical page.
 *   seq_lens      (device) int32 [batch]: cached tokens per sequence, 0 <= len <= max_seq_len.
 *   max_seq_len   host-side upper bound of seq_lens (sizes the split-K grid).
 *   scale         softmax scale; 0 selects 1/sqrt(128).
 *   out           (device) float32 [batch, n_q_heads, 128].
 * Query head h reads KV head h / (n_q_heads / n_kv_heads). Per token t:
 *   l_t = scale * ( |k_t| <R_K q, c[code_t]> + |r_t| sqrt(pi/2)/m <S R_K q, sign(S r_t)> ),
 * softmax over t, a = sum_t w_t |v_t| c_v[code_v,t], out = R_V^T a. A sequence of
 * length 0 yields zeros. Block-table entries outside the pool set TQ_DEV_BAD_PAGE
 * (that page is skipped).
 */
tq_status tq_decode_attention(tq_ctx* ctx, const void* q, tq_dtype q_dtype, const void* cache,
                              int64_t n_cache_pages, const int32_t* block_tables,
                              int max_pages_per_seq, const int32_t* seq_lens, int batch,
                              int n_q_heads, int n_kv_heads, int max_seq_len, float scale,
                              float* out, void* workspace, size_t workspace_bytes,
                              tq_stream stream);

/*
 * One decode step: append one new token per sequence, then attend. For each
 * sequence b with seq_lens[b] > 0, the key/value k_new[b], v_new[b]
 * ([batch, n_kv_heads, 128], dtype kv_dtype) are quantized exactly as by
 * tq_quantize_append and stored at logical position seq_lens[b] - 1 (page
 * block_tables[b][(seq_lens[b]-1)/16]); then q is attended over positions
 * [0, seq_lens[b]) exactly as by tq_decode_attention, so the new token is seen.
 * Same arguments, workspace and error behaviour as tq_decode_attention. The
 * attention kernel starts streaming the cache while the new token is being
 * quantized (every page except each sequence's last one).
 */
tq_status tq_decode_step(tq_ctx* ctx, const void* k_new, const void* v_new, tq_dtype kv_dtype,
                         const void* q, tq_dtype q_dtype, void* cache, int64_t n_cache_pages,
                         const int32_t* block_tables, int max_pages_per_seq, const int32_t* seq_lens,
                         int batch, int n_q_heads, int n_kv_heads, int max_seq_len, float scale, float* out,
                         void* workspace, size_t workspace_bytes, tq_stream stream);

/*
 * Attention logits only (leviatan.io page, sections "Accélération jusqu'à 8× du
 * calcul d'attention" and "Comparaison 4-bit vs 32-bit": the logit computation on
 * compressed keys against full-precision keys). Writes, for every sequence b,
 * query head h and cached position t < seq_lens[b],
 *   logits[(b * n_q_heads + h) * logits_stride + t]
 *     = scale * ( |k_t| <R_K q, c[code_t]> + |r_t| sqrt(pi/2)/m <S R_K q, sign(S r_t)> )
 * (natural-log units, float32), exactly the logits tq_decode_attention softmaxes.
 * Positions >= seq_lens[b] are not written. Only the key codes, sign bits and
 * norms of each block are read. logits: (device) float32, logits_stride >=
 * max_seq_len. No workspace. Other arguments and errors as tq_decode_attention.
 */
tq_status tq_decode_logits(tq_ctx* ctx, const void* q, tq_dtype q_dtype, const void* cache,
                           int64_t n_cache_pages, const int32_t* block_tables, int max_pages_per_seq,
                           const int32_t* seq_lens, int batch, int n_q_heads, int n_kv_heads, int max_seq_len,
                           float scale, float* logits, int64_t logits_stride, tq_stream stream);

/*
 * Sparse V (wis-web.com llama.cpp-fork post, third finding: decoding that skips
 * the V positions with a low attention weight). With tau > 0, every later decode
 * call of this context (tq_decode_attention, tq_decode_step and the no-alloc
 * variant) gives no value contribution to a position whose softmax weight is
 * below tau times the largest weight; the softmax denominator still covers every
 * position, and a page whose values are all skipped costs no value work. The
 * comparison is made against the largest weight seen so far by the warp that
 * reads the page (never more than the largest overall), so a call skips a subset
 * of the positions the definition allows; the output differs from the dense one
 * by at most the sum over skipped positions of w_t ||v_t c_t||. The pages give no
 * threshold. tau = 0 (the default) is dense attention; tau in [0, 1], else
 * TQ_ERR_INVALID_ARG. Host-side setting; no device work.
 */
tq_status tq_set_sparse_v(tq_ctx* ctx, float tau);

/*
 * tq_decode_attention without a caller workspace. The pages have no counterpart
 * to this call: it is a library convenience, computing exactly what
 * tq_decode_attention computes, with the same arguments minus the workspace.
 *
 * Who needs it: callers that cannot hand the library device memory of their
 * own -- a host program that reaches the GPU only through this C ABI and has no
 * CUDA allocator binding, a runtime that has reserved its whole device budget
 * in a pool it does not lend out, or a decode path where an allocation that
 * can fail or stall is not acceptable. Instead of a workspace, the call uses a
 * fixed scratch array compiled into libtq.so: 4 MiB (4194304 bytes) per device,
 * 256-byte aligned, allocated when the library's device code is loaded. It
 * allocates nothing, itself or through any library routine.
 *
 * Size limit: the call needs tq_decode_workspace_bytes(ctx, batch, n_q_heads,
 * n_kv_heads, max_seq_len) bytes of scratch; above 4194304 it returns
 * TQ_ERR_WORKSPACE and enqueues nothing (use tq_decode_attention then).
 *
 * State: the scratch's completion counters must be zero when a call starts.
 * They are zero when the device code is loaded, and every call that runs to
 * the end -- including one that records a device error -- leaves them at zero.
 * The scratch is shared by every context of the process on that device, so
 * calls on one device must not overlap: issue them on one stream, or order
 * them with events. Two calls in flight at once race on the scratch and give
 * wrong results.
 *
 * First call: the first call on a device looks up the scratch's device
 * address (cudaGetSymbolAddress), which may load the library's device code on
 * that device. Make that first call before any stream capture begins; later
 * calls only enqueue the kernel. Arguments and the size limit are checked
 * before that lookup, so a rejected call touches no device. The address is
 * kept for the life of the process: after a cudaDeviceReset of that device the
 * call must not be used again.
 */
tq_status tq_decode_attention_noalloc(tq_ctx* ctx, const void* q, tq_dtype q_dtype, const void* cache,
                                      int64_t n_cache_pages, const int32_t* block_tables,
                                      int max_pages_per_seq, const int32_t* seq_lens, int batch,
                                      int n_q_heads, int n_kv_heads, int max_seq_len, float scale,
                                      float* out, tq_stream stream);

/*
 * Test hook (no counterpart on the pages): makes a device-side failure path run
 * without any fault. With TQ_TEST_WAIT_RUNS_OUT set, in every later decode call
 * of this context warp 0 of thread block 0 first waits, with a short limit
 * (2^16 clock cycles), on a shared-memory barrier that nothing completes. That
 * wait runs out: the warp records TQ_DEV_TIMEOUT, lets its copies in flight
 * land, stops reading pages and joins the merge, so the call finishes and its
 * output stays finite but leaves out that warp's pages. flags = 0 (the
 * default) turns it off. Unknown bits: TQ_ERR_INVALID_ARG. Host-side setting.
 */
#define TQ_TEST_WAIT_RUNS_OUT 0x1u
tq_status tq_set_test_flags(tq_ctx* ctx, unsigned flags);

/* Synchronise `stream`, then read and clear the device error word (TQ_DEV_* bits). */
tq_status tq_get_device_error(tq_ctx* ctx, uint32_t* code, tq_stream stream);

/* ---- Host-only table generators (no device needed; what tq_init_* upload) ---- */

/* D in {+1,-1}^d for `seed` (see tq_init_rotation). out: (host) int8 [d]. */
tq_status tq_host_sign_vector(uint64_t seed, int d, int8_t* out);

/* S (m x d) for `seed` as fp16 bit patterns, row-major. out: (host) uint16 [m*d]. */
tq_status tq_host_gaussian_sketch(uint64_t seed, int m, int d, uint16_t* out);

/* b-bit codebook for head_dim d: centroids (host, fp16 bits [2^b], ascending) and
 * thresholds (host, float [2^b - 1]). */
tq_status tq_host_codebook(int bits, int d, uint16_t* centroids, float* thresholds);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
