// Instantiations of libtq's decode and prefill kernels for one (key bits,
// value bits) pair, chosen by TQ_BK and TQ_BV on the compiler command line; the
// build compiles this file once per supported pair, in parallel.
#include "tq_kernels.cuh"

#if !defined(TQ_BK) || !defined(TQ_BV)
#error "compile with -DTQ_BK=<2|3|4|8> -DTQ_BV=<2|3|4>"
#endif

namespace tq {
namespace {

template <int BK, int BV, int NH, int MODE>
cudaError_t launch_decode_t(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s) {
  return a.balanced ? launch_decode_tb<BK, BV, NH, MODE, true>(T, a, grid, s)
                    : launch_decode_tb<BK, BV, NH, MODE, false>(T, a, grid, s);
}

template <int BK, int BV, int MODE>
cudaError_t dispatch_nh(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s) {
  switch (a.n_hg) {
    case 1: return launch_decode_t<BK, BV, 1, MODE>(T, a, grid, s);
    case 2: return launch_decode_t<BK, BV, 2, MODE>(T, a, grid, s);
    case 3: return launch_decode_t<BK, BV, 3, MODE>(T, a, grid, s);
    default: return launch_decode_t<BK, BV, 4, MODE>(T, a, grid, s);
  }
}

}  // namespace

#define TQ_PASTE2(a, b, c, d) a##b##_##c
#define TQ_NAME(a, b, c) TQ_PASTE2(a, b, c, 0)

cudaError_t TQ_NAME(decode_bits_, TQ_BK, TQ_BV)(const Tables& T, const DecodeArgs& a, dim3 grid, cudaStream_t s,
                                                int mode) {
  switch (mode) {
    case 0: return dispatch_nh<TQ_BK, TQ_BV, 0>(T, a, grid, s);
    case 1: return dispatch_nh<TQ_BK, TQ_BV, 1>(T, a, grid, s);
    default: return dispatch_nh<TQ_BK, TQ_BV, 2>(T, a, grid, s);
  }
}

cudaError_t TQ_NAME(prefill_bits_, TQ_BK, TQ_BV)(const Tables& t, const void* k, const void* v, int dtype,
                                                 int n_tokens, int n_kv, const int32_t* block_table, int start_pos,
                                                 void* cache, int64_t n_pages, cudaStream_t s) {
  return launch_prefill_t<TQ_BK, TQ_BV>(t, k, v, dtype, n_tokens, n_kv, block_table, start_pos, cache, n_pages, s);
}

}  // namespace tq
