// C-ABI plumbing of libsparseattn: error reporting, shape checks and the
// sparse prefill entry point (which picks the tensor-core or the CUDA-core
// kernel for the request).
#include <string>

#include "attn_simt.cuh"

namespace sa {

namespace {
thread_local std::string g_last_error;
}

void set_error(const std::string& msg) { g_last_error = msg; }

sa_status check_shape(const sa_shape& s, const char* fn) {
  if (s.B < 0 || s.H < 0 || s.N < 0 || s.d <= 0 || s.block <= 0)
    return fail(SA_ERR_INVALID_ARG, std::string(fn) + ": negative or zero size");
  if (s.d != 64 && s.d != 128) return fail(SA_ERR_UNSUPPORTED, std::string(fn) + ": d must be 64 or 128");
  if (s.block != 64 && s.block != 128)
    return fail(SA_ERR_UNSUPPORTED, std::string(fn) + ": block must be 64 or 128");
  if (s.N % s.block) return fail(SA_ERR_INVALID_ARG, std::string(fn) + ": N must be a multiple of block");
  return SA_OK;
}

}  // namespace sa

extern "C" const char* sa_last_error(void) { return sa::g_last_error.c_str(); }

extern "C" const char* sa_version(void) { return "libsparseattn 0.1 (sm_100a)"; }

namespace sa {
namespace {
// lse2: the rows' log-sum-exp output (sa_sparse_attn_fwd_lse) or null
sa_status fwd_entry(const void* Q, const void* K, const void* V, sa_dtype dtype, sa_shape shape,
                    const int32_t* block_idx, int32_t topk, sa_tail_mode tail, const float* alpha,
                    const sa_block_stats* stats, float scale, void* O, float* lse2, void* stream) {
  sa_status r = check_shape(shape, "sa_sparse_attn_fwd");
  if (r != SA_OK) return r;
  const int nb = shape.N / shape.block;
  if (dtype != SA_FP32 && dtype != SA_BF16)
    return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd: dtype must be SA_FP32 or SA_BF16");
  if (tail == SA_TAIL_RESIDUAL_LINEAR)
    return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd: SA_TAIL_RESIDUAL_LINEAR is a decode tail");
  if (tail != SA_TAIL_DROP && tail != SA_TAIL_ZERO_ORDER && tail != SA_TAIL_LINEAR_MIX &&
      tail != SA_TAIL_FIRST_ORDER)
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd: unknown tail mode");
  if (shape.B == 0 || shape.H == 0 || shape.N == 0) return SA_OK;  // nothing to compute
  if (!Q || !K || !V || !O) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd: Q, K, V and O are required");
  if (topk < 0 || topk > nb) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd: topk must be in [0, N/block]");
  if (topk > 0 && !block_idx) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd: block_idx is required");
  if (nb > kMaxAttnBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd: at most 4096 blocks per head");
  sa_block_stats st{};
  if (stats) st = *stats;
  if (tail == SA_TAIL_ZERO_ORDER && (!st.kmean || !st.vsum))
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd: SA_TAIL_ZERO_ORDER needs stats->kmean and stats->vsum");
  if (tail == SA_TAIL_FIRST_ORDER && (!st.kmean || !st.vsum || !st.hbar))
    return fail(SA_ERR_INVALID_ARG,
                "sa_sparse_attn_fwd: SA_TAIL_FIRST_ORDER needs stats->kmean, stats->vsum and stats->hbar");
  if (tail == SA_TAIL_LINEAR_MIX && (!alpha || !st.zrelu || !st.htot || !st.ztot))
    return fail(SA_ERR_INVALID_ARG,
                "sa_sparse_attn_fwd: SA_TAIL_LINEAR_MIX needs alpha and stats->zrelu, htot, ztot");
  const void* ptrs[] = {Q, K, V, O, block_idx, alpha, st.kmean, st.vsum, st.zrelu, st.htot, st.ztot,
                        st.kmean_bf16, st.vmean_bf16, st.hbar, st.hbarT_bf16};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_sparse_attn_fwd: pointers must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  // the tensor-core kernel reads the tails' operands as bf16 tiles
  const bool tc_operands = (tail != SA_TAIL_ZERO_ORDER && tail != SA_TAIL_FIRST_ORDER) ||
                           (st.kmean_bf16 && st.vmean_bf16 && (tail == SA_TAIL_ZERO_ORDER || st.hbarT_bf16));
  const bool tc = attn_tc_supports(dtype, shape, tail) && tc_operands;
  if (lse2) {
    if (!tc || (tail != SA_TAIL_DROP && tail != SA_TAIL_ZERO_ORDER && tail != SA_TAIL_FIRST_ORDER))
      return fail(SA_ERR_UNSUPPORTED,
                  "sa_sparse_attn_fwd_lse: the log-sum-exp comes from the bf16 tensor-core kernel (d = 128, "
                  "block 128, SA_TAIL_DROP, SA_TAIL_ZERO_ORDER or SA_TAIL_FIRST_ORDER with the bf16 centroids)");
    if (!aligned16(lse2)) return fail(SA_ERR_ALIGNMENT, "sa_sparse_attn_fwd_lse: lse2 must be 16-byte aligned");
  }
  if (tc) return attn_tc(Q, K, V, shape, block_idx, topk, tail, alpha, st, scale, O, lse2, s);
  return attn_simt(Q, K, V, dtype, shape, block_idx, topk, tail, alpha, st, scale, O, s);
}
}  // namespace
}  // namespace sa

extern "C" sa_status sa_sparse_attn_fwd(const void* Q, const void* K, const void* V,
                                        sa_dtype dtype, sa_shape shape,
                                        const int32_t* block_idx, int32_t topk,
                                        sa_tail_mode tail, const float* alpha,
                                        const sa_block_stats* stats, float scale, void* O,
                                        void* stream) {
  return sa::fwd_entry(Q, K, V, dtype, shape, block_idx, topk, tail, alpha, stats, scale, O, nullptr, stream);
}

extern "C" sa_status sa_sparse_attn_fwd_lse(const void* Q, const void* K, const void* V, sa_dtype dtype,
                                            sa_shape shape, const int32_t* block_idx, int32_t topk,
                                            sa_tail_mode tail, const sa_block_stats* stats, float scale,
                                            void* O, float* lse2, void* stream) {
  if (!lse2) return sa::fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd_lse: lse2 is required");
  return sa::fwd_entry(Q, K, V, dtype, shape, block_idx, topk, tail, nullptr, stats, scale, O, lse2, stream);
}
