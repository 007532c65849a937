// Tensor-core sparse prefill (tcgen05 + TMEM + TMA), bf16, block 128.
#include "attn_simt.cuh"

namespace sa {

bool attn_tc_supports(sa_dtype, const sa_shape&, sa_tail_mode) { return false; }

sa_status attn_tc(const void*, const void*, const void*, const sa_shape&, const int32_t*, int,
                  sa_tail_mode, const float*, const sa_block_stats&, float, void*, cudaStream_t) {
  return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd: tensor-core path not built");
}

}  // namespace sa
