// Internal launchers of the sparse prefill kernels (not part of the C ABI).
#pragma once

#include "common.cuh"

namespace sa {

constexpr int kMaxAttnBlocks = 4096;

// CUDA-core path: any supported dtype, d, block and tail mode.
sa_status attn_simt(const void* Q, const void* K, const void* V, sa_dtype dtype, const sa_shape& s,
                    const int32_t* block_idx, int topk, sa_tail_mode tail, const float* alpha,
                    const sa_block_stats& st, float scale, void* O, cudaStream_t stream);

// Tensor-core path (tcgen05 + TMEM + TMA): bf16, block 128, d 128, tails
// drop and zero-order (attn_tc_supports says which requests it takes).
sa_status attn_tc(const void* Q, const void* K, const void* V, const sa_shape& s,
                  const int32_t* block_idx, int topk, sa_tail_mode tail, const float* alpha,
                  const sa_block_stats& st, float scale, void* O, cudaStream_t stream);

bool attn_tc_supports(sa_dtype dtype, const sa_shape& s, sa_tail_mode tail);

// H_tot = Σ_n relu(k_n) v_nᵀ per head on the tensor cores (bf16, d = 128, N a
// multiple of 128); adds into htot, which the caller zeroes first.  Returns
// SA_ERR_UNSUPPORTED (without setting an error) for other shapes.
sa_status htot_tc(const void* K, const void* V, const sa_shape& s, float* htot, cudaStream_t stream);

}  // namespace sa
