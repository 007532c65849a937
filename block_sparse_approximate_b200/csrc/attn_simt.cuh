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
// drop, zero-order, first-order and linear mix (attn_tc_supports says which
// requests it takes).
sa_status attn_tc(const void* Q, const void* K, const void* V, const sa_shape& s,
                  const int32_t* block_idx, int topk, sa_tail_mode tail, const float* alpha,
                  const sa_block_stats& st, float scale, void* O, cudaStream_t stream);

bool attn_tc_supports(sa_dtype dtype, const sa_shape& s, sa_tail_mode tail);

// d×d sums per head on the tensor cores (bf16, d = 128, N a multiple of 128),
// added into `out`, which the caller zeroes first:
//   kmean == NULL: H_tot = Σ_n relu(k_n) v_nᵀ (oscale 1);
//   kmean != NULL: oscale · Σ_j Σ_{n∈j} (k_n − k̄_j) v_nᵀ over 128-token blocks
//                  with centroids kmean [B,H,N/128,d] (H̄ with oscale = 1/nb).
// Returns SA_ERR_UNSUPPORTED (without setting an error) for other shapes.
sa_status kv_outer_tc(const void* K, const void* V, const sa_shape& s, const float* kmean, float oscale,
                      float* out, cudaStream_t stream);

}  // namespace sa
