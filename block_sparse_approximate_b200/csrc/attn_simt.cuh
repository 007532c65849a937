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
                  const sa_block_stats& st, float scale, void* O, float* lse_out, cudaStream_t stream);

bool attn_tc_supports(sa_dtype dtype, const sa_shape& s, sa_tail_mode tail);

// d×d sums per head on the tensor cores (bf16, d = 128, N a multiple of 128),
// added into `out`, which the caller zeroes first:
//   kKvRelu:   H_tot = Σ_n relu(k_n) v_nᵀ (oscale 1);
//   kKvCentre: oscale · Σ_j Σ_{n∈j} (k_n − k̄_j) v_nᵀ over 128-token blocks
//              with centroids kmean and value sums vsum [B,H,N/128,d]
//              (H̄ with oscale = 1/nb);
//   kKvExp:    Σ_n φ(k_n) v_nᵀ with φ = phi_exp rounded to bf16 (SPLA's
//              residual linear state; oscale 1).
// Returns SA_ERR_UNSUPPORTED (without setting an error) for other shapes.
enum { kKvRelu = 0, kKvCentre = 1, kKvExp = 2 };
sa_status kv_outer_tc(const void* K, const void* V, const sa_shape& s, int feature, const float* kmean,
                      const float* vsum, float oscale, float* out, cudaStream_t stream);

// PISA's block covariance norms M_j = ‖H_j − H̄‖₂ on the tensor cores (bf16,
// d = block = 128): covnorm [B,H,nb] from K, V and the statistics kmean,
// vsum [B,H,nb,d] and hbar [B,H,d,d].  Returns SA_ERR_UNSUPPORTED (without
// setting an error) for other shapes.
sa_status covnorm_tc(const void* K, const void* V, const sa_shape& s, const float* kmean, const float* vsum,
                     const float* hbar, float* covnorm, cudaStream_t stream);

// Tensor maps and device error words shared by the tensor-core translation
// units: a 3-D [outer][rows][cols] map with a {128 bytes, 128 rows, 1} box
// and 128-byte swizzle (elem = 2 for bf16, 1 for e4m3), and the read-and-clear
// of the covariance kernel's bounded-wait error word.
bool make_tmap_128x128(void* map, const void* base, int elem, uint64_t cols, uint64_t rows, uint64_t outer);
uint32_t covnorm_error_take();

// Backward of the sparse prefill on the tensor cores (bwd_mma.cu): bf16,
// d = 128, block 64 or 128 (zero-order needs the bf16 centroids).  lse2,
// delta [B·H·N] and the per-KV-block query lists offs/list come from the
// caller's workspace (offs/list filled beforehand).
bool bwd_tc_supports(sa_dtype dtype, const sa_shape& s, bool zo, const sa_block_stats& st);
// Tail terms of the block-128 tensor-core backward, each pointer optional:
// PISA's first-order tail: doff [B·H·N] = dO_t·f_t / B (input), delta_c
// [B·H·N] the centroid keys' δ and lam [2][B·H·N] the two element-wise groups'
// shares of λ_t (outputs); SLA2's linear mix: delta_in [B·H·N] the rows' δ of
// the softmax branch, used instead of dO·O (input), and dq_add: the dQ kernel
// adds to dQ instead of overwriting it.
struct BwdTailTerms {
  const float* doff;
  float* delta_c;
  float* lam;
  const float* delta_in;
  bool dq_add;
};
sa_status bwd_tc(const void* Q, const void* K, const void* V, const void* O, const void* dO, const sa_shape& s,
                 const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st, float scale, float* dQ,
                 float* dK, float* dV, const float* lse_in, float* lse2, float* delta, const int32_t* offs,
                 const int32_t* list, float* part, cudaStream_t stream, const BwdTailTerms* fo = nullptr);
// bytes of the centroid pass's partial sums (workspace)
size_t bwd_tc_part_bytes(const sa_shape& s);
// dQ (with lse2 and delta) on tcgen05 (bwd_tc.cu): block 128, d = 128, at
// least one tile per query block (topk > 0 or the zero-order tail); and the
// read-and-clear of that kernel's bounded-wait error word.
sa_status bwd_dq_tc(const void* Q, const void* K, const void* V, const void* O, const void* dO, const sa_shape& s,
                    const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st, float scale,
                    const float* lse_in, float* lse2, float* delta, float* dQ, cudaStream_t stream,
                    const BwdTailTerms* fo = nullptr);
// dK, dV on tcgen05 (bwd_tc.cu), block 128, d = 128, written for every key:
// the exact keys' sums plus, with the zero-order tail (zo), each block's
// pseudo-key gradients ÷B (formed first in `part`, nsplit query ranges);
// delta_cent (or delta when null) is the pseudo-keys' δ.
sa_status bwd_dkv_tc(const void* Q, const void* K, const void* V, const void* dO, const sa_shape& s,
                     const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st, const int32_t* offs,
                     const int32_t* list, float scale, const float* lse2, const float* delta, float* dK, float* dV,
                     float* part, int nsplit, cudaStream_t stream, const float* delta_cent = nullptr);
uint32_t bwd_error_take();
// PISA's first-order tail in the backward (bwd_fo.cu; bf16, d = block = 128):
// the zero-order tensor-core backward with the pseudo-keys' δ shifted, then
// the terms through H̄.  fo_ws: bwd_fo_bytes(s) of workspace.
size_t bwd_fo_bytes(const sa_shape& s);
// SLA2's linear mix in the backward (bwd_lin.cu; bf16, d = block = 128): the
// drop backward of α⊙dO with the softmax branch's δ, then the linear branch.
// lin_ws: bwd_lin_bytes(s) of workspace.
size_t bwd_lin_bytes(const sa_shape& s);
sa_status bwd_linear_mix(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                         const sa_shape& s, const int32_t* block_idx, int topk, const float* alpha,
                         const sa_block_stats& st, float scale, float* dQ, float* dK, float* dV, float* lse2,
                         float* delta, const int32_t* offs, const int32_t* list, float* part, char* lin_ws,
                         cudaStream_t stream);
sa_status bwd_first_order(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                          const sa_shape& s, const int32_t* block_idx, int topk, const sa_block_stats& st, float scale,
                          float* dQ, float* dK, float* dV, const float* lse_in, float* lse2, float* delta,
                          const int32_t* offs, const int32_t* list, float* part, float* fo_ws, cudaStream_t stream);

}  // namespace sa
