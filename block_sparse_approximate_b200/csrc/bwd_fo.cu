// Backward of PISA's first-order tail ("Algoritmo Central", the hybrid
// order), the terms the zero-order backward does not have.  The forward adds
// λ_t f_t to the zero-order output, with f_t = s H̄ᵀ q_t (H̄ the mean over the
// head's blocks of H_j = Σ_{n∈j} (k_n − k̄_j) v_nᵀ) and λ_t = Σ_{j∈U} P_tj / B
// (the pseudo-keys' share of the row's softmax).  So a pseudo-key's value
// seen by row t is v̄_j + f_t / B, and with G = s Σ_t λ_t q_t dO_tᵀ:
//   pseudo-keys:  dS = P (dP − δ + doff_t),  doff_t = dO_t·f_t / B
//                 (taken by the tensor-core dQ and centroid dK/dV kernels),
//   dq_t  += s λ_t H̄ dO_t,
//   dk_m  += G (v_m − v̄_j) / nb,   dv_m += Gᵀ (k_m − k̄_j) / nb   (m in block j).
// Three kernels here, all 128 x 128 x 128 contractions on mma.sync
// (m16n8k16, bf16 operands, fp32 accumulation) over 128-row tiles staged in
// shared memory with 16-byte chunks of row r at chunk ^ (r & 7):
//   fo_pre_kernel    y_t = H̄ dO_t, doff_t = s q_t·y_t / B;
//   fo_gram_kernel   partial G over a range of rows (then fo_reduce_kernel
//                    sums the ranges in order: no atomics);
//   fo_apply_kernel  the dq, dk, dv terms above, added to the gradients the
//                    zero-order kernels wrote.
// H̄ and G enter the products rounded to bf16 (2^-9 relative), like every
// operand of the tensor-core backward.
#include "mma_tile.cuh"

namespace sa {
namespace {

using namespace mt;

// doff_t = s q_t·(H̄ dO_t) / B for the 128 rows of query block blockIdx.x.
__global__ void __launch_bounds__(kFoThreads)
fo_pre_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ dO,
              const float* __restrict__ hbar, int N, float scale, float inv_blk, float* __restrict__ doff) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int i = blockIdx.x, bh = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t row0 = (size_t)bh * N + (size_t)i * FT;
  uint8_t* hb = fsm;                 // H̄ [c][e]
  uint8_t* gt = fsm + kTileB;        // dO [t][e]
  stage_bf16(gt, dO + row0 * FD);
  stage_f32(hb, hbar + (size_t)bh * FD * FD);
  fo_cp_wait_all();
  __syncthreads();
  float acc[16][4];
  zero_acc(acc);
  // y[t][c] = Σ_e dO[t][e] H̄[c][e]: A = dO [t][e], B[e][c] = H̄[c][e] stored [c][e]
  warp_gemm<kRowsMK, kRowsMK>(acc, (uint32_t)__cvta_generic_to_shared(gt), (uint32_t)__cvta_generic_to_shared(hb),
                              16 * warp, lane);
  const int ra = 16 * warp + (lane >> 2), rb = ra + 8;
  float wa = 0.f, wb = 0.f;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int c = 8 * nt + 2 * (lane & 3);
    const float2 qa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Q + (row0 + ra) * FD + c));
    const float2 qb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Q + (row0 + rb) * FD + c));
    wa = fmaf(qa.x, acc[nt][0], fmaf(qa.y, acc[nt][1], wa));
    wb = fmaf(qb.x, acc[nt][2], fmaf(qb.y, acc[nt][3], wb));
  }
  wa += __shfl_xor_sync(0xffffffffu, wa, 1);
  wa += __shfl_xor_sync(0xffffffffu, wa, 2);
  wb += __shfl_xor_sync(0xffffffffu, wb, 1);
  wb += __shfl_xor_sync(0xffffffffu, wb, 2);
  if ((lane & 3) == 0) {
    doff[row0 + ra] = scale * wa * inv_blk;
    doff[row0 + rb] = scale * wb * inv_blk;
  }
}

// part[bh][chunk] = s Σ_{t in the chunk's rows} λ_t q_t dO_tᵀ  (d x d, row c, column e)
__global__ void __launch_bounds__(kFoThreads)
fo_gram_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ dO,
               const float* __restrict__ lam, size_t lam_stride, int N, float scale, float* __restrict__ part) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int chunk = blockIdx.x, bh = blockIdx.y, nchunk = gridDim.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* qt = fsm;                 // λ q [t][c]
  uint8_t* gt = fsm + kTileB;        // dO [t][e]
  float acc[16][4];
  zero_acc(acc);
  const int r_end = min(N, (chunk + 1) * kGramRows);
  for (int r0 = chunk * kGramRows; r0 < r_end; r0 += FT) {
    const size_t row0 = (size_t)bh * N + r0;
    __syncthreads();   // the previous tile has been read
    stage_bf16(gt, dO + row0 * FD);
    for (int o = threadIdx.x; o < FT * 16; o += kFoThreads) {
      const int r = o >> 4, c = o & 15;
      const float l = lam[row0 + r] + lam[lam_stride + row0 + r];
      const uint4 x = *reinterpret_cast<const uint4*>(Q + (row0 + r) * FD + 8 * c);
      const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv[e]));
        w[e] = fo_pack2(l * f.x, l * f.y);
      }
      *reinterpret_cast<uint4*>(qt + swz(r, c)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fo_cp_wait_all();
    __syncthreads();
    // G[c][e] += Σ_t (λq)[t][c] dO[t][e]: A[c][t] stored [t][c], B[t][e] stored [t][e]
    warp_gemm<kRowsKM, kRowsKM>(acc, (uint32_t)__cvta_generic_to_shared(qt), (uint32_t)__cvta_generic_to_shared(gt),
                                16 * warp, lane);
  }
  float* out = part + ((size_t)bh * nchunk + chunk) * FD * FD;
  const int ra = 16 * warp + (lane >> 2), rb = ra + 8;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int c = 8 * nt + 2 * (lane & 3);
    *reinterpret_cast<float2*>(out + (size_t)ra * FD + c) = make_float2(scale * acc[nt][0], scale * acc[nt][1]);
    *reinterpret_cast<float2*>(out + (size_t)rb * FD + c) = make_float2(scale * acc[nt][2], scale * acc[nt][3]);
  }
}

// G[bh] = Σ_chunk part[bh][chunk], in chunk order
__global__ void fo_reduce_kernel(const float* __restrict__ part, int nchunk, float* __restrict__ G) {
  const int bh = blockIdx.y;
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= FD * FD) return;
  float s = 0.f;
  for (int c = 0; c < nchunk; ++c) s += part[((size_t)bh * nchunk + c) * FD * FD + x];
  G[(size_t)bh * FD * FD + x] = s;
}

// One CTA per 128-row block j (queries and keys alike):
//   dQ_t += s λ_t H̄ dO_t,  dK_m += G (v_m − v̄_j) / nb,  dV_m += Gᵀ (k_m − k̄_j) / nb.
__global__ void __launch_bounds__(kFoThreads)
fo_apply_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                const __nv_bfloat16* __restrict__ dO, const float* __restrict__ kmean, const float* __restrict__ vsum,
                const float* __restrict__ hbar, const float* __restrict__ G, const float* __restrict__ lam,
                size_t lam_stride, int N, float scale, float* __restrict__ dQ, float* __restrict__ dK,
                float* __restrict__ dV) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int j = blockIdx.x, bh = blockIdx.y;
  const int nb = N / FT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t row0 = (size_t)bh * N + (size_t)j * FT;
  const size_t blk = (size_t)bh * nb + j;
  uint8_t* hb = fsm;                 // H̄ [c][e]
  uint8_t* gb = fsm + kTileB;        // G [c][e]
  uint8_t* at = fsm + 2 * kTileB;    // the A tile of each product
  const uint32_t hs = (uint32_t)__cvta_generic_to_shared(hb), gs = (uint32_t)__cvta_generic_to_shared(gb),
                 as = (uint32_t)__cvta_generic_to_shared(at);
  const int ra = 16 * warp + (lane >> 2), rb = ra + 8;
  const float inv_nb = 1.0f / nb;
  float acc[16][4];
  stage_bf16(at, dO + row0 * FD);
  stage_f32(hb, hbar + (size_t)bh * FD * FD);
  stage_f32(gb, G + (size_t)bh * FD * FD);
  fo_cp_wait_all();
  __syncthreads();
  // dQ: y[t][c] = Σ_e dO[t][e] H̄[c][e]
  zero_acc(acc);
  warp_gemm<kRowsMK, kRowsMK>(acc, as, hs, 16 * warp, lane);
  add_rows(dQ + row0 * FD, acc, ra, rb, lane, scale * (lam[row0 + ra] + lam[lam_stride + row0 + ra]),
           scale * (lam[row0 + rb] + lam[lam_stride + row0 + rb]));
  __syncthreads();
  // dK: Σ_e (v − v̄_j)[m][e] G[c][e]
  stage_centred(at, V + row0 * FD, vsum + blk * FD, 1.0f / FT);
  __syncthreads();
  zero_acc(acc);
  warp_gemm<kRowsMK, kRowsMK>(acc, as, gs, 16 * warp, lane);
  add_rows(dK + row0 * FD, acc, ra, rb, lane, inv_nb, inv_nb);
  __syncthreads();
  // dV: Σ_c (k − k̄_j)[m][c] G[c][e]
  stage_centred(at, K + row0 * FD, kmean + blk * FD, 1.0f);
  __syncthreads();
  zero_acc(acc);
  warp_gemm<kRowsMK, kRowsKM>(acc, as, gs, 16 * warp, lane);
  add_rows(dV + row0 * FD, acc, ra, rb, lane, inv_nb, inv_nb);
}

}  // namespace

size_t bwd_fo_bytes(const sa_shape& s) {
  const size_t BH = (size_t)s.B * s.H;
  const size_t nchunk = (size_t)((s.N + kGramRows - 1) / kGramRows);
  return 4 * BH * s.N * sizeof(float) + (nchunk + 1) * BH * FD * FD * sizeof(float);
}

sa_status bwd_first_order(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                          const sa_shape& s, const int32_t* block_idx, int topk, const sa_block_stats& st, float scale,
                          float* dQ, float* dK, float* dV, const float* lse_in, float* lse2, float* delta,
                          const int32_t* offs, const int32_t* list, float* part, float* fo_ws, cudaStream_t stream) {
  typedef __nv_bfloat16 bf;
  const size_t BH = (size_t)s.B * s.H, rows = BH * s.N;
  const int nqb = s.N / FT, nchunk = (s.N + kGramRows - 1) / kGramRows;
  float* doff = fo_ws;
  float* delta_c = doff + rows;
  float* lam = delta_c + rows;                  // [2][rows]
  float* gpart = lam + 2 * rows;                // [BH][nchunk][d][d]
  float* G = gpart + (size_t)nchunk * BH * FD * FD;
  const bf* q = static_cast<const bf*>(Q);
  const bf* k = static_cast<const bf*>(K);
  const bf* v = static_cast<const bf*>(V);
  const bf* g = static_cast<const bf*>(dO);
  const dim3 grid(nqb, (unsigned)BH);
  const size_t smem2 = 2 * kTileB, smem3 = 3 * kTileB;
  if (cudaFuncSetAttribute(fo_pre_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) != cudaSuccess ||
      cudaFuncSetAttribute(fo_gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) != cudaSuccess ||
      cudaFuncSetAttribute(fo_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(first-order backward kernels)");
  fo_pre_kernel<<<grid, kFoThreads, smem2, stream>>>(q, g, st.hbar, s.N, scale, 1.0f / FT, doff);
  sa_status r = launch_status("fo_pre_kernel");
  if (r != SA_OK) return r;
  // the zero-order backward with the pseudo-keys' shifted δ
  const BwdTailTerms fo{doff, delta_c, lam, nullptr, false};
  r = bwd_tc(Q, K, V, O, dO, s, block_idx, topk, true, st, scale, dQ, dK, dV, lse_in, lse2, delta, offs, list, part,
             stream, &fo);
  if (r != SA_OK) return r;
  fo_gram_kernel<<<dim3(nchunk, (unsigned)BH), kFoThreads, smem2, stream>>>(q, g, lam, rows, s.N, scale, gpart);
  r = launch_status("fo_gram_kernel");
  if (r != SA_OK) return r;
  fo_reduce_kernel<<<dim3(FD * FD / 256, (unsigned)BH), 256, 0, stream>>>(gpart, nchunk, G);
  r = launch_status("fo_reduce_kernel");
  if (r != SA_OK) return r;
  fo_apply_kernel<<<grid, kFoThreads, smem3, stream>>>(k, v, g, st.kmean, st.vsum, st.hbar, G, lam, rows, s.N, scale,
                                                       dQ, dK, dV);
  return launch_status("fo_apply_kernel");
}

}  // namespace sa
