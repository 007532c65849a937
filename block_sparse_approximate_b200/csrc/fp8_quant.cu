// Per-block e4m3 quantisation of the sparse branch (SLA2 §2C quantises the
// sparse branch to 8 bits).  One scale per (head, block of `block` rows):
// σ = absmax / 448 (1 for an all-zero block), code = e4m3(x / σ) with
// round-to-nearest-even and saturation.  The division is the correctly
// rounded fp32 one, so the codes are reproducible bit for bit from fp32.
// HBM-bound: each element is read once (bf16) and written once (1 byte).
#include <cuda_fp8.h>

#include "common.cuh"

namespace sa {
namespace {

constexpr int kQThreads = 256;

// One CTA per (block, head); rows beyond N (a ragged last block) are skipped.
template <int D, int BLK>
__global__ void __launch_bounds__(kQThreads)
quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ X, int N, uint8_t* __restrict__ codes,
                     float* __restrict__ scales, float* __restrict__ scale_max) {
  constexpr int COLS = D / 8;
  constexpr int RPP = kQThreads / COLS;
  constexpr int ROWS = BLK / RPP;
  const int j = blockIdx.x, bh = blockIdx.y;
  const int nblk = (N + BLK - 1) / BLK;
  const int tid = threadIdx.x, col = tid % COLS, r0 = tid / COLS;
  const size_t base = (size_t)bh * N * D;
  __shared__ float red[kQThreads / 32];

  float x[ROWS][8];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const int row = j * BLK + r0 + r * RPP;
    if (row < N) {
      load8<__nv_bfloat16>(X + base + (size_t)row * D + col * 8, x[r]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[r][e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[r][e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) m = fmaxf(m, red[w]);
  const float sigma = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
  if (tid == 0) {
    scales[(size_t)bh * nblk + j] = sigma;
    if (scale_max) atomicMax(reinterpret_cast<unsigned int*>(scale_max + bh), __float_as_uint(sigma));
  }
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const int row = j * BLK + r0 + r * RPP;
    if (row >= N) continue;
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(x[r][4 * h + 0], sigma), __fdiv_rn(x[r][4 * h + 1], sigma)), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(x[r][4 * h + 2], sigma), __fdiv_rn(x[r][4 * h + 3], sigma)), __NV_SATFINITE, __NV_E4M3);
      w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    *reinterpret_cast<uint2*>(codes + base + (size_t)row * D + col * 8) = make_uint2(w[0], w[1]);
  }
}

}  // namespace
}  // namespace sa

extern "C" sa_status sa_quantize_e4m3(const void* X, int64_t BH, int32_t N, int32_t d, int32_t block,
                                      uint8_t* codes, float* scales, float* scale_max, void* stream) {
  using namespace sa;
  if (BH < 0 || N < 0) return fail(SA_ERR_INVALID_ARG, "sa_quantize_e4m3: negative size");
  if (d != 128 && d != 64) return fail(SA_ERR_UNSUPPORTED, "sa_quantize_e4m3: d must be 64 or 128");
  if (block != 128 && block != 64) return fail(SA_ERR_UNSUPPORTED, "sa_quantize_e4m3: block must be 64 or 128");
  if (BH == 0 || N == 0) return SA_OK;
  if (BH > 65535) return fail(SA_ERR_UNSUPPORTED, "sa_quantize_e4m3: at most 65535 heads per call");
  if (!X || !codes || !scales) return fail(SA_ERR_INVALID_ARG, "sa_quantize_e4m3: X, codes and scales are required");
  if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) || (scale_max && !aligned16(scale_max)))
    return fail(SA_ERR_ALIGNMENT, "sa_quantize_e4m3: pointers must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  if (scale_max && cudaMemsetAsync(scale_max, 0, (size_t)BH * sizeof(float), s) != cudaSuccess)
    return launch_status("cudaMemsetAsync(scale_max)");
  dim3 grid((N + block - 1) / block, (unsigned)BH);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(X);
  if (d == 128 && block == 128) quantize_e4m3_kernel<128, 128><<<grid, kQThreads, 0, s>>>(x, N, codes, scales, scale_max);
  else if (d == 128) quantize_e4m3_kernel<128, 64><<<grid, kQThreads, 0, s>>>(x, N, codes, scales, scale_max);
  else if (block == 128) quantize_e4m3_kernel<64, 128><<<grid, kQThreads, 0, s>>>(x, N, codes, scales, scale_max);
  else quantize_e4m3_kernel<64, 64><<<grid, kQThreads, 0, s>>>(x, N, codes, scales, scale_max);
  return launch_status("quantize_e4m3_kernel");
}
