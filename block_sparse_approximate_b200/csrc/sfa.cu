// Sparse feature attention ("Scaling Attention via Feature Sparsity", §2):
// every query and key keeps its kf coordinates of largest magnitude and the
// score of a pair is the sum over the overlap of the two supports; softmax
// and the dense V are as in ordinary attention.
//
//   sa_sfa_encode   one warp per row: keys pack the bf16 magnitude above the
//                   inverted channel index (distinct; a tie in magnitude goes
//                   to the smaller index); the kf-th largest key is found by
//                   kf rounds of a warp-wide maximum (redux.sync) over each
//                   lane's largest untaken key (lanes pre-sort their keys),
//                   and the keys at or above it are kept; writes the codes in
//                   ascending channel order and, optionally, the zero-filled
//                   row.
//   sa_sfa_densify  codes back to zero-filled rows (a KV cache kept as codes).
//   sa_sfa_attn_fwd the overlap score of two sparse vectors is the dot
//                   product of their zero-filled forms, so FlashSFA's online
//                   softmax over tiles is the tensor-core attention kernel run
//                   over every KV tile: on sm_100 a 128×128×128 bf16 MMA on
//                   zero-filled tiles takes a few hundred cycles of a tensor
//                   pipe that the softmax leaves idle, which is cheaper than
//                   intersecting supports index by index on the CUDA cores.
#include "attn_simt.cuh"

namespace sa {
namespace {

constexpr int kSfaWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kSfaWarps)
sfa_encode_kernel(const __nv_bfloat16* __restrict__ X, int64_t rows, int kf, __nv_bfloat16* __restrict__ vals,
                  uint8_t* __restrict__ idx, __nv_bfloat16* __restrict__ dense) {
  constexpr int CPL = D / 32;                         // channels per lane: lane l holds CPL l .. CPL l + CPL - 1
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kSfaWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const __nv_bfloat16* xr = X + row * D;
  __nv_bfloat16 x[CPL];
  if (CPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(xr + CPL * lane);
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
    for (int e = 0; e < CPL; ++e) x[e] = h[e];
  } else {
#pragma unroll
    for (int e = 0; e < CPL; ++e) x[e] = xr[CPL * lane + e];
  }
  // key: |x| as its 15 bf16 bits, then 255 − channel (distinct for every channel)
  uint32_t key[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    const uint32_t mag = (uint32_t)__bfloat16_as_ushort(x[e]) & 0x7fffu;
    key[e] = (mag << 8) | (uint32_t)(255 - (CPL * lane + e));
  }
  // the kf-th largest key of the row: every lane sorts its keys (descending)
  // and offers its largest not yet taken; each round the warp's maximum is
  // taken and its lane moves on to its next key
  uint32_t srt[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) srt[e] = key[e];
#pragma unroll
  for (int i = 0; i < CPL; ++i)
#pragma unroll
    for (int j = 0; j + 1 < CPL - i; ++j) {
      const uint32_t a = srt[j], b = srt[j + 1];
      srt[j] = max(a, b);
      srt[j + 1] = min(a, b);
    }
  uint32_t thr = 0u;
  for (int r = 0; r < kf; ++r) {
    thr = __reduce_max_sync(0xffffffffu, srt[0]);
    if (srt[0] == thr) {
#pragma unroll
      for (int e = 0; e + 1 < CPL; ++e) srt[e] = srt[e + 1];
      srt[CPL - 1] = 0u;
    }
  }
  uint32_t taken = 0u;                               // bit e: channel CPL lane + e is kept
#pragma unroll
  for (int e = 0; e < CPL; ++e)
    if (key[e] >= thr) taken |= 1u << e;
  // ascending channel order: this lane's kept channels start after those of
  // the lanes below it
  const int mine = __popc(taken);
  int before = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, before, o);
    if (lane >= o) before += v;
  }
  int pos = before - mine;
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    if ((taken >> e) & 1u) {
      vals[row * kf + pos] = x[e];
      idx[row * kf + pos] = (uint8_t)(CPL * lane + e);
      ++pos;
    }
  }
  if (dense) {
    __nv_bfloat16* dr = dense + row * D;
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
    __nv_bfloat16 y[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) y[e] = ((taken >> e) & 1u) ? x[e] : zero;
    if (CPL == 4) {
      *reinterpret_cast<uint2*>(dr + CPL * lane) = *reinterpret_cast<const uint2*>(y);
    } else {
#pragma unroll
      for (int e = 0; e < CPL; ++e) dr[CPL * lane + e] = y[e];
    }
  }
}

template <int D>
__global__ void __launch_bounds__(32 * kSfaWarps)
sfa_densify_kernel(const __nv_bfloat16* __restrict__ vals, const uint8_t* __restrict__ idx, int64_t rows, int kf,
                   __nv_bfloat16* __restrict__ dense) {
  constexpr int CPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kSfaWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  // lane i < kf holds code i; each lane fills its own channels
  const uint32_t my_idx = lane < kf ? (uint32_t)idx[row * kf + lane] : 0xffu;
  const __nv_bfloat16 my_val = lane < kf ? vals[row * kf + lane] : __float2bfloat16_rn(0.f);
  float out[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) out[e] = 0.f;
  for (int i = 0; i < kf; ++i) {
    const uint32_t c = __shfl_sync(0xffffffffu, my_idx, i);
    const float v = __bfloat162float(__shfl_sync(0xffffffffu, my_val, i));
#pragma unroll
    for (int e = 0; e < CPL; ++e)
      if (c == (uint32_t)(CPL * lane + e)) out[e] = v;
  }
  __nv_bfloat16* dr = dense + row * D;
#pragma unroll
  for (int e = 0; e < CPL; ++e) dr[CPL * lane + e] = __float2bfloat16_rn(out[e]);
}

// block_idx[bh][i][t] = t: every query block attends to every KV block
__global__ void identity_index_kernel(int32_t* __restrict__ block_idx, int64_t total, int nb) {
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += (int64_t)gridDim.x * blockDim.x)
    block_idx[x] = (int32_t)(x % nb);
}

sa_status check_codes(int32_t d, int32_t kf, const char* fn) {
  if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, std::string(fn) + ": d must be 64 or 128");
  if (kf < 1 || kf > 32 || kf > d) return fail(SA_ERR_INVALID_ARG, std::string(fn) + ": kf must be in [1, min(d, 32)]");
  return SA_OK;
}

}  // namespace
}  // namespace sa

extern "C" sa_status sa_sfa_encode(const void* X, int64_t rows, int32_t d, int32_t kf, void* vals, uint8_t* idx,
                                   void* dense, void* stream) {
  using namespace sa;
  sa_status r = check_codes(d, kf, "sa_sfa_encode");
  if (r != SA_OK) return r;
  if (rows < 0) return fail(SA_ERR_INVALID_ARG, "sa_sfa_encode: rows must be >= 0");
  if (rows == 0) return SA_OK;
  if (!X || !vals || !idx) return fail(SA_ERR_INVALID_ARG, "sa_sfa_encode: X, vals and idx are required");
  if (!aligned16(X) || (dense && !aligned16(dense)))
    return fail(SA_ERR_ALIGNMENT, "sa_sfa_encode: X and dense must be 16-byte aligned");
  const dim3 grid((unsigned)((rows + kSfaWarps - 1) / kSfaWarps));
  cudaStream_t s = as_stream(stream);
  auto* xv = static_cast<const __nv_bfloat16*>(X);
  auto* ov = static_cast<__nv_bfloat16*>(vals);
  auto* od = static_cast<__nv_bfloat16*>(dense);
  if (d == 128) sfa_encode_kernel<128><<<grid, 32 * kSfaWarps, 0, s>>>(xv, rows, kf, ov, idx, od);
  else sfa_encode_kernel<64><<<grid, 32 * kSfaWarps, 0, s>>>(xv, rows, kf, ov, idx, od);
  return launch_status("sfa_encode_kernel");
}

extern "C" sa_status sa_sfa_densify(const void* vals, const uint8_t* idx, int64_t rows, int32_t d, int32_t kf,
                                    void* dense, void* stream) {
  using namespace sa;
  sa_status r = check_codes(d, kf, "sa_sfa_densify");
  if (r != SA_OK) return r;
  if (rows < 0) return fail(SA_ERR_INVALID_ARG, "sa_sfa_densify: rows must be >= 0");
  if (rows == 0) return SA_OK;
  if (!vals || !idx || !dense) return fail(SA_ERR_INVALID_ARG, "sa_sfa_densify: vals, idx and dense are required");
  const dim3 grid((unsigned)((rows + kSfaWarps - 1) / kSfaWarps));
  cudaStream_t s = as_stream(stream);
  auto* iv = static_cast<const __nv_bfloat16*>(vals);
  auto* od = static_cast<__nv_bfloat16*>(dense);
  if (d == 128) sfa_densify_kernel<128><<<grid, 32 * kSfaWarps, 0, s>>>(iv, idx, rows, kf, od);
  else sfa_densify_kernel<64><<<grid, 32 * kSfaWarps, 0, s>>>(iv, idx, rows, kf, od);
  return launch_status("sfa_densify_kernel");
}

extern "C" size_t sa_sfa_workspace_size(sa_shape shape) {
  using namespace sa;
  if (check_shape(shape, "sa_sfa_workspace_size") != SA_OK) return 0;
  const size_t nb = (size_t)(shape.N / shape.block);
  return ((size_t)shape.B * shape.H * nb * nb * sizeof(int32_t) + 255) & ~(size_t)255;
}

extern "C" sa_status sa_sfa_attn_fwd(const void* Qs, const void* Ks, const void* V, sa_dtype dtype, sa_shape shape,
                                     float scale, void* O, void* workspace, size_t workspace_bytes, void* stream) {
  using namespace sa;
  sa_status r = check_shape(shape, "sa_sfa_attn_fwd");
  if (r != SA_OK) return r;
  if (dtype != SA_FP32 && dtype != SA_BF16)
    return fail(SA_ERR_UNSUPPORTED, "sa_sfa_attn_fwd: dtype must be SA_FP32 or SA_BF16");
  if (shape.B == 0 || shape.H == 0 || shape.N == 0) return SA_OK;
  if (!Qs || !Ks || !V || !O) return fail(SA_ERR_INVALID_ARG, "sa_sfa_attn_fwd: Qs, Ks, V and O are required");
  const int nb = shape.N / shape.block;
  if (nb > kMaxAttnBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_sfa_attn_fwd: at most 4096 blocks per head");
  const size_t need = sa_sfa_workspace_size(shape);
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "sa_sfa_attn_fwd: workspace missing or smaller than sa_sfa_workspace_size()");
  const void* ptrs[] = {Qs, Ks, V, O, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_sfa_attn_fwd: pointers must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  int32_t* idx = static_cast<int32_t*>(workspace);
  const int64_t total = (int64_t)shape.B * shape.H * nb * nb;
  identity_index_kernel<<<(unsigned)std::min<int64_t>((total + 255) / 256, 4096), 256, 0, s>>>(idx, total, nb);
  r = launch_status("identity_index_kernel");
  if (r != SA_OK) return r;
  sa_block_stats st{};
  if (attn_tc_supports(dtype, shape, SA_TAIL_DROP))
    return attn_tc(Qs, Ks, V, shape, idx, nb, SA_TAIL_DROP, nullptr, st, scale, O, nullptr, s);
  return attn_simt(Qs, Ks, V, dtype, shape, idx, nb, SA_TAIL_DROP, nullptr, st, scale, O, s);
}
