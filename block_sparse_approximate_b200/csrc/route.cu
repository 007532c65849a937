// Router: block scores and top-k selection of KV blocks per query block.
//   dot      q̄_i·k̄_j                        (SLA2 §2B, mean pooling)
//   proj     (q̄_i P_q)·(k̄_j P_k)              (SLA2 §2B, learnable router)
//   taylor2  s q̄_i·k̄_j + log1p(½ s² Σ q̄²var)  (SPLA §2.1, log of the
//            second-order block score with diagonal covariance)
// The proj score (q̄_i P_q)·(k̄_j P_k) is evaluated as k̄_j·u_i with
// u_i = P_k P_qᵀ q̄_i (x P is the row vector x times P), so no projected copy
// of the key centroids is needed: u_i costs 2d² multiply-adds per query block.
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kRouteThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRouteThreads)
route_kernel(sa_block_stats st, int H, int nb, sa_route_mode mode, const float* __restrict__ Pq,
             const float* __restrict__ Pk, float scale, int topk, int32_t* __restrict__ block_idx,
             float* __restrict__ scores_out) {
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t bh = (size_t)b * H + h;
  extern __shared__ unsigned long long smem_u64[];
  unsigned long long* keys = smem_u64;                       // next_pow2(nb)
  int n2 = 1;
  while (n2 < nb) n2 <<= 1;
  float* sc = reinterpret_cast<float*>(keys + n2);           // nb
  float* u = sc + nb;                                        // D
  float* w = u + D;                                          // D
  float* t = w + D;                                          // D

  const float* qm = st.qmean + (bh * nb + i) * D;
  if (tid < D) {
    const float q = qm[tid];
    t[tid] = q;
    u[tid] = (mode == SA_ROUTE_TAYLOR2) ? scale * q : q;
    w[tid] = 0.5f * scale * scale * q * q;
  }
  __syncthreads();
  if (mode == SA_ROUTE_PROJ) {
    // t <- q̄ P_q ; u <- P_k t   so that (q̄P_q)·(k̄P_k) = k̄·u
    float a = 0.f;
    if (tid < D) {
      for (int r = 0; r < D; ++r) a = fmaf(t[r], Pq[(size_t)r * D + tid], a);
    }
    __syncthreads();
    if (tid < D) t[tid] = a;
    __syncthreads();
    if (tid < D) {
      float c = 0.f;
      const float* row = Pk + (size_t)tid * D;
      for (int e = 0; e < D; ++e) c = fmaf(row[e], t[e], c);
      u[tid] = c;
    }
    __syncthreads();
  }
  // scores: one warp per KV block; lanes split the channels
  constexpr int PER = D / 32;
  float uv[PER], wv[PER];
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    uv[p] = u[lane * PER + p];
    wv[p] = w[lane * PER + p];
  }
  const float* km = st.kmean + bh * nb * D;
  const float* kv = st.kvar ? st.kvar + bh * nb * D : nullptr;
  for (int j = warp; j < nb; j += kRouteThreads / 32) {
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int p = 0; p < PER; ++p) s1 = fmaf(uv[p], km[(size_t)j * D + lane * PER + p], s1);
    if (mode == SA_ROUTE_TAYLOR2) {
#pragma unroll
      for (int p = 0; p < PER; ++p) s2 = fmaf(wv[p], kv[(size_t)j * D + lane * PER + p], s2);
    }
    s1 = warp_sum(s1);
    if (mode == SA_ROUTE_TAYLOR2) s1 += log1pf(warp_sum(s2));
    if (lane == 0) sc[j] = s1;
  }
  __syncthreads();
  if (scores_out) {
    float* so = scores_out + (bh * nb + i) * (size_t)nb;
    for (int j = tid; j < nb; j += kRouteThreads) so[j] = sc[j];
  }
  block_topk_ascending(sc, nb, topk, keys, block_idx + (bh * nb + i) * (size_t)topk);
}

size_t route_smem_bytes(int nb, int d) {
  int n2 = 1;
  while (n2 < nb) n2 <<= 1;
  return (size_t)n2 * 8 + (size_t)nb * 4 + 3 * (size_t)d * 4;
}

}  // namespace
}  // namespace sa

extern "C" sa_status sa_route(const sa_block_stats* stats, sa_shape shape, sa_route_mode mode,
                              const float* proj_q, const float* proj_k, float scale,
                              int32_t topk, int32_t* block_idx, float* scores, void* stream) {
  using namespace sa;
  sa_status r = check_shape(shape, "sa_route");
  if (r != SA_OK) return r;
  const int nb = shape.N / shape.block;
  if (shape.N == 0 || shape.B == 0 || shape.H == 0) return SA_OK;  // nothing to compute
  if (!stats || !stats->qmean || !stats->kmean || (topk > 0 && !block_idx))
    return fail(SA_ERR_INVALID_ARG, "sa_route: stats->qmean, stats->kmean and block_idx are required");
  if (mode != SA_ROUTE_DOT && mode != SA_ROUTE_PROJ && mode != SA_ROUTE_TAYLOR2)
    return fail(SA_ERR_INVALID_ARG, "sa_route: unknown route mode");
  if (mode == SA_ROUTE_PROJ && (!proj_q || !proj_k))
    return fail(SA_ERR_INVALID_ARG, "sa_route: SA_ROUTE_PROJ needs proj_q and proj_k");
  if (mode == SA_ROUTE_TAYLOR2 && !stats->kvar)
    return fail(SA_ERR_INVALID_ARG, "sa_route: SA_ROUTE_TAYLOR2 needs stats->kvar");
  if (topk < 0 || topk > nb) return fail(SA_ERR_INVALID_ARG, "sa_route: topk must be in [0, N/block]");
  if (nb > kMaxRouteBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_route: at most 4096 blocks per head");
  const void* ptrs[] = {stats->qmean, stats->kmean, stats->kvar, proj_q, proj_k, block_idx, scores};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_route: pointers must be 16-byte aligned");
  const size_t smem = route_smem_bytes(nb, shape.d);
  dim3 grid(nb, shape.H, shape.B);
  cudaStream_t s = as_stream(stream);
  if (shape.d == 128) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    route_kernel<128><<<grid, kRouteThreads, smem, s>>>(*stats, shape.H, nb, mode, proj_q, proj_k,
                                                        scale, topk, block_idx, scores);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    route_kernel<64><<<grid, kRouteThreads, smem, s>>>(*stats, shape.H, nb, mode, proj_q, proj_k,
                                                       scale, topk, block_idx, scores);
  }
  return launch_status("route_kernel");
}
