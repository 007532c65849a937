// Router: block scores and top-k selection of KV blocks per query block.
//   dot      q̄_i·k̄_j                        (SLA2 §2B, mean pooling)
//   proj     (q̄_i P_q)·(k̄_j P_k)              (SLA2 §2B, learnable router)
//   taylor2  s q̄_i·k̄_j + log1p(½ s² Σ q̄²var)  (SPLA §2.1, log of the
//            second-order block score with diagonal covariance)
// The proj score (q̄_i P_q)·(k̄_j P_k) is evaluated as k̄_j·u_i with
// u_i = P_k P_qᵀ q̄_i (x P is the row vector x times P), so no projected copy
// of the key centroids is needed: u_i costs 2d² multiply-adds per query block.
//
// One CTA handles kRouteQB query blocks of one head (one warp each), so every
// centroid tile it stages in shared memory serves kRouteQB score rows.  Scores
// are computed with lane = KV block (a full dot product per lane against a
// padded shared-memory row).  Selection: for small k each warp takes its k
// winners by repeated warp arg-max over (score desc, index asc) keys, then
// emits them in ascending order from a bitmap; for large k the CTA sorts each
// row with a bitonic sort.
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteQB = kRouteThreads / 32;   // query blocks per CTA
constexpr int kRouteTile = 32;                 // centroids per shared-memory tile
constexpr int kWarpTopkMax = 64;               // largest k taken by the warp arg-max path

__device__ __forceinline__ unsigned long long rank_key(float score, int j) {
  // smaller key = better: higher score first, then smaller index
  return ((unsigned long long)(~order_key(score)) << 32) | (unsigned)j;
}

__device__ __forceinline__ unsigned long long warp_min_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w < v ? w : v;
  }
  return v;
}

template <int D>
__global__ void __launch_bounds__(kRouteThreads)
route_kernel(sa_block_stats st, int H, int nb, sa_route_mode mode, const float* __restrict__ Pq,
             const float* __restrict__ Pk, float scale, int topk, int32_t* __restrict__ block_idx,
             float* __restrict__ scores_out) {
  constexpr int KS = D + 1;
  const int h = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * kRouteQB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i = i0 + warp;                       // this warp's query block
  const bool has_row = i < nb;
  const size_t bh = (size_t)b * H + h;
  const bool t2 = mode == SA_ROUTE_TAYLOR2;

  extern __shared__ float rsm[];
  float* u = rsm;                                // [QB][D]  query vector per warp
  float* w = u + kRouteQB * D;                   // [QB][D]  ½ s² q̄² (taylor2) / scratch (proj)
  float* kt = w + kRouteQB * D;                  // [TILE][KS] centroid tile
  float* vt = kt + kRouteTile * KS;              // [TILE][KS] variance tile (taylor2)
  // the tile region doubles as the sort keys of the large-k path
  int tile_floats = 2 * kRouteTile * KS;
  if (topk > kWarpTopkMax) {
    int n2 = 1;
    while (n2 < nb) n2 <<= 1;
    if (2 * n2 > tile_floats) tile_floats = 2 * n2;
  }
  float* sc = kt + tile_floats;                  // [QB][nb] scores
  const int nwords = (nb + 31) >> 5;
  uint32_t* bits = reinterpret_cast<uint32_t*>(sc + (size_t)kRouteQB * nb);   // [QB][nwords]

  // ---- query vectors (one warp per query block)
  float* uw = u + warp * D;
  float* ww = w + warp * D;
  for (int c = lane; c < D; c += 32) {
    const float q = has_row ? st.qmean[(bh * nb + i) * D + c] : 0.f;
    uw[c] = t2 ? scale * q : q;
    ww[c] = 0.5f * scale * scale * q * q;
  }
  __syncwarp();
  if (mode == SA_ROUTE_PROJ) {
    // t = q̄ P_q (into ww), then u = P_k t
    float tq[D / 32];
#pragma unroll
    for (int p = 0; p < D / 32; ++p) {
      const int c = lane + 32 * p;
      float a = 0.f;
      for (int r = 0; r < D; ++r) a = fmaf(uw[r], __ldg(Pq + (size_t)r * D + c), a);
      tq[p] = a;
    }
    __syncwarp();
#pragma unroll
    for (int p = 0; p < D / 32; ++p) ww[lane + 32 * p] = tq[p];
    __syncwarp();
#pragma unroll
    for (int p = 0; p < D / 32; ++p) {
      const int rr = lane + 32 * p;
      const float* row = Pk + (size_t)rr * D;
      float a = 0.f;
      for (int e = 0; e < D; ++e) a = fmaf(__ldg(row + e), ww[e], a);
      tq[p] = a;
    }
    __syncwarp();
#pragma unroll
    for (int p = 0; p < D / 32; ++p) uw[lane + 32 * p] = tq[p];
    __syncwarp();
  }

  // ---- scores: tiles of 32 centroids shared by the CTA's warps
  const float* km = st.kmean + bh * (size_t)nb * D;
  const float* kv = t2 ? st.kvar + bh * (size_t)nb * D : nullptr;
  float* scw = sc + (size_t)warp * nb;
  for (int j0 = 0; j0 < nb; j0 += kRouteTile) {
    __syncthreads();
    for (int idx = tid; idx < kRouteTile * D; idx += kRouteThreads) {
      const int n = idx / D, c = idx % D;
      const int j = j0 + n;
      kt[n * KS + c] = j < nb ? km[(size_t)j * D + c] : 0.f;
      if (t2) vt[n * KS + c] = j < nb ? kv[(size_t)j * D + c] : 0.f;
    }
    __syncthreads();
    const int j = j0 + lane;
    float s1 = 0.f, s2 = 0.f;
    const float* kr = kt + lane * KS;
#pragma unroll 8
    for (int c = 0; c < D; ++c) s1 = fmaf(uw[c], kr[c], s1);
    if (t2) {
      const float* vr = vt + lane * KS;
#pragma unroll 8
      for (int c = 0; c < D; ++c) s2 = fmaf(ww[c], vr[c], s2);
      s1 += log1pf(s2);
    }
    if (j < nb) scw[j] = s1;
  }
  __syncwarp();
  if (has_row && scores_out) {
    float* so = scores_out + (bh * nb + i) * (size_t)nb;
    for (int j = lane; j < nb; j += 32) so[j] = scw[j];
  }

  // ---- selection
  if (topk <= kWarpTopkMax) {
    uint32_t* bw = bits + (size_t)warp * nwords;
    for (int x = lane; x < nwords; x += 32) bw[x] = 0u;
    __syncwarp();
    if (has_row) {
      // repeated arg-max: round r takes the best key strictly worse than the
      // previous round's winner (keys are distinct: they carry the index)
      unsigned long long prev = 0ull;
      for (int r = 0; r < topk; ++r) {
        unsigned long long mine = ~0ull;
        for (int j = lane; j < nb; j += 32) {
          const unsigned long long k = rank_key(scw[j], j);
          if ((r == 0 || k > prev) && k < mine) mine = k;
        }
        const unsigned long long best = warp_min_u64(mine);
        if (lane == 0) {
          const int jb = (int)(best & 0xffffffffu);
          bw[jb >> 5] |= 1u << (jb & 31);
        }
        prev = best;
      }
      __syncwarp();
      // ascending emission from the bitmap
      int32_t* out = block_idx + (bh * nb + i) * (size_t)topk;
      int base = 0;
      for (int x0 = 0; x0 < nwords; x0 += 32) {
        const int x = x0 + lane;
        const uint32_t word = x < nwords ? bw[x] : 0u;
        const int cnt = __popc(word);
        int pre = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, pre, o);
          if (lane >= o) pre += y;
        }
        int pos = base + pre - cnt;
        uint32_t m = word;
        while (m) {
          const int bpos = __ffs(m) - 1;
          out[pos++] = x * 32 + bpos;
          m &= m - 1;
        }
        base += __shfl_sync(0xffffffffu, pre, 31);
      }
    }
  } else {
    // large k: each row in turn is sorted by the whole CTA
    __syncthreads();
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(kt);   // reuses the tile space
    for (int q = 0; q < kRouteQB && i0 + q < nb; ++q)
      block_topk_ascending(sc + (size_t)q * nb, nb, topk, keys,
                           block_idx + (bh * nb + i0 + q) * (size_t)topk);
  }
}

size_t route_smem_bytes(int nb, int d, int topk) {
  const int nwords = (nb + 31) / 32;
  size_t tiles = 2 * (size_t)kRouteTile * (d + 1) * 4;
  if (topk > kWarpTopkMax) {
    int n2 = 1;
    while (n2 < nb) n2 <<= 1;
    if ((size_t)n2 * 8 > tiles) tiles = (size_t)n2 * 8;
  }
  return 2 * (size_t)kRouteQB * d * 4 + tiles + (size_t)kRouteQB * nb * 4 + (size_t)kRouteQB * nwords * 4;
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
  const size_t smem = route_smem_bytes(nb, shape.d, topk);
  dim3 grid((nb + kRouteQB - 1) / kRouteQB, shape.H, shape.B);
  cudaStream_t s = as_stream(stream);
  if (shape.d == 128) {
    if (cudaFuncSetAttribute(route_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(route_kernel)");
    route_kernel<128><<<grid, kRouteThreads, smem, s>>>(*stats, shape.H, nb, mode, proj_q, proj_k,
                                                        scale, topk, block_idx, scores);
  } else {
    if (cudaFuncSetAttribute(route_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(route_kernel)");
    route_kernel<64><<<grid, kRouteThreads, smem, s>>>(*stats, shape.H, nb, mode, proj_q, proj_k,
                                                       scale, topk, block_idx, scores);
  }
  return launch_status("route_kernel");
}
