// Block statistics: the pre-computation step of PISA ("Implementação de
// Hardware": block centroids and value sums), the mean pooling of SLA2's
// router (§2B) and the block mean / diagonal covariance of SPLA's score
// (§2.1).  HBM-bound: every input element is read once with 16-byte loads.
#include "attn_simt.cuh"

namespace sa {
namespace {

constexpr int kPoolThreads = 256;

// One CTA per (block j, head h, batch b).  Thread t covers the 8 channels
// [8*(t % COLS), +8) of rows t / COLS, t / COLS + RPP, ...  Means are reduced
// through shared memory; the key variance is the exact two-pass form over the
// register-resident block.
template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kPoolThreads)
block_pool_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                  int H, int N, sa_block_stats st) {
  constexpr int COLS = D / 8;                 // 16-byte vectors per row
  constexpr int RPP = kPoolThreads / COLS;    // rows per pass
  constexpr int ROWS = BLK / RPP;             // rows per thread
  static_assert(BLK % RPP == 0, "block must be a multiple of rows per pass");
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = N / BLK;
  const int tid = threadIdx.x;
  const int col = tid % COLS, r0 = tid / COLS;
  const size_t head_off = ((size_t)b * H + h) * (size_t)N * D;
  const size_t row0 = (size_t)j * BLK;
  const size_t stat_off = (((size_t)b * H + h) * nb + j) * D;
  // launched with programmatic stream serialization: wait for the previous
  // launch (which may still read the statistics this kernel rewrites), then
  // let the next launch on the stream (the router) schedule its CTAs
  pdl_wait();
  pdl_trigger();

  __shared__ float red[RPP][D];
  __shared__ float mean_sh[D];

  auto reduce_rows = [&](float acc[8]) {
    // sums acc over the RPP threads that share a column; result for channel
    // c is left in red[0][c]
#pragma unroll
    for (int i = 0; i < 8; ++i) red[r0][col * 8 + i] = acc[i];
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
#pragma unroll 8
      for (int r = 0; r < RPP; ++r) s += red[r][tid];
      mean_sh[tid] = s;
    }
    __syncthreads();
  };

  float x[ROWS][8];
  // ---- keys: mean, variance, relu sums
  {
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      load8<T>(K + head_off + (row0 + r0 + r * RPP) * D + col * 8, x[r]);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < ROWS; ++r) s += x[r][i];
      acc[i] = s;
    }
    reduce_rows(acc);
    const float inv = 1.0f / BLK;
    float mu[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mu[i] = mean_sh[col * 8 + i] * inv;
    if (tid < D) {
      const float m = mean_sh[tid] * inv;
      st.kmean[stat_off + tid] = m;
      if (st.kmean_bf16)
        reinterpret_cast<__nv_bfloat16*>(st.kmean_bf16)[stat_off + tid] = __float2bfloat16_rn(m);
    }
    __syncthreads();
    if (st.kvar || st.kvar_bf16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
          const float dlt = x[r][i] - mu[i];
          s = fmaf(dlt, dlt, s);
        }
        acc[i] = s;
      }
      reduce_rows(acc);
      if (tid < D) {
        const float v = mean_sh[tid] * inv;
        if (st.kvar) st.kvar[stat_off + tid] = v;
        if (st.kvar_bf16) reinterpret_cast<__nv_bfloat16*>(st.kvar_bf16)[stat_off + tid] = __float2bfloat16_rn(v);
      }
      __syncthreads();
    }
    if (st.zrelu) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) s += fmaxf(x[r][i], 0.f);
        acc[i] = s;
      }
      reduce_rows(acc);
      if (tid < D) st.zrelu[stat_off + tid] = mean_sh[tid];
      __syncthreads();
    }
  }
  // ---- values: block sums
  {
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      load8<T>(V + head_off + (row0 + r0 + r * RPP) * D + col * 8, x[r]);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < ROWS; ++r) s += x[r][i];
      acc[i] = s;
    }
    reduce_rows(acc);
    if (tid < D) {
      st.vsum[stat_off + tid] = mean_sh[tid];
      if (st.vmean_bf16)
        reinterpret_cast<__nv_bfloat16*>(st.vmean_bf16)[stat_off + tid] =
            __float2bfloat16_rn(mean_sh[tid] * (1.0f / BLK));
    }
    __syncthreads();
  }
  // ---- queries: block means (query blocks have the same size as KV blocks)
  if (Q != nullptr && st.qmean != nullptr) {
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      load8<T>(Q + head_off + (row0 + r0 + r * RPP) * D + col * 8, x[r]);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < ROWS; ++r) s += x[r][i];
      acc[i] = s;
    }
    reduce_rows(acc);
    if (tid < D) st.qmean[stat_off + tid] = mean_sh[tid] * (1.0f / BLK);
  }
}

// One chunk of tokens per CTA adds its d×d outer-product sum Σ_n f(k_n) v_nᵀ
// to out[b,h]:
//   kFeatRelu:   f(k) = relu(k), and ztot[b,h] += Σ relu(k_n) — the totals of
//                the SLA2/SALAD linear branch;
//   kFeatCentre: f(k_n) = k_n − k̄_j for the block j of BLK tokens that holds
//                n, each chunk's sum scaled by oscale = 1/nb — PISA's mean
//                first-order statistic H̄ (§2 "Algoritmo Central");
//   kFeatExp:    f(k) = exp(k) — the all-token state of SPLA's residual
//                linear attention (§2.2-2.3).
// Thread t owns row c = t / (256/D) of the d×d sum and D*D/256 of its columns.
constexpr int kLinChunk = 1024;
constexpr int kLinTile = 32;

enum { kFeatRelu = 0, kFeatCentre = 1, kFeatExp = 2 };

template <typename T, int D, int FEAT, int BLK = 1>
__global__ void __launch_bounds__(256)
linear_totals_kernel(const T* __restrict__ K, const T* __restrict__ V, int H, int N,
                     float* __restrict__ htot, float* __restrict__ ztot,
                     const float* __restrict__ kmean = nullptr, float oscale = 1.f) {
  static_assert(kLinChunk % BLK == 0, "a chunk holds whole blocks");
  constexpr int TPR = 256 / D;       // threads per output row
  constexpr int CPT = D / TPR;       // columns per thread
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t head_off = ((size_t)b * H + h) * (size_t)N * D;
  const int tid = threadIdx.x;
  const int c = tid / TPR, e0 = (tid % TPR) * CPT;
  __shared__ float ks[kLinTile][D];
  __shared__ float vs[kLinTile][D];
  float acc[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
  float z = 0.f;
  const int n_begin = chunk * kLinChunk;
  const int n_end = min(N, n_begin + kLinChunk);
  for (int n0 = n_begin; n0 < n_end; n0 += kLinTile) {
    __syncthreads();
    for (int idx = tid; idx < kLinTile * D; idx += 256) {
      const int r = idx / D, cc = idx % D;
      const int n = n0 + r;
      float kv = 0.f, vv = 0.f;
      if (n < n_end) {
        kv = to_f<T>(K[head_off + (size_t)n * D + cc]);
        vv = to_f<T>(V[head_off + (size_t)n * D + cc]);
        if (FEAT == kFeatCentre) kv -= kmean[(((size_t)b * H + h) * (N / BLK) + n / BLK) * D + cc];
        if (FEAT == kFeatExp) kv = phi_exp(kv);
      }
      ks[r][cc] = FEAT == kFeatRelu ? fmaxf(kv, 0.f) : kv;
      vs[r][cc] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < kLinTile; ++r) {
      const float kr = ks[r][c];
      if (FEAT == kFeatRelu && e0 == 0) z += kr;
#pragma unroll
      for (int i = 0; i < CPT; ++i) acc[i] = fmaf(kr, vs[r][e0 + i], acc[i]);
    }
  }
  float* hp = htot + ((size_t)b * H + h) * D * D + (size_t)c * D + e0;
#pragma unroll
  for (int i = 0; i < CPT; ++i) atomicAdd(hp + i, acc[i] * oscale);
  if (FEAT == kFeatRelu && e0 == 0) atomicAdd(ztot + ((size_t)b * H + h) * D + c, z);
}

// bf16 copy of H̄ᵀ: out[b,h][e][c] = H̄[b,h][c][e] (the B operand of the
// tensor-core S' = Q H̄, which wants the reduced index c innermost).
template <int D>
__global__ void hbar_transpose_kernel(const float* __restrict__ hbar, __nv_bfloat16* __restrict__ out) {
  __shared__ float t[32][33];
  const size_t off = (size_t)blockIdx.z * D * D;
  const int c0 = blockIdx.y * 32, e0 = blockIdx.x * 32;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) t[y][threadIdx.x] = hbar[off + (size_t)(c0 + y) * D + e0 + threadIdx.x];
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y)
    out[off + (size_t)(e0 + y) * D + c0 + threadIdx.x] = __float2bfloat16_rn(t[threadIdx.x][y]);
}

// z_tot = Σ_j zrelu_j over the head's blocks (one thread per channel).
template <int D>
__global__ void ztot_from_blocks_kernel(const float* __restrict__ zrelu, int H, int nb, float* __restrict__ ztot) {
  const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  const float* z = zrelu + ((size_t)b * H + h) * nb * D + c;
  float acc = 0.f;
  for (int j = 0; j < nb; ++j) acc += z[(size_t)j * D];
  ztot[((size_t)b * H + h) * D + c] = acc;
}

// M_j = ‖H_j − H̄‖₂ of one block per CTA on CUDA cores (every shape; the
// tensor-core kernel in cov_tc.cu takes bf16 with d = block = 128): the CTA
// accumulates A = Σ_n (k_n − k̄_j) v_nᵀ − H̄ in shared memory (thread t owns
// row t / (256/D) and D·D/256 of its columns), then runs the power iteration
// x ← Aᵀ A x / ‖Aᵀ A x‖ until the Rayleigh quotient ‖A x‖² / ‖x‖² changes by
// less than 1e-6 (relative) or 256 steps have run; M_j is its square root.
constexpr int kCovSteps = 256;

template <typename T, int D, int BLK>
__global__ void __launch_bounds__(256)
covnorm_simt_kernel(const T* __restrict__ K, const T* __restrict__ V, int H, int N,
                    const float* __restrict__ kmean, const float* __restrict__ hbar, float* __restrict__ covnorm) {
  constexpr int TPR = 256 / D;       // threads per row
  constexpr int CPT = D / TPR;       // columns per thread
  constexpr int AS = D + 1;          // padded row of A
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = N / BLK;
  const size_t bh = (size_t)b * H + h;
  const size_t head_off = bh * (size_t)N * D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid / TPR, e0 = (tid % TPR) * CPT;
  extern __shared__ float cs[];
  float* A = cs;                          // [D][AS]
  float* ks = A + D * AS;                 // [kLinTile][D]
  float* vs = ks + kLinTile * D;          // [kLinTile][D]
  float* x = vs + kLinTile * D;           // [D]
  float* y = x + D;                       // [D]
  float* red = y + D;                     // [2][8 warps][3]

  const float* km = kmean + (bh * nb + j) * D;
  float acc[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) acc[i] = 0.f;
  for (int n0 = 0; n0 < BLK; n0 += kLinTile) {
    __syncthreads();
    for (int idx = tid; idx < kLinTile * D; idx += 256) {
      const int r = idx / D, cc = idx % D;
      const size_t g = head_off + ((size_t)j * BLK + n0 + r) * D + cc;
      ks[idx] = to_f<T>(K[g]) - km[cc];
      vs[idx] = to_f<T>(V[g]);
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < kLinTile; ++r) {
      const float kr = ks[r * D + c];
#pragma unroll
      for (int i = 0; i < CPT; ++i) acc[i] = fmaf(kr, vs[r * D + e0 + i], acc[i]);
    }
  }
  const float* hb = hbar + (bh * D + c) * D;
#pragma unroll
  for (int i = 0; i < CPT; ++i) A[c * AS + e0 + i] = acc[i] - hb[e0 + i];
  for (int i = tid; i < D; i += 256) x[i] = 0.5f + (float)((((uint32_t)i * 2654435761u) >> 24) & 0xffu) * (1.0f / 256.0f);
  __syncthreads();

  float lam = 0.f, lam_prev = -1.f;
  for (int it = 0; it < kCovSteps; ++it) {
    // y = A x (rows split over TPR adjacent lanes), with ‖y‖² and ‖x‖²
    float py = 0.f;
#pragma unroll
    for (int i = 0; i < CPT; ++i) py = fmaf(A[c * AS + e0 + i], x[e0 + i], py);
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) py += __shfl_xor_sync(0xffffffffu, py, o);
    if (e0 == 0) y[c] = py;
    float p1 = (e0 == 0) ? py * py : 0.f;
    float p3 = (tid < D) ? x[tid] * x[tid] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      p1 += __shfl_xor_sync(0xffffffffu, p1, o);
      p3 += __shfl_xor_sync(0xffffffffu, p3, o);
    }
    const int rb = (it & 1) * 16;
    if (lane == 0) {
      red[rb + 2 * warp] = p1;
      red[rb + 2 * warp + 1] = p3;
    }
    __syncthreads();
    float S1 = 0.f, S3 = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      S1 += red[rb + 2 * w];
      S3 += red[rb + 2 * w + 1];
    }
    lam = S3 > 0.f ? S1 / S3 : 0.f;
    if (!(S1 > 0.f) || fabsf(lam - lam_prev) <= 1e-6f * lam) break;
    lam_prev = lam;
    // x = Aᵀ y / ‖Aᵀ y‖ scaled only by ‖y‖ (the quotient ignores the scale):
    // column e of A over its D rows, thread t covering columns t, t + 256 ...
    const float inv = rsqrtf(S1);
    float z = 0.f;
    if (tid < D) {
      for (int r = 0; r < D; ++r) z = fmaf(A[r * AS + tid], y[r], z);
    }
    __syncthreads();
    if (tid < D) x[tid] = z * inv;
    __syncthreads();
  }
  if (tid == 0) covnorm[bh * nb + j] = sqrtf(fmaxf(lam, 0.f));
}

template <typename T, int D, int BLK>
sa_status launch_pool(const void* Q, const void* K, const void* V, const sa_shape& s,
                      const sa_block_stats& st, cudaStream_t stream) {
  dim3 grid(s.N / BLK, s.H, s.B);
  const cudaError_t le = launch_pdl(block_pool_kernel<T, D, BLK>, grid, dim3(kPoolThreads), 0, stream,
                                    static_cast<const T*>(Q), static_cast<const T*>(K), static_cast<const T*>(V),
                                    s.H, s.N, st);
  if (le != cudaSuccess) return fail(SA_ERR_CUDA, std::string("block_pool_kernel: ") + cudaGetErrorString(le));
  sa_status r = launch_status("block_pool_kernel");
  if (r != SA_OK) return r;
  if (st.htot || st.ztot) {
    const size_t hbytes = (size_t)s.B * s.H * s.d * s.d * sizeof(float);
    const size_t zbytes = (size_t)s.B * s.H * s.d * sizeof(float);
    if (cudaMemsetAsync(st.htot, 0, hbytes, stream) != cudaSuccess ||
        cudaMemsetAsync(st.ztot, 0, zbytes, stream) != cudaSuccess)
      return launch_status("cudaMemsetAsync(htot/ztot)");
    // bf16, d = 128: H_tot on the tensor cores and z_tot from the block sums
    if (sizeof(T) == 2 && D == 128 && st.zrelu &&
        kv_outer_tc(K, V, s, kKvRelu, nullptr, nullptr, 1.f, st.htot, stream) == SA_OK) {
      ztot_from_blocks_kernel<D><<<dim3(s.H, s.B), D, 0, stream>>>(st.zrelu, s.H, s.N / BLK, st.ztot);
      return launch_status("ztot_from_blocks_kernel");
    }
    dim3 g2((s.N + kLinChunk - 1) / kLinChunk, s.H, s.B);
    linear_totals_kernel<T, D, kFeatRelu><<<g2, 256, 0, stream>>>(
        static_cast<const T*>(K), static_cast<const T*>(V), s.H, s.N, st.htot, st.ztot);
    r = launch_status("linear_totals_kernel");
    if (r != SA_OK) return r;
  }
  if (st.sexp) {
    // SPLA's all-token state Σ_n exp(k_n) v_nᵀ
    const size_t hbytes = (size_t)s.B * s.H * s.d * s.d * sizeof(float);
    if (cudaMemsetAsync(st.sexp, 0, hbytes, stream) != cudaSuccess) return launch_status("cudaMemsetAsync(sexp)");
    if (!(sizeof(T) == 2 && D == 128 && kv_outer_tc(K, V, s, kKvExp, nullptr, nullptr, 1.f, st.sexp, stream) == SA_OK)) {
      dim3 g2((s.N + kLinChunk - 1) / kLinChunk, s.H, s.B);
      linear_totals_kernel<T, D, kFeatExp><<<g2, 256, 0, stream>>>(
          static_cast<const T*>(K), static_cast<const T*>(V), s.H, s.N, st.sexp, nullptr);
      r = launch_status("linear_totals_kernel(sexp)");
      if (r != SA_OK) return r;
    }
  }
  if (st.hbar) {
    // PISA's H̄ from the block centroids written above (same stream)
    const size_t hbytes = (size_t)s.B * s.H * s.d * s.d * sizeof(float);
    if (cudaMemsetAsync(st.hbar, 0, hbytes, stream) != cudaSuccess) return launch_status("cudaMemsetAsync(hbar)");
    const float inv_nb = 1.0f / (float)(s.N / BLK);
    if (!(sizeof(T) == 2 && D == 128 && BLK == 128 &&
          kv_outer_tc(K, V, s, kKvCentre, st.kmean, st.vsum, inv_nb, st.hbar, stream) == SA_OK)) {
      dim3 g2((s.N + kLinChunk - 1) / kLinChunk, s.H, s.B);
      linear_totals_kernel<T, D, kFeatCentre, BLK><<<g2, 256, 0, stream>>>(
          static_cast<const T*>(K), static_cast<const T*>(V), s.H, s.N, st.hbar, nullptr, st.kmean, inv_nb);
      r = launch_status("linear_totals_kernel(hbar)");
      if (r != SA_OK) return r;
    }
    if (st.hbarT_bf16) {
      hbar_transpose_kernel<D><<<dim3(D / 32, D / 32, s.B * s.H), dim3(32, 8), 0, stream>>>(
          st.hbar, reinterpret_cast<__nv_bfloat16*>(st.hbarT_bf16));
      r = launch_status("hbar_transpose_kernel");
      if (r != SA_OK) return r;
    }
    if (st.covnorm) {
      // PISA's M_j from the H̄ just written (same stream)
      if (sizeof(T) == 2 && D == 128 && BLK == 128 &&
          covnorm_tc(K, V, s, st.kmean, st.vsum, st.hbar, st.covnorm, stream) == SA_OK)
        return SA_OK;
      const size_t smem = sizeof(float) * ((size_t)D * (D + 1) + 2 * (size_t)kLinTile * D + 2 * D + 32);
      auto kern = covnorm_simt_kernel<T, D, BLK>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return launch_status("cudaFuncSetAttribute(covnorm_simt_kernel)");
      kern<<<dim3(s.N / BLK, s.H, s.B), 256, smem, stream>>>(
          static_cast<const T*>(K), static_cast<const T*>(V), s.H, s.N, st.kmean, st.hbar, st.covnorm);
      r = launch_status("covnorm_simt_kernel");
    }
  }
  return r;
}

template <typename T>
sa_status dispatch_pool(const void* Q, const void* K, const void* V, const sa_shape& s,
                        const sa_block_stats& st, cudaStream_t stream) {
  if (s.d == 128 && s.block == 128) return launch_pool<T, 128, 128>(Q, K, V, s, st, stream);
  if (s.d == 128 && s.block == 64) return launch_pool<T, 128, 64>(Q, K, V, s, st, stream);
  if (s.d == 64 && s.block == 128) return launch_pool<T, 64, 128>(Q, K, V, s, st, stream);
  if (s.d == 64 && s.block == 64) return launch_pool<T, 64, 64>(Q, K, V, s, st, stream);
  return fail(SA_ERR_UNSUPPORTED, "sa_block_pool: d and block must be 64 or 128");
}

}  // namespace
}  // namespace sa

extern "C" sa_status sa_block_pool(const void* Q, const void* K, const void* V, sa_dtype dtype,
                                   sa_shape shape, const sa_block_stats* stats, void* stream) {
  using namespace sa;
  sa_status r = check_shape(shape, "sa_block_pool");
  if (r != SA_OK) return r;
  if (shape.N == 0 || shape.B == 0 || shape.H == 0) return SA_OK;  // nothing to compute
  if (!K || !V || !stats || !stats->kmean || !stats->vsum)
    return fail(SA_ERR_INVALID_ARG, "sa_block_pool: K, V, stats, stats->kmean and stats->vsum are required");
  if ((stats->htot == nullptr) != (stats->ztot == nullptr))
    return fail(SA_ERR_INVALID_ARG, "sa_block_pool: htot and ztot go together");
  if ((stats->hbarT_bf16 || stats->covnorm) && !stats->hbar)
    return fail(SA_ERR_INVALID_ARG, "sa_block_pool: hbarT_bf16 and covnorm need hbar");
  const void* ptrs[] = {Q, K, V, stats->qmean, stats->kmean, stats->vsum, stats->kvar,
                        stats->zrelu, stats->htot, stats->ztot, stats->kmean_bf16, stats->vmean_bf16,
                        stats->hbar, stats->hbarT_bf16, stats->covnorm, stats->sexp, stats->kvar_bf16};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_block_pool: pointers must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  if (dtype == SA_BF16) return dispatch_pool<__nv_bfloat16>(Q, K, V, shape, *stats, s);
  if (dtype == SA_FP32) return dispatch_pool<float>(Q, K, V, shape, *stats, s);
  return fail(SA_ERR_UNSUPPORTED, "sa_block_pool: dtype must be SA_FP32 or SA_BF16");
}
