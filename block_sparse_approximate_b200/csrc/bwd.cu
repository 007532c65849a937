// Backward of the sparse prefill for the drop and zero-order tails, on CUDA
// cores (fp32 arithmetic; Q, K, V, O, dO of the forward's dtype; dQ, dK, dV
// fp32): the general path (fp32, d = 64), and the parity reference of the
// tensor-core kernels in bwd_mma.cu, which take bf16 with d = 128.  The forward is softmax attention of query block i to the key list
// [k_n, n ∈ S_i] + [k̄_j, j ∈ U_i] with logit biases 0 / ln B and values v_n /
// v̄_j = vsum_j / B (PISA "Algoritmo Central"), so the gradients are
//   p = exp(s q·k + bias − lse),  δ_t = dO_t·o_t,  ds = p (dO·v − δ),
//   dQ = s Σ ds k,  dK_key = s Σ ds q,  dV_key = Σ p dO,
// and a pseudo-key's gradients reach the tokens of its block divided by B.
// Five launches:
//   bwd_stats_kernel     lse (log2 domain) and δ per query row;
//   bwd_transpose_kernel per KV block, the query blocks that selected it
//                        (ascending, so every sum below has a fixed order);
//   bwd_dq_kernel        dQ per query row over its exact and centroid keys;
//   bwd_dkv_kernel       dK, dV of every key over the query blocks that
//                        selected its block (written, not accumulated);
//   bwd_centroid_kernel  (zero-order) dk̄_j, dv̄_j over every query row whose
//                        block left j unselected, added to the block's tokens.
#include "attn_simt.cuh"

namespace sa {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kBwdRows = 64;                    // query rows per CTA (stats, dQ)
constexpr int kBwdRpw = kBwdRows / kBwdWarps;   // rows per warp
constexpr int kBwdKT = 32;                      // keys per staged tile

// Stages a tile of kBwdKT keys (rows [row0, row0 + n) of src, [.][D] of T,
// or fp32 statistics scaled by `mul`) into dst [kBwdKT][D + 4] (the padding
// keeps 16-byte rows and spreads the lanes' rows over the banks); missing
// rows are zero.
template <typename T, int D>
__device__ __forceinline__ void stage_keys(float* dst, const T* src, int row0, int n, float mul = 1.f) {
  for (int x = threadIdx.x; x < kBwdKT * D; x += kBwdThreads) {
    const int r = x / D, c = x % D;
    dst[r * (D + 4) + c] = r < n ? to_f<T>(src[(size_t)(row0 + r) * D + c]) * mul : 0.f;
  }
}

// selection bitmap of one query block into sel_bits (nwords words)
__device__ __forceinline__ void load_selection(uint32_t* sel_bits, int nwords, const int32_t* sel, int topk) {
  for (int w = threadIdx.x; w < nwords; w += kBwdThreads) sel_bits[w] = 0u;
  __syncthreads();
  for (int s = threadIdx.x; s < topk; s += kBwdThreads) atomicOr(&sel_bits[sel[s] >> 5], 1u << (sel[s] & 31));
  __syncthreads();
}

// ---- lse and δ per query row ---------------------------------------------
// One CTA per 64 query rows (warp = 8 rows, lane = key of the staged tile).
template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads)
bwd_stats_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ O,
                 const T* __restrict__ dO, int H, int N, const int32_t* __restrict__ block_idx, int topk,
                 int zo, const float* __restrict__ kmean, float scale2, float* __restrict__ lse2,
                 float* __restrict__ delta) {
  constexpr int PER = D / 32;
  const int nb = N / BLK;
  const int row0 = blockIdx.x * kBwdRows, i = row0 / BLK;
  const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
  const size_t head = bh * (size_t)N * D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwords = (nb + 31) >> 5;
  extern __shared__ float bsm[];
  float* qs = bsm;                                   // [64][D]
  float* ks = qs + kBwdRows * D;                     // [KT][D + 4]
  uint32_t* sel_bits = reinterpret_cast<uint32_t*>(ks + kBwdKT * (D + 4));
  for (int x = tid; x < kBwdRows * D; x += kBwdThreads) qs[x] = to_f<T>(Q[head + (size_t)row0 * D + x]);
  const int32_t* sel = block_idx + (bh * nb + i) * (size_t)topk;
  load_selection(sel_bits, nwords, sel, topk);
  float m[kBwdRpw], l[kBwdRpw];
#pragma unroll
  for (int r = 0; r < kBwdRpw; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
  }
  const int pe = topk * (BLK / kBwdKT), pc = zo ? (nb + kBwdKT - 1) / kBwdKT : 0;
  const float bias_c = log2f((float)BLK);
  for (int piece = 0; piece < pe + pc; ++piece) {
    __syncthreads();
    bool valid;
    float bias = 0.f;
    if (piece < pe) {
      const int j = sel[piece / (BLK / kBwdKT)];
      stage_keys<T, D>(ks, K + head, j * BLK + (piece % (BLK / kBwdKT)) * kBwdKT, kBwdKT);
      valid = true;
    } else {
      const int j0 = (piece - pe) * kBwdKT, j = j0 + lane;
      stage_keys<float, D>(ks, kmean + bh * (size_t)nb * D, j0, min(kBwdKT, nb - j0));
      valid = j < nb && !((sel_bits[j >> 5] >> (j & 31)) & 1u);
      bias = bias_c;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kBwdRpw; ++r) {
      const float* qr = qs + (warp * kBwdRpw + r) * D;
      const float* kr = ks + lane * (D + 4);
      float x = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 a = *reinterpret_cast<const float4*>(qr + c), k4 = *reinterpret_cast<const float4*>(kr + c);
        x = fmaf(a.x, k4.x, x);
        x = fmaf(a.y, k4.y, x);
        x = fmaf(a.z, k4.z, x);
        x = fmaf(a.w, k4.w, x);
      }
      x = valid ? fmaf(x, scale2, bias) : -INFINITY;
      const float tmax = warp_max(x);
      if (tmax == -INFINITY) continue;
      const float mn = fmaxf(m[r], tmax);
      const float ps = warp_sum(fast_exp2(x - mn));
      l[r] = l[r] * (m[r] == -INFINITY ? 0.f : fast_exp2(m[r] - mn)) + ps;
      m[r] = mn;
    }
  }
#pragma unroll
  for (int r = 0; r < kBwdRpw; ++r) {
    const int row = row0 + warp * kBwdRpw + r;
    float dd = 0.f;
#pragma unroll
    for (int c = 0; c < PER; ++c) {
      const size_t g = head + (size_t)row * D + lane * PER + c;
      dd = fmaf(to_f<T>(dO[g]), to_f<T>(O[g]), dd);
    }
    dd = warp_sum(dd);
    if (lane == 0) {
      lse2[bh * N + row] = l[r] > 0.f ? m[r] + log2f(l[r]) : INFINITY;   // no keys: p = 0
      delta[bh * N + row] = dd;
    }
  }
}

// ---- query blocks that selected each KV block ------------------------------
// One CTA per (batch, head): offs[j] .. offs[j + 1] index list[], which holds
// the query blocks i with j ∈ S_i in ascending order (rows of block_idx are
// ascending, so membership is a binary search).
__global__ void __launch_bounds__(kBwdThreads)
bwd_transpose_kernel(const int32_t* __restrict__ block_idx, int nb, int topk, int32_t* __restrict__ offs,
                     int32_t* __restrict__ list) {
  const size_t bh = blockIdx.x;
  const int32_t* idx = block_idx + bh * (size_t)nb * topk;
  int32_t* off = offs + bh * (size_t)(nb + 1);
  int32_t* lst = list + bh * (size_t)nb * topk;
  auto member = [&](int i, int j) {
    const int32_t* row = idx + (size_t)i * topk;
    int lo = 0, hi = topk;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (row[mid] < j) lo = mid + 1;
      else hi = mid;
    }
    return lo < topk && row[lo] == j;
  };
  for (int j = threadIdx.x; j < nb; j += kBwdThreads) {
    int c = 0;
    for (int i = 0; i < nb; ++i) c += member(i, j);
    off[j + 1] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    off[0] = 0;
    for (int j = 0; j < nb; ++j) off[j + 1] += off[j];
  }
  __syncthreads();
  for (int j = threadIdx.x; j < nb; j += kBwdThreads) {
    int p = off[j];
    for (int i = 0; i < nb; ++i)
      if (member(i, j)) lst[p++] = i;
  }
}

// The same lists from a selection bitmap in shared memory (nb ≤ 1024: at
// most 128 KB): bit (i, j) set for j ∈ S_i, then one thread per KV block j
// counts its column, a warp scans the counts, and each thread writes its
// column's query blocks in ascending order.
constexpr int kTrThreads = 1024;
constexpr int kTrMaxBlocks = 1024;
__global__ void __launch_bounds__(kTrThreads)
bwd_transpose_bitmap_kernel(const int32_t* __restrict__ block_idx, int nb, int topk, int32_t* __restrict__ offs,
                            int32_t* __restrict__ list) {
  extern __shared__ uint32_t trs[];
  const int W = (nb + 31) >> 5;
  uint32_t* bm = trs;                                                 // [nb][W]
  int32_t* cnt = reinterpret_cast<int32_t*>(trs + (size_t)nb * W);    // [nb]
  const size_t bh = blockIdx.x;
  const int32_t* idx = block_idx + bh * (size_t)nb * topk;
  int32_t* off = offs + bh * (size_t)(nb + 1);
  int32_t* lst = list + bh * (size_t)nb * topk;
  for (int x = threadIdx.x; x < nb * W; x += blockDim.x) bm[x] = 0u;
  __syncthreads();
  for (int e = threadIdx.x; e < nb * topk; e += blockDim.x) {
    const int i = e / topk, j = idx[e];
    if ((unsigned)j < (unsigned)nb) atomicOr(&bm[i * W + (j >> 5)], 1u << (j & 31));
  }
  __syncthreads();
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    int c = 0;
    for (int i = 0; i < nb; ++i) c += (bm[i * W + (j >> 5)] >> (j & 31)) & 1u;
    cnt[j] = c;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // exclusive scan: lane l sums a contiguous chunk, the warp scans the sums
    const int lane = threadIdx.x, per = (nb + 31) / 32;
    const int a = min(nb, lane * per), b = min(nb, a + per);
    int sum = 0;
    for (int x = a; x < b; ++x) sum += cnt[x];
    int incl = sum;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
    for (int x = a; x < b; ++x) {
      const int c = cnt[x];
      cnt[x] = run;
      off[x] = run;
      run += c;
    }
    if (lane == 31) off[nb] = incl;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    int p = cnt[j];
    for (int i = 0; i < nb; ++i)
      if ((bm[i * W + (j >> 5)] >> (j & 31)) & 1u) lst[p++] = i;
  }
}

sa_status launch_transpose(const int32_t* block_idx, int nb, int topk, int32_t* offs, int32_t* list, int BH,
                           cudaStream_t stream) {
  if (nb <= kTrMaxBlocks) {
    const size_t smem = sizeof(uint32_t) * ((size_t)nb * ((nb + 31) / 32) + nb);
    if (cudaFuncSetAttribute(bwd_transpose_bitmap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return launch_status("cudaFuncSetAttribute(bwd_transpose_bitmap_kernel)");
    bwd_transpose_bitmap_kernel<<<BH, kTrThreads, smem, stream>>>(block_idx, nb, topk, offs, list);
    return launch_status("bwd_transpose_bitmap_kernel");
  }
  bwd_transpose_kernel<<<BH, kBwdThreads, 0, stream>>>(block_idx, nb, topk, offs, list);
  return launch_status("bwd_transpose_kernel");
}

// ---- dQ -------------------------------------------------------------------
// One CTA per 64 query rows; per staged tile of 32 keys (exact or centroid)
// every warp computes, for each of its rows, p and dP with lane = key, then
// ds = p (dP − δ) and dq += Σ_key ds k_key with lane = channels.
template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads)
bwd_dq_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
              const T* __restrict__ dO, int H, int N, const int32_t* __restrict__ block_idx, int topk, int zo,
              const float* __restrict__ kmean, const float* __restrict__ vsum, float scale,
              const float* __restrict__ lse2, const float* __restrict__ delta, float* __restrict__ dQ) {
  constexpr int PER = D / 32;
  const int nb = N / BLK;
  const int row0 = blockIdx.x * kBwdRows, i = row0 / BLK;
  const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
  const size_t head = bh * (size_t)N * D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwords = (nb + 31) >> 5;
  const float scale2 = scale * kLog2e;
  extern __shared__ float bsm[];
  float* qs = bsm;                                   // [64][D]
  float* gs = qs + kBwdRows * D;                     // [64][D] dO rows
  float* ks = gs + kBwdRows * D;                     // [KT][D + 4]
  float* vs = ks + kBwdKT * (D + 4);                 // [KT][D + 4]
  uint32_t* sel_bits = reinterpret_cast<uint32_t*>(vs + kBwdKT * (D + 4));
  for (int x = tid; x < kBwdRows * D; x += kBwdThreads) {
    qs[x] = to_f<T>(Q[head + (size_t)row0 * D + x]);
    gs[x] = to_f<T>(dO[head + (size_t)row0 * D + x]);
  }
  const int32_t* sel = block_idx + (bh * nb + i) * (size_t)topk;
  load_selection(sel_bits, nwords, sel, topk);
  float l2[kBwdRpw], dl[kBwdRpw], acc[kBwdRpw][PER];
#pragma unroll
  for (int r = 0; r < kBwdRpw; ++r) {
    const int row = row0 + warp * kBwdRpw + r;
    l2[r] = lse2[bh * N + row];
    dl[r] = delta[bh * N + row];
#pragma unroll
    for (int c = 0; c < PER; ++c) acc[r][c] = 0.f;
  }
  const int pe = topk * (BLK / kBwdKT), pc = zo ? (nb + kBwdKT - 1) / kBwdKT : 0;
  const float bias_c = log2f((float)BLK);
  for (int piece = 0; piece < pe + pc; ++piece) {
    __syncthreads();
    bool valid;
    float bias = 0.f;
    if (piece < pe) {
      const int j = sel[piece / (BLK / kBwdKT)];
      const int r0 = j * BLK + (piece % (BLK / kBwdKT)) * kBwdKT;
      stage_keys<T, D>(ks, K + head, r0, kBwdKT);
      stage_keys<T, D>(vs, V + head, r0, kBwdKT);
      valid = true;
    } else {
      const int j0 = (piece - pe) * kBwdKT, j = j0 + lane;
      stage_keys<float, D>(ks, kmean + bh * (size_t)nb * D, j0, min(kBwdKT, nb - j0));
      stage_keys<float, D>(vs, vsum + bh * (size_t)nb * D, j0, min(kBwdKT, nb - j0), 1.0f / BLK);
      valid = j < nb && !((sel_bits[j >> 5] >> (j & 31)) & 1u);
      bias = bias_c;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kBwdRpw; ++r) {
      const float* qr = qs + (warp * kBwdRpw + r) * D;
      const float* gr = gs + (warp * kBwdRpw + r) * D;
      const float* kr = ks + lane * (D + 4);
      const float* vr = vs + lane * (D + 4);
      float x = 0.f, dp = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 a = *reinterpret_cast<const float4*>(qr + c), k4 = *reinterpret_cast<const float4*>(kr + c);
        const float4 gg = *reinterpret_cast<const float4*>(gr + c), v4 = *reinterpret_cast<const float4*>(vr + c);
        x = fmaf(a.x, k4.x, x);
        x = fmaf(a.y, k4.y, x);
        x = fmaf(a.z, k4.z, x);
        x = fmaf(a.w, k4.w, x);
        dp = fmaf(gg.x, v4.x, dp);
        dp = fmaf(gg.y, v4.y, dp);
        dp = fmaf(gg.z, v4.z, dp);
        dp = fmaf(gg.w, v4.w, dp);
      }
      const float p = valid ? fast_exp2(fmaf(x, scale2, bias) - l2[r]) : 0.f;
      const float ds = p * (dp - dl[r]);
#pragma unroll 4
      for (int t = 0; t < kBwdKT; ++t) {
        const float dst = __shfl_sync(0xffffffffu, ds, t);
#pragma unroll
        for (int c = 0; c < PER; ++c) acc[r][c] = fmaf(dst, ks[t * (D + 4) + lane * PER + c], acc[r][c]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kBwdRpw; ++r) {
    const int row = row0 + warp * kBwdRpw + r;
#pragma unroll
    for (int c = 0; c < PER; ++c) dQ[head + (size_t)row * D + lane * PER + c] = scale * acc[r][c];
  }
}

// ---- dK, dV of the exact keys ---------------------------------------------
// One CTA per 64 keys of one KV block; thread = (key, part): four threads per
// key, part p owning the 16-byte channel chunks 4 i + p (float4 shared reads
// that the four parts take from four different chunks).  The
// query rows of every query block that selected the block are staged 32 at a
// time; s and dP are reduced over the four parts with two shuffles.
constexpr int kKvKeys = 64;
constexpr int kKvParts = kBwdThreads / kKvKeys;    // 4
constexpr int kKvRows = 32;

template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads)
bwd_dkv_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
               const T* __restrict__ dO, int H, int N, const int32_t* __restrict__ offs,
               const int32_t* __restrict__ list, int topk, float scale, const float* __restrict__ lse2,
               const float* __restrict__ delta, float* __restrict__ dK, float* __restrict__ dV) {
  constexpr int CPT = D / kKvParts;
  const int nb = N / BLK;
  const int j = blockIdx.x / (BLK / kKvKeys), half = blockIdx.x % (BLK / kKvKeys);
  const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
  const size_t head = bh * (size_t)N * D;
  const int tid = threadIdx.x, key = tid / kKvParts, part = tid % kKvParts;
  const int n = j * BLK + half * kKvKeys + key;       // this thread's key token
  const float scale2 = scale * kLog2e;
  __shared__ __align__(16) float qs[kKvRows][D];
  __shared__ __align__(16) float gs[kKvRows][D];
  __shared__ float ls[kKvRows], ds_[kKvRows];
  // channel of element e: chunk kKvParts (e / 4) + part, lane e % 4 in it
  auto ch = [&](int e) { return 4 * (kKvParts * (e >> 2) + part) + (e & 3); };
  float kr[CPT], vr[CPT], dk[CPT], dv[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    kr[e] = to_f<T>(K[head + (size_t)n * D + ch(e)]);
    vr[e] = to_f<T>(V[head + (size_t)n * D + ch(e)]);
    dk[e] = 0.f;
    dv[e] = 0.f;
  }
  const int32_t* off = offs + bh * (size_t)(nb + 1);
  const int32_t* lst = list + bh * (size_t)nb * topk;
  for (int li = off[j]; li < off[j + 1]; ++li) {
    const int i = lst[li];
    for (int r0 = i * BLK; r0 < (i + 1) * BLK; r0 += kKvRows) {
      __syncthreads();
      for (int x = tid; x < kKvRows * D; x += kBwdThreads) {
        qs[x / D][x % D] = to_f<T>(Q[head + (size_t)r0 * D + x]);
        gs[x / D][x % D] = to_f<T>(dO[head + (size_t)r0 * D + x]);
      }
      if (tid < kKvRows) {
        ls[tid] = lse2[bh * N + r0 + tid];
        ds_[tid] = delta[bh * N + r0 + tid];
      }
      __syncthreads();
#pragma unroll 2
      for (int r = 0; r < kKvRows; ++r) {
        float x = 0.f, dp = 0.f;
        float4 q4[CPT / 4], g4[CPT / 4];
#pragma unroll
        for (int e4 = 0; e4 < CPT / 4; ++e4) {
          q4[e4] = *reinterpret_cast<const float4*>(&qs[r][ch(4 * e4)]);
          g4[e4] = *reinterpret_cast<const float4*>(&gs[r][ch(4 * e4)]);
          x = fmaf(q4[e4].x, kr[4 * e4], x);
          x = fmaf(q4[e4].y, kr[4 * e4 + 1], x);
          x = fmaf(q4[e4].z, kr[4 * e4 + 2], x);
          x = fmaf(q4[e4].w, kr[4 * e4 + 3], x);
          dp = fmaf(g4[e4].x, vr[4 * e4], dp);
          dp = fmaf(g4[e4].y, vr[4 * e4 + 1], dp);
          dp = fmaf(g4[e4].z, vr[4 * e4 + 2], dp);
          dp = fmaf(g4[e4].w, vr[4 * e4 + 3], dp);
        }
#pragma unroll
        for (int o = 1; o < kKvParts; o <<= 1) {
          x += __shfl_xor_sync(0xffffffffu, x, o);
          dp += __shfl_xor_sync(0xffffffffu, dp, o);
        }
        const float p = fast_exp2(fmaf(x, scale2, -ls[r]));
        const float d = p * (dp - ds_[r]);
#pragma unroll
        for (int e4 = 0; e4 < CPT / 4; ++e4) {
          dv[4 * e4] = fmaf(p, g4[e4].x, dv[4 * e4]);
          dv[4 * e4 + 1] = fmaf(p, g4[e4].y, dv[4 * e4 + 1]);
          dv[4 * e4 + 2] = fmaf(p, g4[e4].z, dv[4 * e4 + 2]);
          dv[4 * e4 + 3] = fmaf(p, g4[e4].w, dv[4 * e4 + 3]);
          dk[4 * e4] = fmaf(d, q4[e4].x, dk[4 * e4]);
          dk[4 * e4 + 1] = fmaf(d, q4[e4].y, dk[4 * e4 + 1]);
          dk[4 * e4 + 2] = fmaf(d, q4[e4].z, dk[4 * e4 + 2]);
          dk[4 * e4 + 3] = fmaf(d, q4[e4].w, dk[4 * e4 + 3]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    dK[head + (size_t)n * D + ch(e)] = scale * dk[e];
    dV[head + (size_t)n * D + ch(e)] = dv[e];
  }
}

// ---- zero-order tail: the centroids' gradients ----------------------------
// One CTA per 32 centroids of a head, thread = (centroid, part) with eight
// parts owning the 16-byte channel chunks 8 i + part; every query row of the head is visited (rows
// whose block selected a centroid get p = 0 for it).  At the end dk̄_j / B and
// dv̄_j / B are added to every token of block j (dK, dV hold the exact part,
// written by bwd_dkv_kernel earlier on the stream).
constexpr int kCtCent = 32;
constexpr int kCtParts = kBwdThreads / kCtCent;    // 8
constexpr int kCtRows = 32;

template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads)
bwd_centroid_kernel(const T* __restrict__ Q, const T* __restrict__ dO, int H, int N,
                    const int32_t* __restrict__ block_idx, int topk, const float* __restrict__ kmean,
                    const float* __restrict__ vsum, float scale, const float* __restrict__ lse2,
                    const float* __restrict__ delta, float* __restrict__ dK, float* __restrict__ dV) {
  constexpr int CPT = D / kCtParts;
  const int nb = N / BLK;
  const int j0 = blockIdx.x * kCtCent;
  const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
  const size_t head = bh * (size_t)N * D;
  const int tid = threadIdx.x, cj = tid / kCtParts, part = tid % kCtParts;
  const int j = j0 + cj;
  const bool live = j < nb;
  const float scale2 = scale * kLog2e, bias = log2f((float)BLK), inv_blk = 1.0f / BLK;
  __shared__ __align__(16) float qs[kCtRows][D];
  __shared__ __align__(16) float gs[kCtRows][D];
  __shared__ float ls[kCtRows], ds_[kCtRows];
  __shared__ uint32_t selm;                          // bit c: centroid j0 + c selected by this query block
  auto ch = [&](int e) { return 4 * (kCtParts * (e >> 2) + part) + (e & 3); };
  float kr[CPT], vr[CPT], dk[CPT], dv[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    const size_t g = (bh * nb + (live ? j : 0)) * D + ch(e);
    kr[e] = live ? kmean[g] : 0.f;
    vr[e] = live ? vsum[g] * inv_blk : 0.f;
    dk[e] = 0.f;
    dv[e] = 0.f;
  }
  for (int r0 = 0; r0 < N; r0 += kCtRows) {
    __syncthreads();
    if (r0 % BLK == 0) {
      // the selection of the query block these rows belong to, on this chunk of centroids
      if (tid == 0) selm = 0u;
      __syncthreads();
      const int32_t* sel = block_idx + (bh * nb + r0 / BLK) * (size_t)topk;
      for (int x = tid; x < topk; x += kBwdThreads) {
        const int c = sel[x] - j0;
        if (c >= 0 && c < kCtCent) atomicOr(&selm, 1u << c);
      }
    }
    for (int x = tid; x < kCtRows * D; x += kBwdThreads) {
      qs[x / D][x % D] = to_f<T>(Q[head + (size_t)r0 * D + x]);
      gs[x / D][x % D] = to_f<T>(dO[head + (size_t)r0 * D + x]);
    }
    if (tid < kCtRows) {
      ls[tid] = lse2[bh * N + r0 + tid];
      ds_[tid] = delta[bh * N + r0 + tid];
    }
    __syncthreads();
    const bool valid = live && !((selm >> cj) & 1u);
#pragma unroll 2
    for (int r = 0; r < kCtRows; ++r) {
      float x = 0.f, dp = 0.f;
      float4 q4[CPT / 4], g4[CPT / 4];
#pragma unroll
      for (int e4 = 0; e4 < CPT / 4; ++e4) {
        q4[e4] = *reinterpret_cast<const float4*>(&qs[r][ch(4 * e4)]);
        g4[e4] = *reinterpret_cast<const float4*>(&gs[r][ch(4 * e4)]);
        x = fmaf(q4[e4].x, kr[4 * e4], x);
        x = fmaf(q4[e4].y, kr[4 * e4 + 1], x);
        x = fmaf(q4[e4].z, kr[4 * e4 + 2], x);
        x = fmaf(q4[e4].w, kr[4 * e4 + 3], x);
        dp = fmaf(g4[e4].x, vr[4 * e4], dp);
        dp = fmaf(g4[e4].y, vr[4 * e4 + 1], dp);
        dp = fmaf(g4[e4].z, vr[4 * e4 + 2], dp);
        dp = fmaf(g4[e4].w, vr[4 * e4 + 3], dp);
      }
#pragma unroll
      for (int o = 1; o < kCtParts; o <<= 1) {
        x += __shfl_xor_sync(0xffffffffu, x, o);
        dp += __shfl_xor_sync(0xffffffffu, dp, o);
      }
      const float p = valid ? fast_exp2(fmaf(x, scale2, bias) - ls[r]) : 0.f;
      const float d = p * (dp - ds_[r]);
#pragma unroll
      for (int e4 = 0; e4 < CPT / 4; ++e4) {
        dv[4 * e4] = fmaf(p, g4[e4].x, dv[4 * e4]);
        dv[4 * e4 + 1] = fmaf(p, g4[e4].y, dv[4 * e4 + 1]);
        dv[4 * e4 + 2] = fmaf(p, g4[e4].z, dv[4 * e4 + 2]);
        dv[4 * e4 + 3] = fmaf(p, g4[e4].w, dv[4 * e4 + 3]);
        dk[4 * e4] = fmaf(d, q4[e4].x, dk[4 * e4]);
        dk[4 * e4 + 1] = fmaf(d, q4[e4].y, dk[4 * e4 + 1]);
        dk[4 * e4 + 2] = fmaf(d, q4[e4].z, dk[4 * e4 + 2]);
        dk[4 * e4 + 3] = fmaf(d, q4[e4].w, dk[4 * e4 + 3]);
      }
    }
  }
  if (!live) return;
  // the pseudo-key's gradients, spread over the block's tokens
  for (int t = 0; t < BLK; ++t) {
    const size_t rowoff = head + ((size_t)j * BLK + t) * D;
#pragma unroll
    for (int e = 0; e < CPT; ++e) {
      const size_t g = rowoff + ch(e);
      dK[g] += scale * dk[e] * inv_blk;
      dV[g] += dv[e] * inv_blk;
    }
  }
}

struct BwdLayout {
  size_t lse_off, delta_off, offs_off, list_off, part_off, fo_off, total;
};

BwdLayout bwd_layout(const sa_shape& s, int topk) {
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t BH = (size_t)s.B * s.H, nb = (size_t)(s.N / s.block);
  BwdLayout L;
  L.lse_off = 0;
  L.delta_off = a256(BH * s.N * sizeof(float));
  L.offs_off = L.delta_off + a256(BH * s.N * sizeof(float));
  L.list_off = L.offs_off + a256(BH * (nb + 1) * sizeof(int32_t));
  L.part_off = L.list_off + a256(BH * nb * (size_t)(topk > 0 ? topk : 1) * sizeof(int32_t));
  // the tensor-core centroid pass's partial sums (d = 128 shapes)
  L.fo_off = L.part_off + (s.d == 128 ? a256(bwd_tc_part_bytes(s)) : 0);
  // the first-order tail's per-row terms and partial H̄ gradients (d = block = 128)
  L.total = L.fo_off + (s.d == 128 && s.block == 128 ? a256(bwd_fo_bytes(s)) : 0);
  return L;
}

template <typename T, int D, int BLK>
sa_status launch_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                     const sa_shape& s, const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st,
                     float scale, float* dQ, float* dK, float* dV, const float* lse_in, char* ws,
                     cudaStream_t stream, bool fo = false) {
  const BwdLayout L = bwd_layout(s, topk);
  const int nb = s.N / BLK;
  float* lse2 = reinterpret_cast<float*>(ws + L.lse_off);
  float* delta = reinterpret_cast<float*>(ws + L.delta_off);
  int32_t* offs = reinterpret_cast<int32_t*>(ws + L.offs_off);
  int32_t* list = reinterpret_cast<int32_t*>(ws + L.list_off);
  const T* q = static_cast<const T*>(Q);
  const T* k = static_cast<const T*>(K);
  const T* v = static_cast<const T*>(V);
  const T* g = static_cast<const T*>(dO);
  const int nwords = (nb + 31) / 32;
  const dim3 gq(s.N / kBwdRows, s.H, s.B);
  const sa_dtype dt = sizeof(T) == 2 ? SA_BF16 : SA_FP32;
  if (bwd_tc_supports(dt, s, zo, st)) {
    // tensor-core kernels: the per-KV-block query lists first
    if (topk > 0) {
      sa_status r = launch_transpose(block_idx, nb, topk, offs, list, s.B * s.H, stream);
      if (r != SA_OK) return r;
    } else if (cudaMemsetAsync(offs, 0, (size_t)s.B * s.H * (nb + 1) * sizeof(int32_t), stream) != cudaSuccess) {
      return launch_status("cudaMemsetAsync(bwd offsets)");
    }
    if (fo)
      return bwd_first_order(Q, K, V, O, dO, s, block_idx, topk, st, scale, dQ, dK, dV, lse_in, lse2, delta, offs,
                             list, reinterpret_cast<float*>(ws + L.part_off), reinterpret_cast<float*>(ws + L.fo_off),
                             stream);
    return bwd_tc(Q, K, V, O, dO, s, block_idx, topk, zo, st, scale, dQ, dK, dV, lse_in, lse2, delta, offs, list,
                  reinterpret_cast<float*>(ws + L.part_off), stream);
  }
  if (fo) return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd: the first-order tail runs on the bf16 d = 128, "
                                          "block 128 tensor-core path only");
  {
    const size_t smem = sizeof(float) * ((size_t)kBwdRows * D + (size_t)kBwdKT * (D + 4)) +
                        sizeof(uint32_t) * nwords;
    auto kern = bwd_stats_kernel<T, D, BLK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(bwd_stats_kernel)");
    kern<<<gq, kBwdThreads, smem, stream>>>(q, k, static_cast<const T*>(O), g, s.H, s.N, block_idx, topk, zo,
                                            st.kmean, scale * kLog2e, lse2, delta);
    sa_status r = launch_status("bwd_stats_kernel");
    if (r != SA_OK) return r;
  }
  if (topk > 0) {
    sa_status r = launch_transpose(block_idx, nb, topk, offs, list, s.B * s.H, stream);
    if (r != SA_OK) return r;
  } else if (cudaMemsetAsync(offs, 0, (size_t)s.B * s.H * (nb + 1) * sizeof(int32_t), stream) != cudaSuccess) {
    return launch_status("cudaMemsetAsync(bwd offsets)");
  }
  {
    const size_t smem = sizeof(float) * (2 * (size_t)kBwdRows * D + 2 * (size_t)kBwdKT * (D + 4)) +
                        sizeof(uint32_t) * nwords;
    auto kern = bwd_dq_kernel<T, D, BLK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(bwd_dq_kernel)");
    kern<<<gq, kBwdThreads, smem, stream>>>(q, k, v, g, s.H, s.N, block_idx, topk, zo, st.kmean, st.vsum, scale,
                                            lse2, delta, dQ);
    sa_status r = launch_status("bwd_dq_kernel");
    if (r != SA_OK) return r;
  }
  bwd_dkv_kernel<T, D, BLK><<<dim3(nb * (BLK / kKvKeys), s.H, s.B), kBwdThreads, 0, stream>>>(
      q, k, v, g, s.H, s.N, offs, list, topk, scale, lse2, delta, dK, dV);
  sa_status r = launch_status("bwd_dkv_kernel");
  if (r != SA_OK || !zo) return r;
  bwd_centroid_kernel<T, D, BLK><<<dim3((nb + kCtCent - 1) / kCtCent, s.H, s.B), kBwdThreads, 0, stream>>>(
      q, g, s.H, s.N, block_idx, topk, st.kmean, st.vsum, scale, lse2, delta, dK, dV);
  return launch_status("bwd_centroid_kernel");
}

template <typename T>
sa_status dispatch_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                       const sa_shape& s, const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st,
                       float scale, float* dQ, float* dK, float* dV, const float* lse_in, char* ws,
                       cudaStream_t stream, bool fo) {
#define SA_BWD_CASE(DD, BB)                                                                              \
  if (s.d == DD && s.block == BB)                                                                        \
    return launch_bwd<T, DD, BB>(Q, K, V, O, dO, s, block_idx, topk, zo, st, scale, dQ, dK, dV, lse_in, ws,  \
                                 stream, fo);
  SA_BWD_CASE(128, 128)
  SA_BWD_CASE(128, 64)
  SA_BWD_CASE(64, 128)
  SA_BWD_CASE(64, 64)
#undef SA_BWD_CASE
  return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd: d and block must be 64 or 128");
}

}  // namespace
}  // namespace sa

extern "C" size_t sa_sparse_attn_bwd_workspace_size(sa_shape shape, int32_t topk) {
  using namespace sa;
  if (check_shape(shape, "sa_sparse_attn_bwd_workspace_size") != SA_OK || topk < 0) return 0;
  return bwd_layout(shape, topk).total;
}

namespace sa {
namespace {
// lse_in: the forward's log-sum-exp (sa_sparse_attn_fwd_lse) or null
sa_status bwd_entry(const void* Q, const void* K, const void* V, const void* O, const void* dO, sa_dtype dtype,
                    sa_shape shape, const int32_t* block_idx, int32_t topk, sa_tail_mode tail,
                    const sa_block_stats* stats, float scale, const float* lse_in, float* dQ, float* dK, float* dV,
                    void* workspace, size_t workspace_bytes, void* stream) {
  sa_status r = check_shape(shape, "sa_sparse_attn_bwd");
  if (r != SA_OK) return r;
  const int nb = shape.N / shape.block;
  if (dtype != SA_FP32 && dtype != SA_BF16)
    return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd: dtype must be SA_FP32 or SA_BF16");
  if (tail != SA_TAIL_DROP && tail != SA_TAIL_ZERO_ORDER && tail != SA_TAIL_FIRST_ORDER)
    return fail(SA_ERR_UNSUPPORTED,
                "sa_sparse_attn_bwd: tail must be SA_TAIL_DROP, SA_TAIL_ZERO_ORDER or SA_TAIL_FIRST_ORDER");
  if (shape.B == 0 || shape.H == 0 || shape.N == 0) return SA_OK;
  if (!Q || !K || !V || !O || !dO || !dQ || !dK || !dV)
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd: Q, K, V, O, dO, dQ, dK and dV are required");
  if (topk < 0 || topk > nb) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd: topk must be in [0, N/block]");
  if (topk > 0 && !block_idx) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd: block_idx is required");
  if (nb > kMaxAttnBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd: at most 4096 blocks per head");
  const bool fo = tail == SA_TAIL_FIRST_ORDER;
  const bool zo = tail == SA_TAIL_ZERO_ORDER || fo;
  sa_block_stats st{};
  if (stats) st = *stats;
  if (zo && (!st.kmean || !st.vsum))
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd: the zero-order tails need stats->kmean and stats->vsum");
  if (fo && (dtype != SA_BF16 || shape.d != 128 || shape.block != 128))
    return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd: SA_TAIL_FIRST_ORDER needs bf16, d = 128 and block 128");
  if (fo && (!st.hbar || !st.kmean_bf16 || !st.vmean_bf16))
    return fail(SA_ERR_INVALID_ARG,
                "sa_sparse_attn_bwd: SA_TAIL_FIRST_ORDER needs stats->hbar, kmean_bf16 and vmean_bf16");
  const size_t need = bwd_layout(shape, topk).total;
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "sa_sparse_attn_bwd: workspace missing or smaller than the workspace size");
  const void* ptrs[] = {Q, K, V, O, dO, dQ, dK, dV, workspace, block_idx, st.kmean, st.vsum, lse_in, st.hbar};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_sparse_attn_bwd: pointers must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  char* ws = static_cast<char*>(workspace);
  if (dtype == SA_BF16)
    return dispatch_bwd<__nv_bfloat16>(Q, K, V, O, dO, shape, block_idx, topk, zo, st, scale, dQ, dK, dV, lse_in,
                                       ws, s, fo);
  return dispatch_bwd<float>(Q, K, V, O, dO, shape, block_idx, topk, zo, st, scale, dQ, dK, dV, lse_in, ws, s, fo);
}
}  // namespace
}  // namespace sa

extern "C" sa_status sa_sparse_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                        sa_dtype dtype, sa_shape shape, const int32_t* block_idx, int32_t topk,
                                        sa_tail_mode tail, const sa_block_stats* stats, float scale, float* dQ,
                                        float* dK, float* dV, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  return sa::bwd_entry(Q, K, V, O, dO, dtype, shape, block_idx, topk, tail, stats, scale, nullptr, dQ, dK, dV,
                       workspace, workspace_bytes, stream);
}

extern "C" sa_status sa_sparse_attn_bwd_lse(const void* Q, const void* K, const void* V, const void* O,
                                            const void* dO, const float* lse2, sa_dtype dtype, sa_shape shape,
                                            const int32_t* block_idx, int32_t topk, sa_tail_mode tail,
                                            const sa_block_stats* stats, float scale, float* dQ, float* dK,
                                            float* dV, void* workspace, size_t workspace_bytes, void* stream) {
  if (!lse2) return sa::fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd_lse: lse2 is required");
  return sa::bwd_entry(Q, K, V, O, dO, dtype, shape, block_idx, topk, tail, stats, scale, lse2, dQ, dK, dV,
                       workspace, workspace_bytes, stream);
}

// ---- SLA2's linear mix -----------------------------------------------------
namespace sa {
namespace {
size_t lin_workspace_bytes(const sa_shape& s, int topk) {
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return a256(bwd_layout(s, topk).total) + bwd_lin_bytes(s);
}
}  // namespace
}  // namespace sa

extern "C" size_t sa_sparse_attn_bwd_linear_mix_workspace_size(sa_shape shape, int32_t topk) {
  using namespace sa;
  if (check_shape(shape, "sa_sparse_attn_bwd_linear_mix_workspace_size") != SA_OK || topk < 0) return 0;
  if (shape.d != 128 || shape.block != 128) return 0;
  return lin_workspace_bytes(shape, topk);
}

extern "C" sa_status sa_sparse_attn_bwd_linear_mix(const void* Q, const void* K, const void* V, const void* O,
                                                   const void* dO, sa_dtype dtype, sa_shape shape,
                                                   const int32_t* block_idx, int32_t topk, const float* alpha,
                                                   const sa_block_stats* stats, float scale, float* dQ, float* dK,
                                                   float* dV, void* workspace, size_t workspace_bytes,
                                                   void* stream) {
  using namespace sa;
  sa_status r = check_shape(shape, "sa_sparse_attn_bwd_linear_mix");
  if (r != SA_OK) return r;
  const int nb = shape.N / shape.block;
  if (dtype != SA_BF16 || shape.d != 128 || shape.block != 128)
    return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd_linear_mix: bf16, d = 128 and block 128 only");
  if (shape.B == 0 || shape.H == 0 || shape.N == 0) return SA_OK;
  if (!Q || !K || !V || !O || !dO || !dQ || !dK || !dV || !alpha || !stats)
    return fail(SA_ERR_INVALID_ARG,
                "sa_sparse_attn_bwd_linear_mix: Q, K, V, O, dO, alpha, stats, dQ, dK and dV are required");
  if (topk < 0 || topk > nb)
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd_linear_mix: topk must be in [0, N/block]");
  if (topk > 0 && !block_idx) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd_linear_mix: block_idx is required");
  if (nb > kMaxAttnBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd_linear_mix: at most 4096 blocks per head");
  const sa_block_stats st = *stats;
  if (!st.htot || !st.ztot || !st.zrelu)
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd_linear_mix: needs stats->htot, ztot and zrelu");
  const size_t need = lin_workspace_bytes(shape, topk);
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE,
                "sa_sparse_attn_bwd_linear_mix: workspace missing or smaller than its workspace size");
  const void* ptrs[] = {Q, K, V, O, dO, dQ, dK, dV, workspace, block_idx, alpha, st.htot, st.ztot, st.zrelu};
  for (const void* p : ptrs)
    if (p && !aligned16(p))
      return fail(SA_ERR_ALIGNMENT, "sa_sparse_attn_bwd_linear_mix: pointers must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  char* ws = static_cast<char*>(workspace);
  const BwdLayout L = bwd_layout(shape, topk);
  int32_t* offs = reinterpret_cast<int32_t*>(ws + L.offs_off);
  int32_t* list = reinterpret_cast<int32_t*>(ws + L.list_off);
  if (topk > 0) {
    r = launch_transpose(block_idx, nb, topk, offs, list, shape.B * shape.H, s);
    if (r != SA_OK) return r;
  } else if (cudaMemsetAsync(offs, 0, (size_t)shape.B * shape.H * (nb + 1) * sizeof(int32_t), s) != cudaSuccess) {
    return launch_status("cudaMemsetAsync(bwd offsets)");
  }
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return bwd_linear_mix(Q, K, V, O, dO, shape, block_idx, topk, alpha, st, scale, dQ, dK, dV,
                        reinterpret_cast<float*>(ws + L.lse_off), reinterpret_cast<float*>(ws + L.delta_off), offs,
                        list, reinterpret_cast<float*>(ws + L.part_off), ws + a256(L.total), s);
}
