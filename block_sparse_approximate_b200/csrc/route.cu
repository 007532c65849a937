// Router: block scores and top-k selection of KV blocks per query block.
//   dot      q̄_i·k̄_j                        (SLA2 §2B, mean pooling)
//   proj     (q̄_i P_q)·(k̄_j P_k)              (SLA2 §2B, learnable router)
//   taylor2  s q̄_i·k̄_j + log1p(½ s² Σ q̄²var)  (SPLA §2.1, log of the
//            second-order block score with diagonal covariance)
//   cov      s q̄_i·k̄_j + log1p(s ‖q̄_i‖ M_j / B) (PISA §2, covariance-aware
//            routing: zero-order mass plus the first-order error bound,
//            M_j = ‖H_j − H̄‖₂ from block_pool)
// The proj score (q̄_i P_q)·(k̄_j P_k) is evaluated as k̄_j·u_i with
// u_i = P_k P_qᵀ q̄_i (x P is the row vector x times P), so no projected copy
// of the key centroids is needed: u_i costs 2d² multiply-adds per query block.
//
// One CTA handles QB = 8 RPW query blocks of one head.  The scores of its QB
// rows against all nb centroids are a small fp32 matrix product, done tile
// by tile: TJ = 32 NCOL centroid rows are staged by cp.async into shared
// memory rows padded to d + 4 floats (two buffers, so the next tile lands
// while this one is used); warp w owns rows [w RPW, w RPW + RPW) and lane l
// the centroids l, l + 32, ... of the tile, reading its centroid rows as
// float4 without bank conflicts and the query rows as warp broadcasts.  The
// proj vector u_i = P_k t_i (t_i = q̄_i P_q) takes the same path with the
// rows of P_k in place of centroids.  Selection: for small k each warp finds
// the key of the k-th best block of each of its rows by a radix select (one
// bit per step, counted with a warp reduction), keeps the blocks above it
// and the smallest indices among those equal to it, and emits them in
// ascending order from a bitmap; for large k the CTA sorts each row with a
// bitonic sort.
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kWarpTopkMax = 64;               // largest k taken by the warp radix select
constexpr int kRegKeys = 16;                   // keys per lane kept in registers (rows of <= 512 blocks)
constexpr size_t kMaxSmemPerCta = 232448;      // opt-in shared memory of one CTA on sm_100
constexpr size_t kSmemTwoPerSm = 115712;       // per CTA when two share an SM (233472 / 2 - 1 KB)

__device__ __forceinline__ void cp_async16r(float* smem_dst, const float* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}

// Stages rows [r0, r0 + n) of a [rows][D] float array into `dst` (TJ rows
// of D + 4 floats); rows past n are zero-filled.
template <int D, int TJ, int NTH = kRouteThreads>
__device__ __forceinline__ void stage_rows(float* dst, const float* src, int r0, int n) {
  constexpr int C4 = D / 4;
  for (int x = threadIdx.x; x < TJ * C4; x += NTH) {
    const int r = x / C4, c = x % C4;
    float* d = dst + r * (D + 4) + 4 * c;
    if (r < n) cp_async16r(d, src + (size_t)(r0 + r) * D + 4 * c);
    else *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// out[r][n] = A[r]·T[lane + 32 n] for the warp's RPW rows of A ([.][D],
// read as broadcasts) and the lane's NCOL rows of the tile T ([TJ][D + 4]).
template <int D, int RPW, int NCOL>
__device__ __forceinline__ void tile_dots(const float* A, const float* T, int lane, float (&out)[RPW][NCOL]) {
#pragma unroll
  for (int r = 0; r < RPW; ++r)
#pragma unroll
    for (int n = 0; n < NCOL; ++n) out[r][n] = 0.f;
#pragma unroll 4
  for (int c = 0; c < D; c += 4) {
    float4 t[NCOL];
#pragma unroll
    for (int n = 0; n < NCOL; ++n) t[n] = *reinterpret_cast<const float4*>(T + (lane + 32 * n) * (D + 4) + c);
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const float4 a = *reinterpret_cast<const float4*>(A + r * D + c);
#pragma unroll
      for (int n = 0; n < NCOL; ++n) {
        out[r][n] = fmaf(a.x, t[n].x, out[r][n]);
        out[r][n] = fmaf(a.y, t[n].y, out[r][n]);
        out[r][n] = fmaf(a.z, t[n].z, out[r][n]);
        out[r][n] = fmaf(a.w, t[n].w, out[r][n]);
      }
    }
  }
}

// The key T of the k-th best block of a row, as the largest X with
// #(key ≥ X) ≥ k, built from the top bit down (one count per bit).  `exact`
// is set once some X has exactly k keys at or above it: those keys are the
// top k and the bits below do not matter.  KPL keys per lane are held in
// registers (rows of at most 32·KPL blocks); lanes past the row hold 0,
// which no X ≥ 1 counts.
template <int KPL>
__device__ __forceinline__ void kth_key_reg(const float* scw, int nb, int k, int lane, unsigned& T, bool& exact) {
  unsigned key[KPL];
#pragma unroll
  for (int m = 0; m < KPL; ++m) {
    const int j = lane + 32 * m;
    key[m] = j < nb ? order_key(scw[j]) : 0u;
  }
  T = 0u;
  exact = false;
  for (int bit = 31; bit >= 0; --bit) {
    const unsigned X = T | (1u << bit);
    unsigned c = 0u;
#pragma unroll
    for (int m = 0; m < KPL; ++m) c += key[m] >= X ? 1u : 0u;
    c = __reduce_add_sync(0xffffffffu, c);
    if ((int)c >= k) {
      T = X;
      if ((int)c == k) {
        exact = true;
        break;
      }
    }
  }
}

// the same search over a row read from shared memory on every step
__device__ __forceinline__ void kth_key_smem(const float* scw, int nb, int k, int lane, unsigned& T, bool& exact) {
  T = 0u;
  exact = false;
  for (int bit = 31; bit >= 0; --bit) {
    const unsigned X = T | (1u << bit);
    unsigned c = 0u;
    for (int j = lane; j < nb; j += 32) c += order_key(scw[j]) >= X ? 1u : 0u;
    c = __reduce_add_sync(0xffffffffu, c);
    if ((int)c >= k) {
      T = X;
      if ((int)c == k) {
        exact = true;
        break;
      }
    }
  }
}

// Top-k of one row of nb scores by one warp, the kept indices written to
// out ascending: the k-th key T, then a bitmap (bw, nwords words of shared
// memory) of the kept blocks, emitted in order.  Kept: every key above T
// and, of the keys equal to T, the smallest indices (a tie in score goes to
// the smaller index); when `exact`, every key at or above T.
__device__ __forceinline__ void select_row(const float* scw, uint32_t* bw, int nb, int nwords, int topk, int lane,
                                           int32_t* out) {
  if (topk <= 0) return;
  unsigned T;
  bool exact;
  if (nb <= 32 * kRegKeys / 2) kth_key_reg<kRegKeys / 2>(scw, nb, topk, lane, T, exact);
  else if (nb <= 32 * kRegKeys) kth_key_reg<kRegKeys>(scw, nb, topk, lane, T, exact);
  else kth_key_smem(scw, nb, topk, lane, T, exact);
  int want = topk;   // places left for the keys equal to T
  if (!exact) {
    unsigned gt = 0u;
    for (int j = lane; j < nb; j += 32) gt += order_key(scw[j]) > T ? 1u : 0u;
    want -= (int)__reduce_add_sync(0xffffffffu, gt);
  }
  for (int m = 0; m < nwords; ++m) {
    const int j = 32 * m + lane;
    const bool valid = j < nb;
    const unsigned key = valid ? order_key(scw[j]) : 0u;
    bool keep;
    if (exact) {
      keep = valid && key >= T;
    } else {
      const bool eq = valid && key == T;
      const unsigned eqb = __ballot_sync(0xffffffffu, eq);
      keep = (valid && key > T) || (eq && __popc(eqb & ((1u << lane) - 1u)) < want);
      want -= min(want, __popc(eqb));
    }
    const unsigned take = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) bw[m] = take;
  }
  __syncwarp();
  // ascending emission from the bitmap
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

template <int D, int RPW, int NCOL>
__global__ void __launch_bounds__(kRouteThreads)
route_kernel(sa_block_stats st, int H, int nb, sa_route_mode mode, const float* __restrict__ Pq,
             const float* __restrict__ Pk, float scale, float inv_blk, int topk, int32_t* __restrict__ block_idx,
             float* __restrict__ scores_out) {
  constexpr int QB = kRouteWarps * RPW;          // query blocks per CTA
  constexpr int TJ = 32 * NCOL;                  // centroids per tile
  constexpr int TS = TJ * (D + 4);               // floats per staged tile
  const int h = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * QB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t bh = (size_t)b * H + h;
  const bool t2 = mode == SA_ROUTE_TAYLOR2;
  const bool cov = mode == SA_ROUTE_COV;
  const int narr = t2 ? 2 : 1;                   // staged arrays per tile

  extern __shared__ __align__(16) float rsm[];
  float* u = rsm;                                // [QB][D]  query vectors
  float* w = u + QB * D;                         // [QB][D]  ½ s² q̄² (taylor2) / q̄ P_q (proj)
  float* tiles = w + QB * D;                     // [2 buffers][narr][TS]
  // the tile region doubles as the sort keys of the large-k path
  size_t tile_floats = 2 * (size_t)narr * TS;
  if (topk > kWarpTopkMax) {
    int n2 = 1;
    while (n2 < nb) n2 <<= 1;
    if (2 * (size_t)n2 > tile_floats) tile_floats = 2 * (size_t)n2;
  }
  float* sc = tiles + tile_floats;               // [QB][nb] scores
  const int nwords = (nb + 31) >> 5;
  uint32_t* bits = reinterpret_cast<uint32_t*>(sc + (size_t)QB * nb);   // [QB][nwords]

  pdl_wait();                                     // the statistics come from the previous launch
  pdl_trigger();
  // ---- query vectors
  for (int x = tid; x < QB * D; x += kRouteThreads) {
    const int r = x / D, c = x % D;
    const int i = i0 + r;
    const float q = i < nb ? st.qmean[(bh * nb + i) * D + c] : 0.f;
    u[x] = (t2 || cov) ? scale * q : q;
    w[x] = 0.5f * scale * scale * q * q;
  }
  __syncthreads();
  if (mode == SA_ROUTE_PROJ) {
    // t = q̄ P_q into w: rows of P_q staged as tiles; lane = output columns
    // lane + 32 p, read from the tile rows without bank conflicts
    float tq[RPW][D / 32];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int p = 0; p < D / 32; ++p) tq[r][p] = 0.f;
    for (int k0 = 0; k0 < D; k0 += TJ) {
      __syncthreads();
      stage_rows<D, TJ>(tiles, Pq, k0, min(TJ, D - k0));
      asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
      __syncthreads();
      for (int k = 0; k < TJ && k0 + k < D; ++k) {
        const float* trow = tiles + k * (D + 4);
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const float a = u[(warp * RPW + r) * D + k0 + k];
#pragma unroll
          for (int p = 0; p < D / 32; ++p) tq[r][p] = fmaf(a, trow[lane + 32 * p], tq[r][p]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int p = 0; p < D / 32; ++p) w[(warp * RPW + r) * D + lane + 32 * p] = tq[r][p];
    __syncwarp();
    // ... then u = P_k t, with the rows of P_k staged like centroid tiles
    for (int r0 = 0; r0 < D; r0 += TJ) {
      __syncthreads();
      stage_rows<D, TJ>(tiles, Pk, r0, min(TJ, D - r0));
      asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
      __syncthreads();
      float o[RPW][NCOL];
      tile_dots<D, RPW, NCOL>(w + warp * RPW * D, tiles, lane, o);
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int n = 0; n < NCOL; ++n)
          if (r0 + lane + 32 * n < D) u[(warp * RPW + r) * D + r0 + lane + 32 * n] = o[r][n];
    }
    __syncthreads();
  }

  // cov: ‖s q̄_r‖ / B of the warp's rows (every lane holds them)
  float qnb[RPW];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    float ss = 0.f;
    if (cov) {
      for (int c = lane; c < D; c += 32) {
        const float v = u[(warp * RPW + r) * D + c];
        ss = fmaf(v, v, ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    qnb[r] = sqrtf(ss) * inv_blk;
  }
  const float* cvn = cov ? st.covnorm + bh * (size_t)nb : nullptr;

  // ---- scores: tiles of TJ centroids, two buffers
  const float* km = st.kmean + bh * (size_t)nb * D;
  const float* kv = t2 ? st.kvar + bh * (size_t)nb * D : nullptr;
  const int ntiles = (nb + TJ - 1) / TJ;
  auto stage = [&](int t, int buf) {
    const int j0 = t * TJ, n = min(TJ, nb - j0);
    stage_rows<D, TJ>(tiles + (size_t)buf * narr * TS, km, j0, n);
    if (t2) stage_rows<D, TJ>(tiles + (size_t)buf * narr * TS + TS, kv, j0, n);
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  stage(0, 0);
  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) {
      stage(t + 1, (t + 1) & 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const float* tk = tiles + (size_t)(t & 1) * narr * TS;
    float o[RPW][NCOL];
    tile_dots<D, RPW, NCOL>(u + warp * RPW * D, tk, lane, o);
    if (t2) {
      float o2[RPW][NCOL];
      tile_dots<D, RPW, NCOL>(w + warp * RPW * D, tk + TS, lane, o2);
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int n = 0; n < NCOL; ++n) o[r][n] += log1pf(o2[r][n]);
    }
    if (cov) {
#pragma unroll
      for (int n = 0; n < NCOL; ++n) {
        const int j = t * TJ + lane + 32 * n;
        const float m = j < nb ? cvn[j] : 0.f;
#pragma unroll
        for (int r = 0; r < RPW; ++r) o[r][n] += log1pf(qnb[r] * m);
      }
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int n = 0; n < NCOL; ++n) {
        const int j = t * TJ + lane + 32 * n;
        if (j < nb) sc[(size_t)(warp * RPW + r) * nb + j] = o[r][n];
      }
    __syncthreads();   // this buffer is restaged by the next iteration's prefetch
  }
  if (scores_out) {
    for (int r = warp * RPW; r < warp * RPW + RPW; ++r) {
      const int i = i0 + r;
      if (i >= nb) break;
      float* so = scores_out + (bh * nb + i) * (size_t)nb;
      for (int j = lane; j < nb; j += 32) so[j] = sc[(size_t)r * nb + j];
    }
  }

  // ---- selection
  if (topk <= kWarpTopkMax) {
    for (int r = warp * RPW; r < warp * RPW + RPW; ++r) {
      const int i = i0 + r;
      if (i >= nb) break;
      select_row(sc + (size_t)r * nb, bits + (size_t)r * nwords, nb, nwords, topk, lane,
                 block_idx + (bh * nb + i) * (size_t)topk);
    }
  } else {
    // large k: each row in turn is sorted by the whole CTA
    __syncthreads();
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(tiles);   // reuses the tile space
    for (int r = 0; r < QB && i0 + r < nb; ++r)
      block_topk_ascending(sc + (size_t)r * nb, nb, topk, keys,
                           block_idx + (bh * nb + i0 + r) * (size_t)topk);
  }
}

// ---- scores on the tensor cores ---------------------------------------------
// route_mma_kernel: the same scores and selection with the dot products on
// mma.sync m16n8k8 in three TF32 products (3xTF32): every fp32 operand x is
// split into hi = x with its 13 low mantissa bits cleared (a TF32 value) and
// lo = x − hi (exact in fp32, truncated to TF32), and
// a·b ≈ a_hi b_hi + a_hi b_lo + a_lo b_hi, each in its own fp32 accumulator,
// an error of ~2^-20 of Σ|a_c b_c|.  One CTA holds kMQ = 16 query blocks (the
// MMA rows) of one head in 16 warps: warp w < 8 takes centroids [8w, 8w + 8)
// of each staged tile of 64, then every warp selects the top k of one row.
// The proj router's u_i = P_k (P_qᵀ q̄_i) is two such products of the 16
// rows with P_q and P_k staged whole (128 rows of the tile space).
constexpr int kMQ = 16;
constexpr int kMT = 64;
constexpr int kMmaThreads = 512;
constexpr int kMmaWarps = 8;

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  const uint32_t h = __float_as_uint(x) & 0xffffe000u;
  hi = h;
  lo = __float_as_uint(x - __uint_as_float(h)) & 0xffffe000u;
}

// acc[p][nt] += the p-th of the three TF32 products of A (16 fp32 rows,
// stride lda) and B for the warp's NT n-tiles of 8 columns from column n0:
// B column n is row n of `bm` ([.][D + 4]) when BROWS_N, else its column n.
template <int D, int NT, bool BROWS_N>
__device__ __forceinline__ void warp_tf32(float (&acc)[3][NT][4], const float* A, int lda, const float* bm, int n0,
                                          int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll 4
  for (int k0 = 0; k0 < D; k0 += 8) {
    uint32_t ah[4], al[4];
    split_tf32(A[g * lda + k0 + t], ah[0], al[0]);
    split_tf32(A[(g + 8) * lda + k0 + t], ah[1], al[1]);
    split_tf32(A[g * lda + k0 + t + 4], ah[2], al[2]);
    split_tf32(A[(g + 8) * lda + k0 + t + 4], ah[3], al[3]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = n0 + 8 * nt + g;
      const float x0 = BROWS_N ? bm[n * (D + 4) + k0 + t] : bm[(k0 + t) * (D + 4) + n];
      const float x1 = BROWS_N ? bm[n * (D + 4) + k0 + t + 4] : bm[(k0 + t + 4) * (D + 4) + n];
      uint32_t bh0, bl0, bh1, bl1;
      split_tf32(x0, bh0, bl0);
      split_tf32(x1, bh1, bl1);
      mma_tf32(acc[0][nt], ah, bh0, bh1);
      mma_tf32(acc[1][nt], ah, bl0, bl1);
      mma_tf32(acc[2][nt], al, bh0, bh1);
    }
  }
}

// the sum of the three products, small terms first
template <int NT>
__device__ __forceinline__ float tf32_sum(const float (&acc)[3][NT][4], int nt, int e) {
  return acc[0][nt][e] + (acc[1][nt][e] + acc[2][nt][e]);
}

// score row stride: past nb, a multiple of 4, so that float2 stores of the
// MMA fragments are aligned and rows g, g + 8 fall in different banks
__host__ __device__ __forceinline__ int route_ldc(int nb) { return ((nb + 3) & ~3) + 8; }

template <int D>
__global__ void __launch_bounds__(kMmaThreads, 2)
route_mma_kernel(sa_block_stats st, int H, int nb, sa_route_mode mode, const float* __restrict__ Pq,
                 const float* __restrict__ Pk, float scale, float inv_blk, int topk, int32_t* __restrict__ block_idx,
                 float* __restrict__ scores_out) {
  constexpr int LD = D + 4;
  constexpr int TS = kMT * LD;                    // floats per staged tile
  constexpr int NTP = D / 64;                     // n-tiles per warp of the proj products
  const int h = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * kMQ;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const size_t bh = (size_t)b * H + h;
  const bool t2 = mode == SA_ROUTE_TAYLOR2;
  const bool cov = mode == SA_ROUTE_COV;
  const bool proj = mode == SA_ROUTE_PROJ;
  const int narr = t2 ? 2 : 1;
  const int nrows = min(kMQ, nb - i0);
  const int ldc = route_ldc(nb);

  extern __shared__ __align__(16) float rsm[];
  __shared__ float qn[kMQ];                       // cov: ‖s q̄_r‖ / B
  float* qa = rsm;                                // [16][LD] query rows: q̄, s q̄ or u
  float* qw = qa + kMQ * LD;                      // [16][LD] ½ s² q̄² (taylor2)
  float* tiles = qw + (t2 ? kMQ * LD : 0);        // [2][narr][TS]; the row bitmaps after the scores
  float* sc = tiles + 2 * (size_t)narr * TS;      // [16][ldc] scores; T = q̄ P_q (proj) before them

  pdl_wait();                                     // the statistics come from the previous launch
  pdl_trigger();
  const float* qm = st.qmean + (bh * nb + i0) * D;
  const float* km = st.kmean + bh * (size_t)nb * D;
  const float* kv = t2 ? st.kvar + bh * (size_t)nb * D : nullptr;
  const int ntiles = (nb + kMT - 1) / kMT;
  auto stage = [&](int tt, int buf) {
    const int j0 = tt * kMT, n = min(kMT, nb - j0);
    stage_rows<D, kMT, kMmaThreads>(tiles + (size_t)buf * narr * TS, km, j0, n);
    if (t2) stage_rows<D, kMT, kMmaThreads>(tiles + (size_t)buf * narr * TS + TS, kv, j0, n);
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  if (!proj) stage(0, 0);                         // the first tile lands while the rows load
  const float mul = (t2 || cov) ? scale : 1.f;
  for (int x = tid; x < kMQ * D / 4; x += kMmaThreads) {
    const int r = x / (D / 4), c = 4 * (x % (D / 4));
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nrows) v = *reinterpret_cast<const float4*>(qm + (size_t)r * D + c);
    *reinterpret_cast<float4*>(qa + r * LD + c) = make_float4(mul * v.x, mul * v.y, mul * v.z, mul * v.w);
    if (t2) {
      const float hs = 0.5f * scale * scale;
      *reinterpret_cast<float4*>(qw + r * LD + c) =
          make_float4(hs * v.x * v.x, hs * v.y * v.y, hs * v.z * v.z, hs * v.w * v.w);
    }
  }
  if (proj) {
    // T = q̄ P_q into the score rows, then u = T P_kᵀ (u_c = Σ_n P_k[c][n] T_n) into qa
    float* T = sc;
    stage_rows<D, 2 * kMT, kMmaThreads>(tiles, Pq, 0, D);   // rows k of P_q
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (warp < kMmaWarps) {
      float acc[3][NTP][4] = {};
      warp_tf32<D, NTP, false>(acc, qa, LD, tiles, 8 * NTP * warp, lane);
#pragma unroll
      for (int nt = 0; nt < NTP; ++nt) {
        const int c = 8 * NTP * warp + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(T + g * LD + c) = make_float2(tf32_sum(acc, nt, 0), tf32_sum(acc, nt, 1));
        *reinterpret_cast<float2*>(T + (g + 8) * LD + c) = make_float2(tf32_sum(acc, nt, 2), tf32_sum(acc, nt, 3));
      }
    }
    __syncthreads();
    stage_rows<D, 2 * kMT, kMmaThreads>(tiles, Pk, 0, D);   // rows c of P_k
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (warp < kMmaWarps) {
      float acc[3][NTP][4] = {};
      warp_tf32<D, NTP, true>(acc, T, LD, tiles, 8 * NTP * warp, lane);
#pragma unroll
      for (int nt = 0; nt < NTP; ++nt) {
        const int c = 8 * NTP * warp + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(qa + g * LD + c) = make_float2(tf32_sum(acc, nt, 0), tf32_sum(acc, nt, 1));
        *reinterpret_cast<float2*>(qa + (g + 8) * LD + c) = make_float2(tf32_sum(acc, nt, 2), tf32_sum(acc, nt, 3));
      }
    }
    __syncthreads();                              // P_k is read before its buffer takes the first tile
    stage(0, 0);
  }
  __syncthreads();
  if (cov && warp < kMQ) {
    float ss = 0.f;
    for (int c = lane; c < D; c += 32) ss = fmaf(qa[warp * LD + c], qa[warp * LD + c], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) qn[warp] = sqrtf(ss) * inv_blk;
  }
  const float* cvn = cov ? st.covnorm + bh * (size_t)nb : nullptr;

  // ---- scores: tiles of kMT centroids, two buffers
  for (int tt = 0; tt < ntiles; ++tt) {
    if (tt + 1 < ntiles) {
      stage(tt + 1, (tt + 1) & 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    if (warp < kMmaWarps) {
      const float* tk = tiles + (size_t)(tt & 1) * narr * TS;
      float acc[3][1][4] = {};
      warp_tf32<D, 1, true>(acc, qa, LD, tk, 8 * warp, lane);
      float o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = tf32_sum(acc, 0, e);
      if (t2) {
        float acc2[3][1][4] = {};
        warp_tf32<D, 1, true>(acc2, qw, LD, tk + TS, 8 * warp, lane);
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] += log1pf(tf32_sum(acc2, 0, e));
      }
      const int j = tt * kMT + 8 * warp + 2 * t;
      if (cov) {
        const float m0 = j < nb ? cvn[j] : 0.f, m1 = j + 1 < nb ? cvn[j + 1] : 0.f;
        o[0] += log1pf(qn[g] * m0);
        o[1] += log1pf(qn[g] * m1);
        o[2] += log1pf(qn[g + 8] * m0);
        o[3] += log1pf(qn[g + 8] * m1);
      }
      if (j + 1 < nb) {
        *reinterpret_cast<float2*>(sc + (size_t)g * ldc + j) = make_float2(o[0], o[1]);
        *reinterpret_cast<float2*>(sc + (size_t)(g + 8) * ldc + j) = make_float2(o[2], o[3]);
      } else if (j < nb) {
        sc[(size_t)g * ldc + j] = o[0];
        sc[(size_t)(g + 8) * ldc + j] = o[2];
      }
    }
    __syncthreads();   // this buffer is restaged by the next iteration's prefetch
  }
  // ---- one row per warp: the scores out, then the selection
  if (warp < nrows) {
    const float* row = sc + (size_t)warp * ldc;
    if (scores_out) {
      float* so = scores_out + (bh * nb + i0 + warp) * (size_t)nb;
      for (int jj = lane; jj < nb; jj += 32) so[jj] = row[jj];
    }
    const int nwords = (nb + 31) >> 5;
    uint32_t* bits = reinterpret_cast<uint32_t*>(tiles) + warp * nwords;
    select_row(row, bits, nb, nwords, topk, lane, block_idx + (bh * nb + i0 + warp) * (size_t)topk);
  }
}

// shared memory of route_mma_kernel (dynamic part): the query rows, two tile
// buffers and the score rows, which the proj router's T = q̄ P_q (16 rows of
// d + 4 floats) uses first
size_t route_mma_smem_bytes(int nb, int d, bool t2, bool proj) {
  const size_t A = (size_t)kMQ * (d + 4) * (t2 ? 2 : 1);
  const size_t tiles = 2 * (size_t)(t2 ? 2 : 1) * kMT * (d + 4);
  size_t rows = (size_t)kMQ * route_ldc(nb);
  if (proj && rows < (size_t)kMQ * (d + 4)) rows = (size_t)kMQ * (d + 4);
  return 4 * (A + tiles + rows);
}

template <int D>
sa_status launch_route_mma(const sa_block_stats& st, sa_shape shape, int nb, sa_route_mode mode, const float* Pq,
                           const float* Pk, float scale, float inv_blk, int topk, int32_t* idx, float* scores,
                           size_t smem, cudaStream_t s) {
  auto kern = route_mma_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(route_mma_kernel)");
  dim3 grid((nb + kMQ - 1) / kMQ, shape.H, shape.B);
  const cudaError_t le = launch_pdl(kern, grid, dim3(kMmaThreads), smem, s, st, shape.H, nb, mode, Pq, Pk, scale,
                                    inv_blk, topk, idx, scores);
  if (le != cudaSuccess) return fail(SA_ERR_CUDA, std::string("route_mma_kernel: ") + cudaGetErrorString(le));
  return launch_status("route_mma_kernel");
}

struct RouteCfg {
  int rpw, ncol;
};

size_t route_smem_bytes(int nb, int d, int topk, bool t2, RouteCfg c) {
  const int qb = kRouteWarps * c.rpw;
  const int nwords = (nb + 31) / 32;
  size_t tiles = 2 * (size_t)(t2 ? 2 : 1) * 32 * c.ncol * (d + 4);
  if (topk > kWarpTopkMax) {
    int n2 = 1;
    while (n2 < nb) n2 <<= 1;
    if (2 * (size_t)n2 > tiles) tiles = 2 * (size_t)n2;
  }
  return 4 * (2 * (size_t)qb * d + tiles + (size_t)qb * nb + (size_t)qb * nwords);
}

// Rows per warp and centroid columns per lane: the first of (2, 2), (2, 1),
// (1, 2), (1, 1) that lets two CTAs share an SM, else the first that fits
// in one CTA.
RouteCfg route_cfg(int nb, int d, int topk, bool t2) {
  const RouteCfg order[4] = {{2, 2}, {2, 1}, {1, 2}, {1, 1}};
  for (const RouteCfg& c : order)
    if (route_smem_bytes(nb, d, topk, t2, c) <= kSmemTwoPerSm) return c;
  for (const RouteCfg& c : order)
    if (route_smem_bytes(nb, d, topk, t2, c) <= kMaxSmemPerCta) return c;
  return order[3];
}

template <int D, int RPW, int NCOL>
sa_status launch_route(const sa_block_stats& st, sa_shape shape, int nb, sa_route_mode mode, const float* Pq,
                       const float* Pk, float scale, float inv_blk, int topk, int32_t* idx, float* scores,
                       size_t smem, cudaStream_t s) {
  auto kern = route_kernel<D, RPW, NCOL>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(route_kernel)");
  constexpr int QB = kRouteWarps * RPW;
  dim3 grid((nb + QB - 1) / QB, shape.H, shape.B);
  const cudaError_t le = launch_pdl(kern, grid, dim3(kRouteThreads), smem, s, st, shape.H, nb, mode, Pq, Pk, scale,
                                    inv_blk, topk, idx, scores);
  if (le != cudaSuccess) return fail(SA_ERR_CUDA, std::string("route_kernel: ") + cudaGetErrorString(le));
  return launch_status("route_kernel");
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
  if (mode != SA_ROUTE_DOT && mode != SA_ROUTE_PROJ && mode != SA_ROUTE_TAYLOR2 && mode != SA_ROUTE_COV)
    return fail(SA_ERR_INVALID_ARG, "sa_route: unknown route mode");
  if (mode == SA_ROUTE_PROJ && (!proj_q || !proj_k))
    return fail(SA_ERR_INVALID_ARG, "sa_route: SA_ROUTE_PROJ needs proj_q and proj_k");
  if (mode == SA_ROUTE_TAYLOR2 && !stats->kvar)
    return fail(SA_ERR_INVALID_ARG, "sa_route: SA_ROUTE_TAYLOR2 needs stats->kvar");
  if (mode == SA_ROUTE_COV && !stats->covnorm)
    return fail(SA_ERR_INVALID_ARG, "sa_route: SA_ROUTE_COV needs stats->covnorm");
  if (topk < 0 || topk > nb) return fail(SA_ERR_INVALID_ARG, "sa_route: topk must be in [0, N/block]");
  if (nb > kMaxRouteBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_route: at most 4096 blocks per head");
  const void* ptrs[] = {stats->qmean, stats->kmean, stats->kvar, stats->covnorm, proj_q, proj_k, block_idx, scores};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_route: pointers must be 16-byte aligned");
  const bool t2 = mode == SA_ROUTE_TAYLOR2;
  cudaStream_t s = as_stream(stream);
  const sa_block_stats& st = *stats;
  const float inv_blk = 1.0f / (float)shape.block;
  // the tensor-core kernel takes every k of the warp select whose rows fit
  const size_t mma_smem = route_mma_smem_bytes(nb, shape.d, t2, mode == SA_ROUTE_PROJ);
  if (topk <= kWarpTopkMax && mma_smem + 1024 <= kMaxSmemPerCta) {
    if (shape.d == 128)
      return launch_route_mma<128>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, mma_smem, s);
    return launch_route_mma<64>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, mma_smem, s);
  }
  const RouteCfg cfg = route_cfg(nb, shape.d, topk, t2);
  const size_t smem = route_smem_bytes(nb, shape.d, topk, t2, cfg);
  const int key = (shape.d == 128 ? 4 : 0) + (cfg.rpw == 2 ? 2 : 0) + (cfg.ncol == 2 ? 1 : 0);
  switch (key) {
    case 7: return launch_route<128, 2, 2>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
    case 6: return launch_route<128, 2, 1>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
    case 5: return launch_route<128, 1, 2>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
    case 4: return launch_route<128, 1, 1>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
    case 3: return launch_route<64, 2, 2>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
    case 2: return launch_route<64, 2, 1>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
    case 1: return launch_route<64, 1, 2>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
    default: return launch_route<64, 1, 1>(st, shape, nb, mode, proj_q, proj_k, scale, inv_blk, topk, block_idx, scores, smem, s);
  }
}

