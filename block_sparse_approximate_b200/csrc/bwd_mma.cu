// Backward of the sparse prefill on the tensor cores (bf16 operands, fp32
// accumulation, warp-level mma.sync m16n8k16) for d = 128: the same
// gradients as the CUDA-core kernels in bwd.cu, which remain the path for
// fp32 and d = 64.  Tiles are 64 rows (or keys) of 128 bf16 channels in
// shared memory with 16-byte chunks XOR-swizzled by the row (conflict-free
// ldmatrix); four warps each own 16 rows (or keys) of a tile.
//   bwd_dq_mma_kernel   per 64 query rows: pass 1 recomputes S over the row's
//                       exact and pseudo-key tiles and writes lse and δ =
//                       dO·O; pass 2 forms P, dP = dO Vᵀ, dS = P (dP − δ) and
//                       accumulates dQ = s dS K.
//   bwd_dkv_mma_kernel  per 64 keys: over the 64-row chunks of the query
//                       blocks that attend to them, Sᵀ = K Qᵀ, Pᵀ, dPᵀ = V dOᵀ,
//                       dV += Pᵀ dO, dK += s dSᵀ Q.  Exact keys: the query
//                       blocks that selected the block, dK and dV written.
//                       Pseudo-keys (zero-order tail): 64 centroids against
//                       every query row whose block left them unselected;
//                       their gradients are added ÷B to their blocks' tokens.
// P and dS are rounded to bf16 for the second products, as the forward
// rounds P.  Sums over query blocks run in a fixed order (no atomics).
#include "attn_simt.cuh"

namespace sa {
namespace {

constexpr int kMD = 128;                        // head dim
constexpr int kMThreads = 128;                  // four warps
constexpr int kMT = 64;                         // rows / keys per tile
constexpr uint32_t kMRowB = kMD * 2;            // bytes per bf16 row
constexpr uint32_t kMTileB = kMT * kMRowB;      // 16 KB

__device__ __forceinline__ uint32_t swz(int r, int chunk) {
  return (uint32_t)r * kMRowB + ((uint32_t)(chunk ^ (r & 7)) << 4);
}
__device__ __forceinline__ void cpa16(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cpa_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pk(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Copies 64 rows of 128 bf16 (rows [0, nvalid) from src with row stride
// kMD, the rest zero) into a swizzled tile; all 128 threads take part.
__device__ __forceinline__ void stage64(uint32_t dst, const __nv_bfloat16* src, int nvalid) {
  for (int x = threadIdx.x; x < kMT * 16; x += kMThreads) {
    const int r = x >> 4, c = x & 15;
    const bool ok = r < nvalid;
    cpa16(dst + swz(r, c), src + (size_t)(ok ? r : 0) * kMD + 8 * c, ok ? 16u : 0u);
  }
}

// A fragment (16 rows from rb, k-step kk of 16 channels) of a swizzled tile
__device__ __forceinline__ void lda(uint32_t (&a)[4], uint32_t tile, int rb, int kk) {
  const int lane = threadIdx.x & 31;
  ldsm4(a, tile + swz(rb + (lane & 15), 2 * kk + (lane >> 4)));
}
// B fragments of one n-tile of 8 rows from nb (rows = n, channels = k) for
// the k-steps 2 kp and 2 kp + 1: b[0], b[1] and b[2], b[3]
__device__ __forceinline__ void ldb_rows(uint32_t (&b)[4], uint32_t tile, int nb, int kp) {
  const int lane = threadIdx.x & 31;
  ldsm4(b, tile + swz(nb + (lane & 7), 4 * kp + (lane >> 3)));
}
// B fragments with k = the tile's rows kb .. kb + 15 and n = channels of the
// four n-tiles 4 nq .. 4 nq + 3: b0 in lo[e], b1 in hi[e]
__device__ __forceinline__ void ldb_cols(uint32_t (&lo)[4], uint32_t (&hi)[4], uint32_t tile, int kb, int nq) {
  const int lane = threadIdx.x & 31;
  ldsm4t(lo, tile + swz(kb + (lane & 7), 4 * nq + (lane >> 3)));
  ldsm4t(hi, tile + swz(kb + 8 + (lane & 7), 4 * nq + (lane >> 3)));
}

// ---- dQ (and lse, δ) --------------------------------------------------------
template <int BLK>
__global__ void __launch_bounds__(kMThreads)
bwd_dq_mma_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                  const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ O,
                  const __nv_bfloat16* __restrict__ dO, const __nv_bfloat16* __restrict__ kb16,
                  const __nv_bfloat16* __restrict__ vb16, int H, int N, const int32_t* __restrict__ block_idx,
                  int topk, int zo, float scale, float* __restrict__ lse2, float* __restrict__ delta,
                  float* __restrict__ dQ) {
  constexpr int PB = BLK / kMT;                     // exact tiles per block
  const int nb = N / BLK;
  const int row0 = blockIdx.x * kMT, i = row0 / BLK;
  const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
  const size_t head = bh * (size_t)N * kMD;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;           // MMA row group, thread in group
  const int rb = 16 * warp;                         // this warp's rows of the tile
  const float scale2 = scale * kLog2e, bias_c = log2f((float)BLK);
  extern __shared__ __align__(128) uint8_t msm[];
  const uint32_t sQ = (uint32_t)__cvta_generic_to_shared(msm);
  const uint32_t sG = sQ + kMTileB;
  const uint32_t sK0 = sG + kMTileB;                // ring of 2 x (K, V)
  uint32_t* sel_bits = reinterpret_cast<uint32_t*>(msm + 6 * kMTileB);
  const int nwords = (nb + 31) >> 5;
  const int32_t* sel = block_idx + (bh * nb + i) * (size_t)topk;
  for (int w = tid; w < nwords; w += kMThreads) sel_bits[w] = 0u;
  __syncthreads();
  for (int x = tid; x < topk; x += kMThreads) atomicOr(&sel_bits[sel[x] >> 5], 1u << (sel[x] & 31));
  const int ntex = topk * PB, ntc = zo ? (nb + kMT - 1) / kMT : 0, nt = ntex + ntc;

  auto issue = [&](int t, int slot) {
    const uint32_t dk = sK0 + slot * 2 * kMTileB, dv = dk + kMTileB;
    if (t < ntex) {
      const size_t off = head + ((size_t)sel[t / PB] * BLK + (t % PB) * kMT) * kMD;
      stage64(dk, K + off, kMT);
      stage64(dv, V + off, kMT);
    } else {
      const int j0 = (t - ntex) * kMT;
      const size_t off = (bh * nb + j0) * (size_t)kMD;
      stage64(dk, kb16 + off, min(kMT, nb - j0));
      stage64(dv, vb16 + off, min(kMT, nb - j0));
    }
    cpa_commit();
  };
  stage64(sQ, Q + head + (size_t)row0 * kMD, kMT);
  stage64(sG, dO + head + (size_t)row0 * kMD, kMT);
  cpa_commit();

  // rows of this thread: rb + g and rb + g + 8
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f}, lse[2], dl[2];
  // key validity and bias of tile t for the thread's columns 8 n + 2 tg + {0, 1}
  auto key_ok = [&](int t, int col) {
    if (t < ntex) return true;
    const int j = (t - ntex) * kMT + col;
    return j < nb && !((sel_bits[j >> 5] >> (j & 31)) & 1u);
  };
  // S = Q Kᵀ of the warp's 16 rows against the staged 64 keys
  auto scores = [&](uint32_t tk, float (&S)[8][4]) {
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) S[n][e] = 0.f;
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {
      uint32_t a0[4], a1[4];
      lda(a0, sQ, rb, 2 * kp);
      lda(a1, sQ, rb, 2 * kp + 1);
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        uint32_t b[4];
        ldb_rows(b, tk, 8 * n, kp);
        mma(S[n], a0, b[0], b[1]);
        mma(S[n], a1, b[2], b[3]);
      }
    }
  };

  // ---- pass 1: lse over every key tile
  for (int pass = 0; pass < 2; ++pass) {
    float dq[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;
    if (nt > 0) issue(0, 0);
    for (int t = 0; t < nt; ++t) {
      if (t + 1 < nt) {
        issue(t + 1, (t + 1) & 1);
        cpa_wait<1>();
      } else {
        cpa_wait<0>();
      }
      __syncthreads();
      const uint32_t tk = sK0 + (t & 1) * 2 * kMTileB, tv = tk + kMTileB;
      const float bias = t < ntex ? 0.f : bias_c;
      float S[8][4];
      scores(tk, S);
      if (pass == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float mx = -INFINITY;
#pragma unroll
          for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float x = key_ok(t, 8 * n + 2 * tg + e) ? fmaf(S[n][2 * h + e], scale2, bias) : -INFINITY;
              S[n][2 * h + e] = x;
              mx = fmaxf(mx, x);
            }
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const float mn = fmaxf(m_r[h], mx);
          if (mn == -INFINITY) continue;
          float sm = 0.f;
#pragma unroll
          for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) sm += fast_exp2(S[n][2 * h + e] - mn);
          sm += __shfl_xor_sync(0xffffffffu, sm, 1);
          sm += __shfl_xor_sync(0xffffffffu, sm, 2);
          l_r[h] = l_r[h] * (m_r[h] == -INFINITY ? 0.f : fast_exp2(m_r[h] - mn)) + sm;
          m_r[h] = mn;
        }
      } else {
        // dP = dO Vᵀ
        float P[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) P[n][e] = 0.f;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          uint32_t a0[4], a1[4];
          lda(a0, sG, rb, 2 * kp);
          lda(a1, sG, rb, 2 * kp + 1);
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            uint32_t b[4];
            ldb_rows(b, tv, 8 * n, kp);
            mma(P[n], a0, b[0], b[1]);
            mma(P[n], a1, b[2], b[3]);
          }
        }
        // dS = p (dP − δ), then dQ += dS K (K as the k = key operand)
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h = e >> 1;
            const float p = key_ok(t, 8 * n + 2 * tg + (e & 1)) ? fast_exp2(fmaf(S[n][e], scale2, bias) - lse[h]) : 0.f;
            S[n][e] = p * (P[n][e] - dl[h]);
          }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t a[4];
          a[0] = pk(S[2 * kk][0], S[2 * kk][1]);
          a[1] = pk(S[2 * kk][2], S[2 * kk][3]);
          a[2] = pk(S[2 * kk + 1][0], S[2 * kk + 1][1]);
          a[3] = pk(S[2 * kk + 1][2], S[2 * kk + 1][3]);
#pragma unroll
          for (int nq = 0; nq < 4; ++nq) {
            uint32_t lo[4], hi[4];
            ldb_cols(lo, hi, tk, 16 * kk, nq);
#pragma unroll
            for (int e = 0; e < 4; ++e) mma(dq[4 * nq + e], a, lo[e], hi[e]);
          }
        }
      }
      __syncthreads();   // the slot is restaged two tiles later
    }
    cpa_wait<0>();
    if (pass == 0) {
      // lse and δ of the thread's two rows (δ from the stored bf16 output)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = row0 + rb + g + 8 * h;
        lse[h] = l_r[h] > 0.f ? m_r[h] + log2f(l_r[h]) : INFINITY;
        float dd = 0.f;
        for (int c = 2 * tg; c < kMD; c += 8) {
          const size_t gi = head + (size_t)row * kMD + c;
          dd = fmaf(__bfloat162float(dO[gi]), __bfloat162float(O[gi]), dd);
          dd = fmaf(__bfloat162float(dO[gi + 1]), __bfloat162float(O[gi + 1]), dd);
        }
        dd += __shfl_xor_sync(0xffffffffu, dd, 1);
        dd += __shfl_xor_sync(0xffffffffu, dd, 2);
        dl[h] = dd;
        if (tg == 0) {
          lse2[bh * N + row] = lse[h];
          delta[bh * N + row] = dd;
        }
      }
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = row0 + rb + g + 8 * h;
          float2 v = make_float2(scale * dq[n][2 * h], scale * dq[n][2 * h + 1]);
          *reinterpret_cast<float2*>(dQ + head + (size_t)row * kMD + 8 * n + 2 * tg) = v;
        }
    }
  }
}

// ---- dK, dV ---------------------------------------------------------------
// CENT = false: 64 exact keys (block j, half `blockIdx.x % (BLK/64)`) over
// the query blocks that selected block j (offs/list).  CENT = true: 64
// centroids over one of kCentSplits ranges of the query rows (so that the
// few centroid tiles still fill the GPU), masked where the row's block
// selected the centroid; the partial dk̄, dv̄ go to `part`, which
// bwd_centroid_scatter_kernel sums in order and spreads ÷B over the blocks.
constexpr int kCentSplits = 16;
template <int BLK, bool CENT>
__global__ void __launch_bounds__(kMThreads)
bwd_dkv_mma_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                   const __nv_bfloat16* __restrict__ V, const __nv_bfloat16* __restrict__ dO,
                   const __nv_bfloat16* __restrict__ kb16, const __nv_bfloat16* __restrict__ vb16, int H, int N,
                   const int32_t* __restrict__ block_idx, int topk, const int32_t* __restrict__ offs,
                   const int32_t* __restrict__ list, float scale, const float* __restrict__ lse2,
                   const float* __restrict__ delta, float* __restrict__ dK, float* __restrict__ dV,
                   float* __restrict__ part) {
  const int nb = N / BLK;
  const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
  const size_t head = bh * (size_t)N * kMD;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tg = lane & 3;
  const int rb = 16 * warp;
  const float scale2 = scale * kLog2e, bias = CENT ? log2f((float)BLK) : 0.f;
  extern __shared__ __align__(128) uint8_t msm[];
  const uint32_t sK = (uint32_t)__cvta_generic_to_shared(msm);
  const uint32_t sV = sK + kMTileB;
  const uint32_t sR0 = sV + kMTileB;                // ring of 2 x (Q chunk, dO chunk)
  float* lsd = reinterpret_cast<float*>(msm + 6 * kMTileB);   // [2 slots][lse 64, δ 64]
  // the CTA's keys: exact tokens or centroids
  int key0, nkeys, j = 0;
  const int split = CENT ? (int)blockIdx.x % kCentSplits : 0;
  if (CENT) {
    key0 = ((int)blockIdx.x / kCentSplits) * kMT;
    nkeys = min(kMT, nb - key0);
    stage64(sK, kb16 + (bh * nb + key0) * (size_t)kMD, nkeys);
    stage64(sV, vb16 + (bh * nb + key0) * (size_t)kMD, nkeys);
  } else {
    j = blockIdx.x / (BLK / kMT);
    key0 = j * BLK + (blockIdx.x % (BLK / kMT)) * kMT;
    nkeys = kMT;
    stage64(sK, K + head + (size_t)key0 * kMD, kMT);
    stage64(sV, V + head + (size_t)key0 * kMD, kMT);
  }
  cpa_commit();
  // row chunks: exact — the BLK / 64 chunks of every listed query block;
  // centroids — every 64-row chunk of the head
  const int32_t* off = offs + bh * (size_t)(nb + 1);
  const int32_t* lst = list + bh * (size_t)nb * topk;
  const int per_q = BLK / kMT;
  // centroids: this split's range [c_lo, c_lo + nchunks) of the head's 64-row chunks
  const int all_chunks = N / kMT;
  const int c_lo = CENT ? (int)(((long)all_chunks * split) / kCentSplits) : 0;
  const int nchunks = CENT ? (int)(((long)all_chunks * (split + 1)) / kCentSplits) - c_lo
                           : (off[j + 1] - off[j]) * per_q;
  auto chunk_row0 = [&](int c) {
    return CENT ? (c_lo + c) * kMT : lst[off[j] + c / per_q] * BLK + (c % per_q) * kMT;
  };
  auto issue = [&](int c, int slot) {
    const int r0 = chunk_row0(c);
    const uint32_t dq = sR0 + slot * 2 * kMTileB;
    stage64(dq, Q + head + (size_t)r0 * kMD, kMT);
    stage64(dq + kMTileB, dO + head + (size_t)r0 * kMD, kMT);
    float* l = lsd + slot * 2 * kMT;
    for (int x = tid; x < kMT / 4; x += kMThreads) {
      cpa16((uint32_t)__cvta_generic_to_shared(l + 4 * x), lse2 + bh * N + r0 + 4 * x, 16u);
      cpa16((uint32_t)__cvta_generic_to_shared(l + kMT + 4 * x), delta + bh * N + r0 + 4 * x, 16u);
    }
    cpa_commit();
  };
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dk[n][e] = 0.f;
      dv[n][e] = 0.f;
    }
  // centroid mode: are the thread's two centroids selected by the chunk's block?
  int cur_q = -1;
  bool unsel[2] = {true, true};
  if (nchunks > 0) issue(0, 0);
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) {
      issue(c + 1, (c + 1) & 1);
      cpa_wait<1>();
    } else {
      cpa_wait<0>();
    }
    __syncthreads();
    const uint32_t tq = sR0 + (c & 1) * 2 * kMTileB, tgo = tq + kMTileB;
    const float* ls = lsd + (c & 1) * 2 * kMT;
    if (CENT) {
      const int qi = chunk_row0(c) / BLK;
      if (qi != cur_q) {
        cur_q = qi;
        const int32_t* sel = block_idx + (bh * nb + qi) * (size_t)topk;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int jj = key0 + rb + g + 8 * h;
          bool s = false;
          for (int x = 0; x < topk; ++x) s |= sel[x] == jj;
          unsel[h] = !s && jj < nb;
        }
      }
    }
    // Sᵀ = K Qᵀ and dPᵀ = V dOᵀ for the warp's 16 keys and the chunk's 64 rows
    float S[8][4], P[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        S[n][e] = 0.f;
        P[n][e] = 0.f;
      }
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {
      uint32_t a0[4], a1[4], v0[4], v1[4];
      lda(a0, sK, rb, 2 * kp);
      lda(a1, sK, rb, 2 * kp + 1);
      lda(v0, sV, rb, 2 * kp);
      lda(v1, sV, rb, 2 * kp + 1);
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        uint32_t b[4], bg[4];
        ldb_rows(b, tq, 8 * n, kp);
        ldb_rows(bg, tgo, 8 * n, kp);
        mma(S[n], a0, b[0], b[1]);
        mma(S[n], a1, b[2], b[3]);
        mma(P[n], v0, bg[0], bg[1]);
        mma(P[n], v1, bg[2], bg[3]);
      }
    }
    // p and ds (rows of the MMA = keys, columns = query rows of the chunk)
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = e >> 1, col = 8 * n + 2 * tg + (e & 1);
        const bool ok = CENT ? unsel[h] : true;
        const float p = ok ? fast_exp2(fmaf(S[n][e], scale2, bias) - ls[col]) : 0.f;
        S[n][e] = p;
        P[n][e] = p * (P[n][e] - ls[kMT + col]);
      }
    // dV += Pᵀ dO, dK += dSᵀ Q (k = the chunk's rows)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ap[4], as[4];
      ap[0] = pk(S[2 * kk][0], S[2 * kk][1]);
      ap[1] = pk(S[2 * kk][2], S[2 * kk][3]);
      ap[2] = pk(S[2 * kk + 1][0], S[2 * kk + 1][1]);
      ap[3] = pk(S[2 * kk + 1][2], S[2 * kk + 1][3]);
      as[0] = pk(P[2 * kk][0], P[2 * kk][1]);
      as[1] = pk(P[2 * kk][2], P[2 * kk][3]);
      as[2] = pk(P[2 * kk + 1][0], P[2 * kk + 1][1]);
      as[3] = pk(P[2 * kk + 1][2], P[2 * kk + 1][3]);
#pragma unroll
      for (int nq = 0; nq < 4; ++nq) {
        uint32_t lo[4], hi[4];
        ldb_cols(lo, hi, tgo, 16 * kk, nq);
#pragma unroll
        for (int e = 0; e < 4; ++e) mma(dv[4 * nq + e], ap, lo[e], hi[e]);
        ldb_cols(lo, hi, tq, 16 * kk, nq);
#pragma unroll
        for (int e = 0; e < 4; ++e) mma(dk[4 * nq + e], as, lo[e], hi[e]);
      }
    }
    __syncthreads();   // the slot is restaged two chunks later
  }
  cpa_wait<0>();
  // results: MMA rows = keys rb + g (+8), columns 8 n + 2 tg (+1) = channels
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int kr = rb + g + 8 * h;
    if (kr >= nkeys) continue;
    if (CENT) {
      // partial sums of this split: part[2][split][bh][centroid][channel]
      const int jj = key0 + kr;
      const size_t BHn = (size_t)gridDim.y * gridDim.z;
      float* pk_ = part + (((size_t)split * BHn + bh) * nb + jj) * kMD;
      float* pv_ = part + (((size_t)(kCentSplits + split) * BHn + bh) * nb + jj) * kMD;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        *reinterpret_cast<float2*>(pk_ + 8 * n + 2 * tg) = make_float2(dk[n][2 * h], dk[n][2 * h + 1]);
        *reinterpret_cast<float2*>(pv_ + 8 * n + 2 * tg) = make_float2(dv[n][2 * h], dv[n][2 * h + 1]);
      }
    } else {
      float* dkr = dK + head + (size_t)(key0 + kr) * kMD;
      float* dvr = dV + head + (size_t)(key0 + kr) * kMD;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        *reinterpret_cast<float2*>(dkr + 8 * n + 2 * tg) = make_float2(scale * dk[n][2 * h], scale * dk[n][2 * h + 1]);
        *reinterpret_cast<float2*>(dvr + 8 * n + 2 * tg) = make_float2(dv[n][2 * h], dv[n][2 * h + 1]);
      }
    }
  }
}

// dk̄_j, dv̄_j = the splits' partial sums in order; s dk̄_j / B and dv̄_j / B
// added to each token of block j (one CTA per centroid, thread = channel).
template <int BLK>
__global__ void __launch_bounds__(kMD)
bwd_centroid_scatter_kernel(const float* __restrict__ part, int H, int N, float scale, float* __restrict__ dK,
                            float* __restrict__ dV) {
  const int nb = N / BLK;
  const int j = blockIdx.x, c = threadIdx.x;
  const size_t bh = (size_t)blockIdx.z * H + blockIdx.y;
  const size_t BHn = (size_t)gridDim.y * gridDim.z;
  float sk = 0.f, sv = 0.f;
  for (int sp = 0; sp < kCentSplits; ++sp) {
    sk += part[(((size_t)sp * BHn + bh) * nb + j) * kMD + c];
    sv += part[(((size_t)(kCentSplits + sp) * BHn + bh) * nb + j) * kMD + c];
  }
  sk *= scale / BLK;
  sv *= 1.0f / BLK;
  const size_t base = (bh * (size_t)N + (size_t)j * BLK) * kMD + c;
  for (int t = 0; t < BLK; ++t) {
    dK[base + (size_t)t * kMD] += sk;
    dV[base + (size_t)t * kMD] += sv;
  }
}

}  // namespace

size_t bwd_tc_part_bytes(const sa_shape& s) {
  return 2 * (size_t)kCentSplits * s.B * s.H * (size_t)(s.N / s.block) * kMD * sizeof(float);
}

bool bwd_tc_supports(sa_dtype dtype, const sa_shape& s, bool zo, const sa_block_stats& st) {
  return dtype == SA_BF16 && s.d == kMD && (s.block == 64 || s.block == 128) &&
         (!zo || (st.kmean_bf16 && st.vmean_bf16));
}

template <int BLK>
sa_status bwd_tc_launch(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                        const sa_shape& s, const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st,
                        float scale, float* dQ, float* dK, float* dV, const float* lse_in, float* lse2,
                        float* delta, const int32_t* offs, const int32_t* list, float* part, cudaStream_t stream,
                        const BwdTailTerms* fo) {
  using bf = __nv_bfloat16;
  const int nb = s.N / BLK;
  const bf* q = static_cast<const bf*>(Q);
  const bf* k = static_cast<const bf*>(K);
  const bf* v = static_cast<const bf*>(V);
  const bf* g = static_cast<const bf*>(dO);
  const bf* kb = reinterpret_cast<const bf*>(st.kmean_bf16);
  const bf* vb = reinterpret_cast<const bf*>(st.vmean_bf16);
  if (BLK == 128 && (topk > 0 || zo)) {
    sa_status r = bwd_dq_tc(Q, K, V, O, dO, s, block_idx, topk, zo, st, scale, lse_in, lse2, delta, dQ, stream, fo);
    if (r != SA_OK) return r;
  } else {
    const size_t smem = 6 * (size_t)kMTileB + sizeof(uint32_t) * ((nb + 31) / 32);
    auto kern = bwd_dq_mma_kernel<BLK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(bwd_dq_mma_kernel)");
    kern<<<dim3(s.N / kMT, s.H, s.B), kMThreads, smem, stream>>>(q, k, v, static_cast<const bf*>(O), g, kb, vb, s.H,
                                                                 s.N, block_idx, topk, zo, scale, lse2, delta, dQ);
    sa_status r = launch_status("bwd_dq_mma_kernel");
    if (r != SA_OK) return r;
  }
  const size_t smem = 6 * (size_t)kMTileB + 2 * 2 * kMT * sizeof(float);
  if constexpr (BLK == 128) {
    return bwd_dkv_tc(Q, K, V, dO, s, block_idx, topk, zo, st, offs, list, scale, lse2, delta, dK, dV, part,
                      kCentSplits, stream, fo ? fo->delta_c : nullptr);
  } else {
    auto kern = bwd_dkv_mma_kernel<BLK, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(bwd_dkv_mma_kernel)");
    kern<<<dim3(nb * (BLK / kMT), s.H, s.B), kMThreads, smem, stream>>>(q, k, v, g, kb, vb, s.H, s.N, block_idx,
                                                                       topk, offs, list, scale, lse2, delta, dK, dV,
                                                                       part);
    sa_status r = launch_status("bwd_dkv_mma_kernel");
    if (r != SA_OK || !zo) return r;
  }
  auto kern = bwd_dkv_mma_kernel<BLK, true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(bwd_dkv_mma_kernel)");
  kern<<<dim3(((nb + kMT - 1) / kMT) * kCentSplits, s.H, s.B), kMThreads, smem, stream>>>(
      q, k, v, g, kb, vb, s.H, s.N, block_idx, topk, offs, list, scale, lse2, delta, dK, dV, part);
  sa_status r = launch_status("bwd_dkv_mma_kernel(centroids)");
  if (r != SA_OK) return r;
  bwd_centroid_scatter_kernel<BLK><<<dim3(nb, s.H, s.B), kMD, 0, stream>>>(part, s.H, s.N, scale, dK, dV);
  return launch_status("bwd_centroid_scatter_kernel");
}

sa_status bwd_tc(const void* Q, const void* K, const void* V, const void* O, const void* dO, const sa_shape& s,
                 const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st, float scale, float* dQ,
                 float* dK, float* dV, const float* lse_in, float* lse2, float* delta, const int32_t* offs,
                 const int32_t* list, float* part, cudaStream_t stream, const BwdTailTerms* fo) {
  if (s.block == 128)
    return bwd_tc_launch<128>(Q, K, V, O, dO, s, block_idx, topk, zo, st, scale, dQ, dK, dV, lse_in, lse2, delta,
                              offs, list, part, stream, fo);
  if (fo) return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_bwd: the first-order tail needs block 128");
  return bwd_tc_launch<64>(Q, K, V, O, dO, s, block_idx, topk, zo, st, scale, dQ, dK, dV, lse_in, lse2, delta,
                           offs, list, part, stream, nullptr);
}

}  // namespace sa
