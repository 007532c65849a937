// Sparse prefill on CUDA cores: the general path for fp32 inputs, block 64,
// d 64, and every tail mode.  One CTA per (64 query rows, head, batch); each
// warp owns 8 query rows whose online-softmax state (max, sum, accumulator)
// lives in shared memory (FlashAttention-style, as PISA's fused kernel
// interleaves the exact and the approximate scans inside one online softmax,
// "Implementação de Hardware").
//   exact part:  the selected KV blocks S_i, token by token;
//   zero-order:  every unselected block j as one pseudo-key with key k̄_j,
//                value vsum_j / B and log-weight ln B (B e^{x} = e^{x + ln B}),
//                which puts exp(s q·k̄_j)·vsum_j in the numerator and
//                B·exp(s q·k̄_j) in the denominator (PISA §2, N_t and D_t);
//   first-order: the zero-order pass, with each row's sum of the pseudo-key
//                weights Λ_t = Σ_{j∈U} e^{s q·k̄_j} (relative to the row's
//                running maximum) kept beside the softmax state; the epilogue
//                adds Λ_t (s q_t)ᵀ H̄ to the numerator (PISA's hybrid order);
//   linear_mix:  O_s from the exact part; O_l = relu(q)ᵀ(H_tot − A_i) /
//                (relu(q)·(z_tot − ζ_i) + eps) with A_i = Σ_{j∈S_i} relu(K_j)ᵀV_j
//                accumulated here from the tiles already in shared memory
//                (SPLA §2.2 subtraction form); O = α⊙O_s + (1−α)⊙O_l (SLA2 §2A).
// Within a warp, logits use lane = key (one full dot product per lane) and the
// accumulators use lane = channel, the probabilities broadcast by shuffles.
#include "attn_simt.cuh"

namespace sa {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtWarps = kSimtThreads / 32;
constexpr int QROWS = 64;                       // query rows per CTA
constexpr int RPW = QROWS / kSimtWarps;         // rows per warp
constexpr int KT = 32;                          // keys per shared-memory tile

template <typename T, int D, int BLK>
__global__ void __launch_bounds__(kSimtThreads)
attn_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                 int H, int N, const int32_t* __restrict__ block_idx, int topk, int tail,
                 const float* __restrict__ alpha, sa_block_stats st, float scale,
                 T* __restrict__ O) {
  constexpr int PER = D / 32;       // channels per lane
  constexpr int KS = D + 1;         // padded key row: lane t reads row t conflict-free
  constexpr int HALVES = BLK / QROWS;
  const int i = blockIdx.x / HALVES, half = blockIdx.x % HALVES;
  const int h = blockIdx.y, b = blockIdx.z;
  const int nb = N / BLK;
  const size_t bh = (size_t)b * H + h;
  const size_t head_off = bh * (size_t)N * D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool linear = tail == SA_TAIL_LINEAR_MIX;
  const bool fo = tail == SA_TAIL_FIRST_ORDER;
  const int nwords = (nb + 31) / 32;
  const size_t row0 = (size_t)i * BLK + (size_t)half * QROWS;   // first query row

  extern __shared__ float sm[];
  float* qs = sm;                                   // QROWS * D
  float* acc = qs + QROWS * D;                      // QROWS * D
  float* mrow = acc + QROWS * D;                    // QROWS
  float* lrow = mrow + QROWS;                       // QROWS
  float* lcrow = lrow + QROWS;                      // QROWS: Λ_t · BLK (first-order)
  float* ks = lcrow + QROWS;                        // KT * KS
  float* vs = ks + KT * KS;                         // KT * D
  float* zeta = vs + KT * D;                        // D
  uint32_t* selmask = reinterpret_cast<uint32_t*>(zeta + D);           // nwords
  float* A = reinterpret_cast<float*>(selmask + ((nwords + 3) & ~3));  // D * D (linear)

  const int32_t* sel = block_idx + (bh * nb + i) * (size_t)topk;
  for (int idx = tid; idx < QROWS * D; idx += kSimtThreads) {
    qs[idx] = to_f<T>(Q[head_off + row0 * D + idx]);
    acc[idx] = 0.f;
  }
  for (int r = tid; r < QROWS; r += kSimtThreads) {
    mrow[r] = -INFINITY;
    lrow[r] = 0.f;
    lcrow[r] = 0.f;
  }
  for (int w = tid; w < nwords; w += kSimtThreads) selmask[w] = 0u;
  if (linear)
    for (int idx = tid; idx < D * D; idx += kSimtThreads) A[idx] = 0.f;
  __syncthreads();
  for (int s = tid; s < topk; s += kSimtThreads) {
    const int j = sel[s];
    atomicOr(&selmask[j >> 5], 1u << (j & 31));
  }
  if (linear) {
    for (int c = tid; c < D; c += kSimtThreads) {
      float z = 0.f;
      for (int s = 0; s < topk; ++s) z += st.zrelu[(bh * nb + sel[s]) * D + c];
      zeta[c] = z;
    }
  }
  __syncthreads();

  const float scale2 = scale * kLog2e;

  // online-softmax update of this warp's rows with the KT keys in ks/vs;
  // bias2 is added to every logit (log2 domain); key `lane` counts if `valid`;
  // `pseudo` tiles also add their weights to lcrow
  auto consume_tile = [&](float bias2, bool valid, bool pseudo) {
    for (int rr = 0; rr < RPW; ++rr) {
      const int r = warp * RPW + rr;
      float x = 0.f;
      const float* qr = qs + r * D;
      const float* kr = ks + lane * KS;
#pragma unroll 8
      for (int c = 0; c < D; ++c) x = fmaf(qr[c], kr[c], x);
      x = valid ? fmaf(x, scale2, bias2) : -INFINITY;
      const float tmax = warp_max(x);
      if (tmax == -INFINITY) continue;
      const float m_old = mrow[r];
      const float m_new = fmaxf(m_old, tmax);
      const float corr = fast_exp2(m_old - m_new);
      const float p = fast_exp2(x - m_new);
      const float psum = warp_sum(p);
      float a[PER];
#pragma unroll
      for (int c = 0; c < PER; ++c) a[c] = acc[r * D + lane * PER + c] * corr;
#pragma unroll 4
      for (int t = 0; t < KT; ++t) {
        const float pt = __shfl_sync(0xffffffffu, p, t);
#pragma unroll
        for (int c = 0; c < PER; ++c) a[c] = fmaf(pt, vs[t * D + lane * PER + c], a[c]);
      }
#pragma unroll
      for (int c = 0; c < PER; ++c) acc[r * D + lane * PER + c] = a[c];
      __syncwarp();
      if (lane == 0) {
        mrow[r] = m_new;
        lrow[r] = lrow[r] * corr + psum;
        lcrow[r] = lcrow[r] * corr + (pseudo ? psum : 0.f);
      }
      __syncwarp();
    }
  };

  // ---- exact part over the selected blocks
  for (int s = 0; s < topk; ++s) {
    const int j = sel[s];
    for (int n0 = 0; n0 < BLK; n0 += KT) {
      __syncthreads();
      for (int idx = tid; idx < KT * D; idx += kSimtThreads) {
        const int n = idx / D, c = idx % D;
        const size_t g = head_off + ((size_t)j * BLK + n0 + n) * D + c;
        ks[n * KS + c] = to_f<T>(K[g]);
        vs[idx] = to_f<T>(V[g]);
      }
      __syncthreads();
      consume_tile(0.f, true, false);
      if (linear) {
        // A[c][e] += Σ_n relu(k_n[c]) v_n[e]; thread -> (c, 8-column chunks)
        for (int item = tid; item < D * (D / 8); item += kSimtThreads) {
          const int c = item / (D / 8), e0 = (item % (D / 8)) * 8;
          float a[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) a[u] = A[c * D + e0 + u];
          for (int n = 0; n < KT; ++n) {
            const float rk = fmaxf(ks[n * KS + c], 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) a[u] = fmaf(rk, vs[n * D + e0 + u], a[u]);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) A[c * D + e0 + u] = a[u];
        }
      }
    }
  }

  // ---- zero-order tail: unselected blocks as pseudo-keys
  if (tail == SA_TAIL_ZERO_ORDER || fo) {
    const float bias2 = log2f((float)BLK);
    const float inv_blk = 1.0f / BLK;
    for (int j0 = 0; j0 < nb; j0 += KT) {
      __syncthreads();
      for (int idx = tid; idx < KT * D; idx += kSimtThreads) {
        const int n = idx / D, c = idx % D;
        const int j = j0 + n;
        float kk = 0.f, vv = 0.f;
        if (j < nb) {
          kk = st.kmean[(bh * nb + j) * D + c];
          vv = st.vsum[(bh * nb + j) * D + c] * inv_blk;
        }
        ks[n * KS + c] = kk;
        vs[idx] = vv;
      }
      __syncthreads();
      const int j = j0 + lane;
      const bool valid = j < nb && !((selmask[j >> 5] >> (j & 31)) & 1u);
      consume_tile(bias2, valid, true);
    }
  }
  __syncthreads();

  // ---- epilogue: one warp per row, lane = channels
  for (int rr = 0; rr < RPW; ++rr) {
    const int r = warp * RPW + rr;
    const float l = lrow[r];
    const float inv_l = l > 0.f ? 1.0f / l : 0.f;
    T* orow = O + head_off + (row0 + r) * D;
    if (fo) {
      // + Λ_t (s q_t)ᵀ H̄, Λ_t = lcrow / BLK on the same running maximum as acc
      const float* qr = qs + r * D;
      const float* Hb = st.hbar + bh * (size_t)D * D;
      float num[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) num[e] = 0.f;
      for (int c = 0; c < D; ++c) {
        const float qc = qr[c];
#pragma unroll
        for (int e = 0; e < PER; ++e) num[e] = fmaf(qc, Hb[(size_t)c * D + lane * PER + e], num[e]);
      }
      const float w = scale * lcrow[r] * (1.0f / BLK);
#pragma unroll
      for (int e = 0; e < PER; ++e)
        orow[lane * PER + e] = from_f<T>(fmaf(w, num[e], acc[r * D + lane * PER + e]) * inv_l);
      continue;
    }
    if (!linear) {
#pragma unroll
      for (int c = 0; c < PER; ++c) orow[lane * PER + c] = from_f<T>(acc[r * D + lane * PER + c] * inv_l);
      continue;
    }
    // linear branch over the unselected blocks, then the SLA2 mixture; with
    // every block selected the unselected set is empty and O_l is 0 (the
    // subtraction H_tot - A_i would only leave rounding noise)
    const float* al = alpha + (size_t)h * D;
    if (topk == nb) {
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int ee = lane * PER + e;
        orow[ee] = from_f<T>(al[ee] * acc[r * D + ee] * inv_l);
      }
      continue;
    }
    const float* qr = qs + r * D;
    const float* zt = st.ztot + bh * D;
    float dp = 0.f;
#pragma unroll
    for (int c = 0; c < PER; ++c) {
      const int cc = lane * PER + c;
      dp = fmaf(fmaxf(qr[cc], 0.f), zt[cc] - zeta[cc], dp);
    }
    const float den = warp_sum(dp) + kLinearEps;
    const float* Ht = st.htot + bh * (size_t)D * D;
    float num[PER];
#pragma unroll
    for (int c = 0; c < PER; ++c) num[c] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float fq = fmaxf(qr[c], 0.f);
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int ee = lane * PER + e;
        num[e] = fmaf(fq, Ht[(size_t)c * D + ee] - A[c * D + ee], num[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int ee = lane * PER + e;
      const float a = al[ee];
      orow[ee] = from_f<T>(a * acc[r * D + ee] * inv_l + (1.0f - a) * num[e] / den);
    }
  }
}

template <typename T, int D, int BLK>
sa_status launch_simt(const void* Q, const void* K, const void* V, const sa_shape& s,
                      const int32_t* block_idx, int topk, sa_tail_mode tail, const float* alpha,
                      const sa_block_stats& st, float scale, void* O, cudaStream_t stream) {
  const int nb = s.N / BLK;
  const int nwords = (nb + 31) / 32;
  size_t smem = sizeof(float) * (2 * (size_t)QROWS * D + 3 * QROWS + (size_t)KT * (D + 1) +
                                 (size_t)KT * D + D) +
                sizeof(uint32_t) * ((nwords + 3) & ~3);
  if (tail == SA_TAIL_LINEAR_MIX) smem += sizeof(float) * (size_t)D * D;
  auto kern = attn_simt_kernel<T, D, BLK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(attn_simt_kernel)");
  dim3 grid(nb * (BLK / QROWS), s.H, s.B);
  kern<<<grid, kSimtThreads, smem, stream>>>(
      static_cast<const T*>(Q), static_cast<const T*>(K), static_cast<const T*>(V), s.H, s.N,
      block_idx, topk, (int)tail, alpha, st, scale, static_cast<T*>(O));
  return launch_status("attn_simt_kernel");
}

template <typename T>
sa_status dispatch_simt(const void* Q, const void* K, const void* V, const sa_shape& s,
                        const int32_t* block_idx, int topk, sa_tail_mode tail, const float* alpha,
                        const sa_block_stats& st, float scale, void* O, cudaStream_t stream) {
#define SA_SIMT_CASE(DD, BB)                                                                   \
  if (s.d == DD && s.block == BB)                                                              \
    return launch_simt<T, DD, BB>(Q, K, V, s, block_idx, topk, tail, alpha, st, scale, O, stream);
  SA_SIMT_CASE(128, 128)
  SA_SIMT_CASE(128, 64)
  SA_SIMT_CASE(64, 128)
  SA_SIMT_CASE(64, 64)
#undef SA_SIMT_CASE
  return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd: d and block must be 64 or 128");
}

}  // namespace

sa_status attn_simt(const void* Q, const void* K, const void* V, sa_dtype dtype, const sa_shape& s,
                    const int32_t* block_idx, int topk, sa_tail_mode tail, const float* alpha,
                    const sa_block_stats& st, float scale, void* O, cudaStream_t stream) {
  if (dtype == SA_FP32)
    return dispatch_simt<float>(Q, K, V, s, block_idx, topk, tail, alpha, st, scale, O, stream);
  return dispatch_simt<__nv_bfloat16>(Q, K, V, s, block_idx, topk, tail, alpha, st, scale, O, stream);
}

}  // namespace sa
