// GQA decode with block routing and the zero-order tail.
//
// SPLA §2 notes that decoding is bound by loading the KV cache and keeps the
// IO profile of sparse decoding: only the selected blocks are read token by
// token; every other block is represented by its precomputed statistics.
// Steps (all on the caller's stream):
//   1. decode_score_kernel  the SPLA §2.1 block score (log form) of every KV
//                           block for each query head, summed over the GQA group
//                           (logsumexp) -> scores[b, g, j]
//   2. decode_topk_kernel   top-k per (sequence, KV head) -> block_idx
//   3. decode_attn_kernel   split over the KV axis: exact online softmax over
//                           this split's share of the selected blocks plus the
//                           PISA zero-order pseudo-keys of this split's share of
//                           the unselected blocks -> partial (max, sum, acc)
//   4. decode_combine_kernel  merges the partial states -> o
#include <mutex>

#include "topk.cuh"

namespace sa {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kMaxGroup = 8;
constexpr int kScoreChunk = 64;   // KV blocks per CTA of the score kernel
constexpr int kTok = 32;          // tokens (or centroids) per warp step

struct DecodeLayout {
  size_t scores_off, idx_off, part_off, total;
  int nsplit;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int decode_splits(const sa_decode_shape& s, int topk) {
  const int nb = s.N / s.block;
  const long chunks = (long)topk * (s.block / kTok) + (nb + kTok - 1) / kTok;
  long ns = (chunks + kDecWarps - 1) / kDecWarps;
  if (ns < 1) ns = 1;
  if (ns > 64) ns = 64;
  return (int)ns;
}

DecodeLayout decode_layout(const sa_decode_shape& s, int topk) {
  DecodeLayout L;
  const int nb = s.N / s.block;
  L.nsplit = decode_splits(s, topk);
  L.scores_off = 0;
  L.idx_off = align256((size_t)s.B * s.Hkv * nb * sizeof(float));
  L.part_off = L.idx_off + align256((size_t)s.B * s.Hkv * (topk > 0 ? topk : 1) * sizeof(int32_t));
  L.total = L.part_off + align256((size_t)s.B * s.Hq * L.nsplit * (s.d + 2) * sizeof(float));
  return L;
}

// ---- 1. scores -----------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_score_kernel(const __nv_bfloat16* __restrict__ q, sa_block_stats st, int Hq, int Hkv,
                    int nb, float scale, float* __restrict__ scores) {
  constexpr int PER = D / 32;
  const int chunk = blockIdx.x, kh = blockIdx.y, b = blockIdx.z;
  const int g = Hq / Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ float qs[kMaxGroup][D];
  __shared__ float ws[kMaxGroup][D];
  for (int idx = threadIdx.x; idx < g * D; idx += kDecThreads) {
    const int hh = idx / D, c = idx % D;
    const float x = __bfloat162float(q[((size_t)b * Hq + kh * g + hh) * D + c]);
    qs[hh][c] = scale * x;
    ws[hh][c] = 0.5f * scale * scale * x * x;
  }
  __syncthreads();
  const size_t base = ((size_t)b * Hkv + kh) * nb;
  const int j_end = min(nb, (chunk + 1) * kScoreChunk);
  for (int j = chunk * kScoreChunk + warp; j < j_end; j += kDecWarps) {
    float km[PER], kv[PER];
#pragma unroll
    for (int p = 0; p < PER; ++p) {
      km[p] = st.kmean[(base + j) * D + lane * PER + p];
      kv[p] = st.kvar[(base + j) * D + lane * PER + p];
    }
    float L[kMaxGroup];
    float mx = -INFINITY;
#pragma unroll
    for (int hh = 0; hh < kMaxGroup; ++hh) {
      if (hh < g) {
        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int p = 0; p < PER; ++p) {
          s1 = fmaf(qs[hh][lane * PER + p], km[p], s1);
          s2 = fmaf(ws[hh][lane * PER + p], kv[p], s2);
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        L[hh] = s1 + log1pf(s2);
        mx = fmaxf(mx, L[hh]);
      }
    }
    float sum = 0.f;
#pragma unroll
    for (int hh = 0; hh < kMaxGroup; ++hh)
      if (hh < g) sum += expf(L[hh] - mx);
    if (lane == 0) scores[base + j] = mx + logf(sum);
  }
}

// ---- 2. top-k ------------------------------------------------------------
__global__ void __launch_bounds__(kDecThreads)
decode_topk_kernel(const float* __restrict__ scores, int Hkv, int nb, int topk,
                   int32_t* __restrict__ idx) {
  const int kh = blockIdx.x, b = blockIdx.y;
  extern __shared__ unsigned long long smem_u64[];
  int n2 = 1;
  while (n2 < nb) n2 <<= 1;
  float* sc = reinterpret_cast<float*>(smem_u64 + n2);
  const size_t base = ((size_t)b * Hkv + kh);
  for (int j = threadIdx.x; j < nb; j += kDecThreads) sc[j] = scores[base * nb + j];
  __syncthreads();
  block_topk_ascending(sc, nb, topk, smem_u64, idx + base * topk);
}

// ---- 3. split attention --------------------------------------------------
// Warp step over kTok keys: lane t computes the logits of key t for the g
// heads (lane = key); the accumulators are then updated with lane = channel,
// the probabilities broadcast by shuffles.
template <int D>
struct WarpState {
  float m[kMaxGroup], l[kMaxGroup], acc[kMaxGroup][D / 32];
};

template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ Kc,
                   const __nv_bfloat16* __restrict__ Vc, sa_block_stats st, int Hq, int Hkv, int N,
                   int blk, const int32_t* __restrict__ idx, int topk, int tail, float scale,
                   int nsplit, float* __restrict__ partial) {
  constexpr int PER = D / 32;
  const int split = blockIdx.x, kh = blockIdx.y, b = blockIdx.z;
  const int g = Hq / Hkv;
  const int nb = N / blk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t kv_base = ((size_t)b * Hkv + kh) * (size_t)N * D;
  const size_t st_base = ((size_t)b * Hkv + kh) * (size_t)nb;
  const int32_t* sel = idx + ((size_t)b * Hkv + kh) * topk;

  extern __shared__ float dsm[];
  float* qs = dsm;                                             // kMaxGroup * D
  uint32_t* selmask = reinterpret_cast<uint32_t*>(qs + kMaxGroup * D);
  const int nwords = (nb + 31) / 32;
  float* red = reinterpret_cast<float*>(selmask + ((nwords + 3) & ~3));  // warps*g*(D+2)

  const float scale2 = scale * kLog2e;
  for (int i = threadIdx.x; i < g * D; i += kDecThreads) {
    const int hh = i / D, c = i % D;
    qs[hh * D + c] = scale2 * __bfloat162float(q[((size_t)b * Hq + kh * g + hh) * D + c]);
  }
  for (int w = threadIdx.x; w < nwords; w += kDecThreads) selmask[w] = 0u;
  __syncthreads();
  for (int s = threadIdx.x; s < topk; s += kDecThreads) {
    const int j = sel[s];
    atomicOr(&selmask[j >> 5], 1u << (j & 31));
  }
  __syncthreads();

  WarpState<D> S;
#pragma unroll
  for (int hh = 0; hh < kMaxGroup; ++hh) {
    S.m[hh] = -INFINITY;
    S.l[hh] = 0.f;
#pragma unroll
    for (int c = 0; c < PER; ++c) S.acc[hh][c] = 0.f;
  }

  // this split's share of the selected blocks and of the block range
  const int s0 = (int)(((long)topk * split) / nsplit), s1 = (int)(((long)topk * (split + 1)) / nsplit);
  const int j0 = (int)(((long)nb * split) / nsplit), j1 = (int)(((long)nb * (split + 1)) / nsplit);
  const int steps_per_block = blk / kTok;
  const int n_exact = (s1 - s0) * steps_per_block;
  const int n_tail = tail == SA_TAIL_ZERO_ORDER ? (j1 - j0 + kTok - 1) / kTok : 0;
  const float bias2 = log2f((float)blk);
  const float inv_blk = 1.0f / blk;

  for (int step = warp; step < n_exact + n_tail; step += kDecWarps) {
    const bool exact = step < n_exact;
    float lg[kMaxGroup];
    bool valid = true;
    int tok0 = 0, jbase = 0;
    if (exact) {
      const int j = sel[s0 + step / steps_per_block];
      tok0 = j * blk + (step % steps_per_block) * kTok;
      // lane = token: logits over the full key row
      const __nv_bfloat16* krow = Kc + kv_base + (size_t)(tok0 + lane) * D;
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh) lg[hh] = 0.f;
#pragma unroll 4
      for (int c8 = 0; c8 < D; c8 += 8) {
        float kx[8];
        load8<__nv_bfloat16>(krow + c8, kx);
#pragma unroll
        for (int hh = 0; hh < kMaxGroup; ++hh) {
          if (hh < g) {
#pragma unroll
            for (int e = 0; e < 8; ++e) lg[hh] = fmaf(qs[hh * D + c8 + e], kx[e], lg[hh]);
          }
        }
      }
    } else {
      jbase = j0 + (step - n_exact) * kTok;
      const int jj = jbase + lane;   // lane = centroid of an unselected block
      valid = jj < j1 && !((selmask[jj >> 5] >> (jj & 31)) & 1u);
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh) lg[hh] = bias2;
      if (jj < j1) {
        const float* kmr = st.kmean + (st_base + jj) * D;
#pragma unroll 4
        for (int c4 = 0; c4 < D; c4 += 4) {
          const float4 k4 = __ldg(reinterpret_cast<const float4*>(kmr + c4));
#pragma unroll
          for (int hh = 0; hh < kMaxGroup; ++hh) {
            if (hh < g) {
              lg[hh] = fmaf(qs[hh * D + c4 + 0], k4.x, lg[hh]);
              lg[hh] = fmaf(qs[hh * D + c4 + 1], k4.y, lg[hh]);
              lg[hh] = fmaf(qs[hh * D + c4 + 2], k4.z, lg[hh]);
              lg[hh] = fmaf(qs[hh * D + c4 + 3], k4.w, lg[hh]);
            }
          }
        }
      }
    }
    // online-softmax bookkeeping per head (lane-local probabilities)
    float p[kMaxGroup];
    bool any = false;
#pragma unroll
    for (int hh = 0; hh < kMaxGroup; ++hh) {
      p[hh] = 0.f;
      if (hh < g) {
        const float x = valid ? lg[hh] : -INFINITY;
        const float tmax = warp_max(x);
        if (tmax != -INFINITY) {
          any = true;
          const float m_new = fmaxf(S.m[hh], tmax);
          const float corr = fast_exp2(S.m[hh] - m_new);
          p[hh] = fast_exp2(x - m_new);
          S.l[hh] = S.l[hh] * corr + p[hh];   // lane-partial sum
#pragma unroll
          for (int c = 0; c < PER; ++c) S.acc[hh][c] *= corr;
          S.m[hh] = m_new;
        }
      }
    }
    if (!any) continue;
    // lane = channel: accumulate the kTok value rows
#pragma unroll 4
    for (int t = 0; t < kTok; ++t) {
      float v[PER];
      if (exact) {
        const __nv_bfloat16* vrow = Vc + kv_base + (size_t)(tok0 + t) * D + lane * PER;
        if constexpr (PER == 4) {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(vrow));
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
          const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
          v[0] = a.x; v[1] = a.y; v[2] = c.x; v[3] = c.y;
        } else {
          const unsigned u = __ldg(reinterpret_cast<const unsigned*>(vrow));
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
          v[0] = a.x; v[1] = a.y;
        }
      } else {
        const int jt = jbase + t;
        if (jt < j1) {
          const float* vr = st.vsum + (st_base + jt) * D + lane * PER;
#pragma unroll
          for (int c = 0; c < PER; ++c) v[c] = __ldg(vr + c) * inv_blk;
        } else {
#pragma unroll
          for (int c = 0; c < PER; ++c) v[c] = 0.f;
        }
      }
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh) {
        if (hh < g) {
          const float pt = __shfl_sync(0xffffffffu, p[hh], t);
#pragma unroll
          for (int c = 0; c < PER; ++c) S.acc[hh][c] = fmaf(pt, v[c], S.acc[hh][c]);
        }
      }
    }
  }

  // merge the warps' states, then write this split's partial state
  float* my = red + (size_t)warp * kMaxGroup * (D + 2);
#pragma unroll
  for (int hh = 0; hh < kMaxGroup; ++hh) {
    if (hh < g) {
      const float lsum = warp_sum(S.l[hh]);
      if (lane == 0) {
        my[hh * (D + 2) + 0] = S.m[hh];
        my[hh * (D + 2) + 1] = lsum;
      }
#pragma unroll
      for (int c = 0; c < PER; ++c) my[hh * (D + 2) + 2 + lane * PER + c] = S.acc[hh][c];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < g * D; i += kDecThreads) {
    const int hh = i / D, c = i % D;
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, red[(w * kMaxGroup + hh) * (D + 2)]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float* r = red + (w * kMaxGroup + hh) * (D + 2);
        if (r[0] == -INFINITY) continue;
        const float f = fast_exp2(r[0] - M);
        L = fmaf(r[1], f, L);
        A = fmaf(r[2 + c], f, A);
      }
    }
    float* out = partial + (((size_t)b * Hq + kh * g + hh) * nsplit + split) * (D + 2);
    if (c == 0) {
      out[0] = M;
      out[1] = L;
    }
    out[2 + c] = A;
  }
}

// ---- 4. combine ----------------------------------------------------------
template <int D>
__global__ void decode_combine_kernel(const float* __restrict__ partial, int Hq, int nsplit,
                                      __nv_bfloat16* __restrict__ O) {
  const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  const float* p = partial + ((size_t)b * Hq + h) * nsplit * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, p[s * (D + 2)]);
  float L = 0.f, A = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float* r = p + s * (D + 2);
      if (r[0] == -INFINITY) continue;
      const float f = fast_exp2(r[0] - M);
      L = fmaf(r[1], f, L);
      A = fmaf(r[2 + c], f, A);
    }
  }
  O[((size_t)b * Hq + h) * D + c] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
}

template <int D>
sa_status launch_decode(const void* q, const void* Kc, const void* Vc, const sa_decode_shape& s,
                        const sa_block_stats& st, int topk, float scale, sa_tail_mode tail,
                        int32_t* idx_out, float* scores_out, void* O, char* ws,
                        cudaStream_t stream) {
  const DecodeLayout L = decode_layout(s, topk);
  const int nb = s.N / s.block;
  float* scores = scores_out ? scores_out : reinterpret_cast<float*>(ws + L.scores_off);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + L.idx_off);
  float* part = reinterpret_cast<float*>(ws + L.part_off);
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);

  dim3 g1((nb + kScoreChunk - 1) / kScoreChunk, s.Hkv, s.B);
  decode_score_kernel<D><<<g1, kDecThreads, 0, stream>>>(qb, st, s.Hq, s.Hkv, nb, scale, scores);
  sa_status r = launch_status("decode_score_kernel");
  if (r != SA_OK) return r;

  int n2 = 1;
  while (n2 < nb) n2 <<= 1;
  const size_t smem2 = (size_t)n2 * 8 + (size_t)nb * 4;
  if (smem2 > 48 * 1024 &&
      cudaFuncSetAttribute(decode_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(decode_topk_kernel)");
  decode_topk_kernel<<<dim3(s.Hkv, s.B), kDecThreads, smem2, stream>>>(scores, s.Hkv, nb, topk, idx);
  r = launch_status("decode_topk_kernel");
  if (r != SA_OK) return r;

  const int nwords = (nb + 31) / 32;
  const size_t smem3 = sizeof(float) * kMaxGroup * D + sizeof(uint32_t) * ((nwords + 3) & ~3) +
                       sizeof(float) * kDecWarps * kMaxGroup * (D + 2);
  if (smem3 > 48 * 1024 &&
      cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(decode_attn_kernel)");
  decode_attn_kernel<D><<<dim3(L.nsplit, s.Hkv, s.B), kDecThreads, smem3, stream>>>(
      qb, static_cast<const __nv_bfloat16*>(Kc), static_cast<const __nv_bfloat16*>(Vc), st, s.Hq,
      s.Hkv, s.N, s.block, idx, topk, (int)tail, scale, L.nsplit, part);
  r = launch_status("decode_attn_kernel");
  if (r != SA_OK) return r;

  decode_combine_kernel<D><<<dim3(s.Hq, s.B), D, 0, stream>>>(part, s.Hq, L.nsplit,
                                                             static_cast<__nv_bfloat16*>(O));
  return launch_status("decode_combine_kernel");
}

sa_status check_decode_shape(const sa_decode_shape& s, int topk) {
  if (s.B < 0 || s.Hq <= 0 || s.Hkv <= 0 || s.N < 0)
    return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: negative or zero size");
  if (s.Hq % s.Hkv) return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: Hq must be a multiple of Hkv");
  if (s.Hq / s.Hkv > kMaxGroup) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: at most 8 query heads per KV head");
  if (s.d != 64 && s.d != 128) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: d must be 64 or 128");
  if (s.block != 64 && s.block != 128) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: block must be 64 or 128");
  if (s.N % s.block) return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: N must be a multiple of block");
  const int nb = s.N / s.block;
  if (nb > kMaxRouteBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: at most 4096 blocks per sequence");
  if (topk < 0 || topk > nb) return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: topk must be in [0, N/block]");
  return SA_OK;
}

}  // namespace
}  // namespace sa

extern "C" size_t sa_decode_workspace_size(sa_decode_shape shape, int32_t topk) {
  using namespace sa;
  if (check_decode_shape(shape, topk) != SA_OK) return 0;
  return decode_layout(shape, topk).total;
}

extern "C" sa_status sa_decode_fwd(const void* q, const void* Kcache, const void* Vcache,
                                   sa_dtype dtype, sa_decode_shape shape,
                                   const sa_block_stats* stats, int32_t topk, float scale,
                                   sa_tail_mode tail, int32_t* block_idx_out, float* scores_out,
                                   void* O, void* workspace, size_t workspace_bytes, void* stream) {
  using namespace sa;
  sa_status r = check_decode_shape(shape, topk);
  if (r != SA_OK) return r;
  if (dtype != SA_BF16) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: bf16 caches only");
  if (tail != SA_TAIL_ZERO_ORDER && tail != SA_TAIL_DROP)
    return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: tail must be SA_TAIL_DROP or SA_TAIL_ZERO_ORDER");
  if (!q || !Kcache || !Vcache || !O || !stats || !stats->kmean || !stats->kvar || !stats->vsum)
    return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: q, caches, O and stats (kmean, kvar, vsum) are required");
  const void* ptrs[] = {q, Kcache, Vcache, O, stats->kmean, stats->kvar, stats->vsum, block_idx_out, scores_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_decode_fwd: pointers must be 16-byte aligned");
  const size_t need = decode_layout(shape, topk).total;
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "sa_decode_fwd: workspace missing or smaller than sa_decode_workspace_size()");
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(SA_ERR_ALIGNMENT, "sa_decode_fwd: workspace must be 256-byte aligned");
  if (shape.B == 0 || shape.N == 0) return SA_OK;
  cudaStream_t s = as_stream(stream);
  char* ws = static_cast<char*>(workspace);
  if (shape.d == 128)
    return launch_decode<128>(q, Kcache, Vcache, shape, *stats, topk, scale, tail, block_idx_out,
                              scores_out, O, ws, s);
  return launch_decode<64>(q, Kcache, Vcache, shape, *stats, topk, scale, tail, block_idx_out,
                           scores_out, O, ws, s);
}

// ---- decode with library-owned scratch ---------------------------------------
// sa_decode_fwd_static runs the same kernels as sa_decode_fwd, with its
// scratch (route scores, selected indices, per-split partial states) in this
// file-scope device array instead of a caller workspace.  The array exists
// once per device that loads the library and stays allocated until the
// process exits.  Host code must not hand `g_decode_scratch` itself to a
// kernel (on the host it names a shadow variable, not device memory); the
// device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[SA_DECODE_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up on the
// first call per device, with that device current).
sa_status static_scratch(void** out) {
  using namespace sa;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return launch_status("sa_decode_fwd_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd_static: device index above 63");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(SA_ERR_CUDA, std::string("sa_decode_fwd_static: cudaGetSymbolAddress failed: ") +
                                   cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SA_OK;
}
}  // namespace

extern "C" sa_status sa_decode_fwd_static(const void* q, const void* Kcache, const void* Vcache,
                                          sa_dtype dtype, sa_decode_shape shape,
                                          const sa_block_stats* stats, int32_t topk, float scale,
                                          sa_tail_mode tail, int32_t* block_idx_out,
                                          float* scores_out, void* O, void* stream) {
  using namespace sa;
  const size_t need = sa_decode_workspace_size(shape, topk);
  if (need > SA_DECODE_STATIC_SCRATCH_BYTES)
    return fail(SA_ERR_WORKSPACE, "sa_decode_fwd_static: this problem needs " + std::to_string(need) +
                                      " bytes of scratch; the library's static scratch holds " +
                                      std::to_string((size_t)SA_DECODE_STATIC_SCRATCH_BYTES) +
                                      " bytes (use sa_decode_fwd with a workspace)");
  void* scratch = nullptr;
  sa_status r = static_scratch(&scratch);
  if (r != SA_OK) return r;
  // every scratch entry the kernels read is written earlier in the same call,
  // so the contents left by a previous call need no clearing
  return sa_decode_fwd(q, Kcache, Vcache, dtype, shape, stats, topk, scale, tail, block_idx_out,
                       scores_out, O, scratch, SA_DECODE_STATIC_SCRATCH_BYTES, stream);
}
