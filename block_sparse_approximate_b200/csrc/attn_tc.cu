// Sparse prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 Q/K/V, 128-token blocks, d = 128, tails drop and zero-order.
//
// PISA's fused kernel ("Implementação de Hardware") interleaves the exact
// scan over the selected blocks and the approximate scan over the block
// aggregates inside one online softmax.  Here both scans are the same tile
// loop: a CTA owns one 128-row query block and walks a list of 128-key tiles,
//   tiles 0..k-1      the selected KV blocks (exact, PISA "Fase 1"),
//   tiles k..k+c-1    the block centroids k̄_j with values vsum_j / B in
//                     groups of 128 blocks (PISA "Fase 2"): logit bias log2 B
//                     and the selected blocks masked out, which adds
//                     e^{s q·k̄_j}·vsum_j to the numerator and B·e^{s q·k̄_j}
//                     to the denominator,
// so the tail costs 1/B of the dense work and no N×N matrix exists.
//
// Warp roles (384 threads, one CTA per SM; the producer warpgroup gives its
// registers to the softmax warpgroups with setmaxnreg):
//   warps 0-3, 4-7  two softmax warpgroups ("streams"): stream s takes the
//              tiles t with t % 2 == s, so the two halves of the tile list are
//              reduced concurrently and merged at the end (the same merge as
//              split-KV decoding).  Thread r of a group owns query row r (TMEM
//              lane r): it reads its S row from TMEM, keeps (max, sum) in
//              registers, writes P back into TMEM as bf16 over the S columns,
//              and rescales its O row in TMEM only when the running max grows
//              by more than 2^8;
//   warp 8     TMA producer: Q once, then K/V tiles into a 3-stage ring;
//   warps 10-11 idle (they complete the producer warpgroup);
//   warp 9     MMA issuer: S = Q·Kᵀ (both operands K-major in shared memory)
//              into the stream's S, and O_s += P·V with P read from TMEM and V
//              as an MN-major shared-memory operand, alternating the streams
//              so one group's softmax overlaps the other group's MMAs.
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
#include <mutex>

#include "attn_simt.cuh"
#include "tc_util.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int TB = 128;                        // rows per tile (queries and keys)
constexpr int TD = 128;                        // head dim
constexpr int NS = 3;                          // K/V pipeline stages
constexpr int kTcThreads = 384;
constexpr int kTmaWarp = 8, kMmaWarp = 9;
// register split: 256 softmax threads x 216 + 128 producer threads x 40 =
// 60416 <= 384 x (launch registers); build.py checks ptxas reports >= 158
constexpr int kSoftmaxRegs = 216, kProducerRegs = 40;
constexpr uint32_t kHalfTile = TB * 64 * 2;    // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr uint32_t kTile = 2 * kHalfTile;      // 128 x 128 bf16
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kLazyRescale = 8.0f;           // log2 units

// barrier slots
constexpr int B_Q = 0;
constexpr int B_KF = 1;                 // NS
constexpr int B_VF = B_KF + NS;         // NS
constexpr int B_KE = B_VF + NS;         // NS
constexpr int B_SF = B_KE + NS;         // 2 (per stream)
constexpr int B_PR = B_SF + 2;          // 2 (per stream)
constexpr int B_OD = B_PR + 2;          // 2 (per stream)
constexpr int B_FIN = B_OD + 2;         // 1
constexpr int NBAR = B_FIN + 1;

constexpr uint32_t kBarOff = kTile * (1 + 2 * NS);
constexpr uint32_t kSlotOff = kBarOff + 8 * NBAR;     // tmem base, abort flag
constexpr uint32_t kMaskOff = kSlotOff + 16;

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) {
  // used only on the abort path, where no other role can release us
  const long long t0 = clock64();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if (clock64() - t0 > kWaitCycles / 8) return false;
  }
}

__device__ __forceinline__ void named_bar_softmax() {
  // barrier 1 over the two softmax warpgroups (256 threads)
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

template <bool ZO>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
               const __grid_constant__ CUtensorMap tmVb, const int32_t* __restrict__ block_idx, int nb,
               int topk, float scale2, __nv_bfloat16* __restrict__ O, int N) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int i = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSlotOff + 4);
  uint32_t* selmask = reinterpret_cast<uint32_t*>(smem + kMaskOff);
  auto bar = [&](int k) { return sb + kBarOff + 8u * k; };

  const int nwords = (nb + 31) >> 5;
  const int ntail = (ZO && topk < nb) ? (nb + TB - 1) / TB : 0;
  const int T = topk + ntail;
  const int32_t* sel = block_idx + ((size_t)bh * nb + i) * topk;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(B_KF + s), 1);
      mbar_init(bar(B_VF + s), 1);
      mbar_init(bar(B_KE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_SF + s), 1);
      mbar_init(bar(B_PR + s), 128);
      mbar_init(bar(B_OD + s), 1);
    }
    mbar_init(bar(B_FIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // selection bitmap, padded with 4 zero words so a tile's 4 words never run past it
  for (int w = threadIdx.x; w < nwords + 4; w += kTcThreads) selmask[w] = 0u;
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  __syncthreads();
  for (int s = threadIdx.x; s < topk; s += kTcThreads) {
    const int j = sel[s];
    atomicOr(&selmask[j >> 5], 1u << (j & 31));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    regs_dec<kProducerRegs>();
    if (lane == 0 && T > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (ZO) {
        prefetch_tmap(&tmKb);
        prefetch_tmap(&tmVb);
      }
      mbar_expect_tx(bar(B_Q), kTile);
      tma_load_3d(sb, &tmQ, 0, i * TB, bh, bar(B_Q));
      tma_load_3d(sb + kHalfTile, &tmQ, 64, i * TB, bh, bar(B_Q));
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % NS;
        if (t >= NS && !mbar_wait(bar(B_KE + s), ((t / NS) - 1) & 1, abort_flag)) break;
        const bool exact = t < topk;
        const CUtensorMap* mk = exact ? &tmK : &tmKb;
        const CUtensorMap* mv = exact ? &tmV : &tmVb;
        const int row = exact ? sel[t] * TB : (t - topk) * TB;
        const uint32_t ka = sb + kTile * (1 + 2 * s), va = ka + kTile;
        mbar_expect_tx(bar(B_KF + s), kTile);
        tma_load_3d(ka, mk, 0, row, bh, bar(B_KF + s));
        tma_load_3d(ka + kHalfTile, mk, 64, row, bh, bar(B_KF + s));
        mbar_expect_tx(bar(B_VF + s), kTile);
        tma_load_3d(va, mv, 0, row, bh, bar(B_VF + s));
        tma_load_3d(va + kHalfTile, mv, 64, row, bh, bar(B_VF + s));
        issued = t + 1;
      }
      if (*abort_flag) {
        // let the loads already in flight land before the CTA goes away
        wait_bounded(bar(B_Q), 0);
        for (int t = issued > NS ? issued - NS : 0; t < issued; ++t) {
          wait_bounded(bar(B_KF + t % NS), (t / NS) & 1);
          wait_bounded(bar(B_VF + t % NS), (t / NS) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kProducerRegs>();
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(TB, TB, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(TB, TD, 0, 1);
      // S(t) = Q K_tᵀ into the S columns of stream t % 2
      auto issue_s = [&](int t) -> bool {
        const int s = t % NS;
        if (!mbar_wait(bar(B_KF + s), (t / NS) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t ka = sb + kTile * (1 + 2 * s);
        const uint32_t d = tbase + (uint32_t)(t & 1) * TB;
#pragma unroll
        for (int k = 0; k < TD / 16; ++k) {
          const uint32_t koff = (k >> 2) * kHalfTile + (k & 3) * 32;
          mma_ss(d, desc_sw128(sb + koff, 16, 1024), desc_sw128(ka + koff, 16, 1024), idS, k > 0);
        }
        mma_commit(bar(B_SF + (t & 1)));
        return true;
      };
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
      if (ok) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t & 1, u = t >> 1, su = t % NS;
        if (!mbar_wait(bar(B_PR + st), u & 1, abort_flag)) break;
        if (!mbar_wait(bar(B_VF + su), (t / NS) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t va = sb + kTile * (2 + 2 * su);
        const uint32_t pa = tbase + (uint32_t)st * TB;
        const uint32_t od = tbase + kColO + (uint32_t)st * TD;
#pragma unroll
        for (int k = 0; k < TB / 16; ++k)
          mma_ts(od, pa + k * 8, desc_sw128(va + k * 16 * 128, kHalfTile, 1024), idO, (u > 0 || k > 0));
        mma_commit(bar(B_KE + su));
        mma_commit(bar(B_OD + st));
        if (t + 2 < T && !issue_s(t + 2)) break;
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(bar(B_FIN));
      wait_bounded(bar(B_FIN), 0);
    }
  } else if (warp >= 8) {
    regs_dec<kProducerRegs>();                  // idle warps of the producer warpgroup
  } else {
    // ------------------------------------------------------------ softmax
    regs_inc<kSoftmaxRegs>();
    const int st = warp >> 2;                   // stream
    const int wq = warp & 3;                    // TMEM lane quarter
    const int r = wq * 32 + lane;               // query row
    const uint32_t lrow = tbase + ((uint32_t)(wq * 32) << 16);
    const uint32_t s_col = (uint32_t)st * TB;
    const uint32_t o_col = kColO + (uint32_t)st * TD;
    const int U = T > st ? (T - st + 1) / 2 : 0;   // tiles of this stream
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int u = 0; u < U; ++u) {
      const int t = 2 * u + st;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_SF + st), u & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lrow + s_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
      tmem_wait_ld();
      const bool centroid = t >= topk;
      float bias = 0.f;
      if (centroid) {
        // validity of the 128 pseudo-keys: inside the head and not selected
        const int jb = (t - topk) * TB;
        bias = 7.0f;   // log2 of the block size 128
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int w0 = (jb >> 5) + c;
          const int lim = nb - (jb + 32 * c);
          const uint32_t range = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : ((1u << lim) - 1u));
          const uint32_t valid = ~selmask[w0] & range;
#pragma unroll
          for (int n = 0; n < 32; ++n)
            if (!((valid >> n) & 1u)) v[32 * c + n] = __float_as_uint(-INFINITY);
        }
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
      for (int n = 0; n < TB / 2; ++n)
        mx8[n & 7] = fmax3(mx8[n & 7], __uint_as_float(v[2 * n]), __uint_as_float(v[2 * n + 1]));
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                             fmaxf(mx8[6], mx8[7]));
      const float m_tile = mx == -INFINITY ? -INFINITY : fmaf(mx, scale2, bias);
      const float m_new = fmaxf(m_used, m_tile);
      const bool need = m_new > m_used + kLazyRescale;
      float factor = 1.f;
      if (need) {
        factor = fast_exp2(m_used - m_new);
        m_used = m_new;
      }
      const bool live = m_used != -INFINITY;
      const float neg = bias - m_used;
      float sm8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) sm8[k] = 0.f;
      const float sc2 = live ? scale2 : 0.f, ng = live ? neg : -INFINITY;   // dead row: p = 0
#pragma unroll
      for (int n = 0; n < TB / 2; ++n) {
        float a0, a1;
        ffma2(a0, a1, __uint_as_float(v[2 * n]), __uint_as_float(v[2 * n + 1]), sc2, sc2, ng, ng);
        const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
        fadd2(sm8[2 * (n & 3)], sm8[2 * (n & 3) + 1], p0, p1);
        v[n] = pack_bf16(p0, p1);
      }
      const float sum = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
      l = l * factor + sum;
      tmem_st32(lrow + s_col, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_st32(lrow + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_st();
      if (u >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B_OD + st), (u - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (__any_sync(0xffffffffu, need)) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lrow + o_col + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(lrow + o_col + 32 * c, o);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_PR + st));
    }
    if (ok && U > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OD + st), (U - 1) & 1, abort_flag));
    // both groups past their last PV: every MMA that reads Q has completed,
    // so the Q tile's shared memory can carry the (max, sum) exchange
    named_bar_softmax();
    float* ex = reinterpret_cast<float*>(smem);   // [2 streams][2][128]
    ex[st * 256 + r] = (U > 0) ? m_used : -INFINITY;
    ex[st * 256 + 128 + r] = l;
    named_bar_softmax();
    const float m0 = ex[r], l0 = ex[128 + r], m1 = ex[256 + r], l1 = ex[384 + r];
    const int U0 = T > 0 ? (T + 1) / 2 : 0, U1 = T > 1 ? T / 2 : 0;
    const float M = fmaxf(m0, m1);
    const float f0 = (U0 > 0 && m0 != -INFINITY) ? fast_exp2(m0 - M) : 0.f;
    const float f1 = (U1 > 0 && m1 != -INFINITY) ? fast_exp2(m1 - M) : 0.f;
    const float L = l0 * f0 + l1 * f1;
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    if (ok) {
      tc_fence_after();
      // stream st writes output columns [64 st, 64 st + 64) of its rows
      uint4* orow = reinterpret_cast<uint4*>(O + ((size_t)bh * N + (size_t)i * TB + r) * TD + 64 * st);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t a[32], b[32];
        if (U0 > 0) {
          tmem_ld32(lrow + kColO + 64 * st + 32 * c, a);
        }
        if (U1 > 0) {
          tmem_ld32(lrow + kColO + TD + 64 * st + 32 * c, b);
        }
        tmem_wait_ld();
        if (U0 == 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = 0u;
        }
        if (U1 == 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) b[e] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            y[e] = (__uint_as_float(a[8 * q + e]) * f0 + __uint_as_float(b[8 * q + e]) * f1) * inv;
          uint4 w;
          w.x = pack_bf16(y[0], y[1]);
          w.y = pack_bf16(y[2], y[3]);
          w.z = pack_bf16(y[4], y[5]);
          w.w = pack_bf16(y[6], y[7]);
          orow[4 * c + q] = w;
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

size_t tc_smem_bytes(int nb) {
  return 1024 + kMaskOff + 4 * (size_t)((nb + 31) / 32 + 4);
}

}  // namespace

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                       uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool attn_tc_supports(sa_dtype dtype, const sa_shape& s, sa_tail_mode tail) {
  return dtype == SA_BF16 && s.block == TB && s.d == TD &&
         (tail == SA_TAIL_DROP || tail == SA_TAIL_ZERO_ORDER);
}

sa_status attn_tc(const void* Q, const void* K, const void* V, const sa_shape& s, const int32_t* block_idx,
                  int topk, sa_tail_mode tail, const float* alpha, const sa_block_stats& st, float scale,
                  void* O, cudaStream_t stream) {
  (void)alpha;
  const int nb = s.N / TB;
  const uint64_t BH = (uint64_t)s.B * s.H;
  CUtensorMap mq, mk, mv, mkb, mvb;
  if (!make_tmap_bf16_3d(&mq, Q, TD, s.N, BH, 64, TB) || !make_tmap_bf16_3d(&mk, K, TD, s.N, BH, 64, TB) ||
      !make_tmap_bf16_3d(&mv, V, TD, s.N, BH, 64, TB))
    return fail(SA_ERR_CUDA, "sa_sparse_attn_fwd: cuTensorMapEncodeTiled failed for Q/K/V");
  const bool zo = tail == SA_TAIL_ZERO_ORDER;
  if (zo) {
    if (!make_tmap_bf16_3d(&mkb, st.kmean_bf16, TD, nb, BH, 64, TB) ||
        !make_tmap_bf16_3d(&mvb, st.vmean_bf16, TD, nb, BH, 64, TB))
      return fail(SA_ERR_CUDA, "sa_sparse_attn_fwd: cuTensorMapEncodeTiled failed for the block centroids");
  } else {
    mkb = mk;
    mvb = mv;
  }
  const size_t smem = tc_smem_bytes(nb);
  auto kern = zo ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(attn_tc_kernel)");
  dim3 grid(nb, (unsigned)BH);
  kern<<<grid, kTcThreads, smem, stream>>>(mq, mk, mv, mkb, mvb, block_idx, nb, topk, scale * kLog2e,
                                           static_cast<__nv_bfloat16*>(O), s.N);
  return launch_status("attn_tc_kernel");
}

}  // namespace sa

extern "C" sa_status sa_device_error(uint32_t* code) {
  using namespace sa;
  if (!code) return fail(SA_ERR_INVALID_ARG, "sa_device_error: code is required");
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, tc::g_device_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return launch_status("sa_device_error");
  *code = v;
  return SA_OK;
}
