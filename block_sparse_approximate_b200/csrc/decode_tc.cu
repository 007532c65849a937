// Statistics pass of the GQA decode path on the 5th-generation tensor cores
// (bf16 block statistics, d = 128).
//
// SPLA §2.1 scores every KV block of a sequence for the query heads of its
// group, s q_h·k̄_j + log(1 + ½ s² Σ_c q_hc² Var_jc), and the zero-order tail
// (PISA §2) needs e^{s q_h·k̄_j} and its product with the block's value mean
// for every block.  Per (sequence, KV head) these are two small products of
// the 2048 blocks' statistics with the group's few query rows, so a tile of
// 128 blocks is the M = 128 side of tcgen05 MMAs and the group's heads the
// N = 16 side (zero rows past the group):
//   S1 = K̄ Qᵀ            q·k̄_j of every (block, head)
//   S2 = Var (W_hi + W_lo)ᵀ  with W = ½ s² q² split into two bf16 terms (q² of a
//                          bf16 q has 16 significant bits: the split is exact)
//   Oᵀ = V̄ᵀ Pᵀ            the tile's zero-order numerator per head, P in bf16
// with the accumulators in TMEM.  One thread per block (TMEM lane) forms the
// group score ln Σ_h e^{s q_h·k̄_j}(1 + S2_h) and, with the tile's maximum of
// each head's log2 weight, P = 2^{x − M}; a tile is one segment of the
// partial states that the combine merges (max, sum, numerator per head).
//
// Roles (384 threads, one CTA per SM): warp 0 loads the tiles by TMA, kmean
// and kvar into one ring of two stages (lane 0) and the value means into
// another (lane 1), so the first ring refills as soon as S1 and S2 have read
// it while the second waits for Oᵀ; warp 1 issues the MMAs, S of tile t + 1
// before Oᵀ of tile t; warps 4-7 and 8-11 are two epilogue groups taking
// alternate tiles (TMEM buffers and stages alternate with them).  Every wait
// is bounded; a wait that gives up sets the device error word and every role
// returns.
#include "attn_simt.cuh"
#include "tc_util.cuh"
#include "topk.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int kStTile = 128;                  // blocks per tile = one segment
constexpr int kStD = 128;                     // head dim
constexpr int kStN = 16;                      // MMA N: the group's heads, zero-padded
constexpr int kStThreads = 384;
constexpr int kStTmaWarp = 0, kStMmaWarp = 1, kStEpiWarp0 = 4;
constexpr uint32_t kStSpan = kStTile * 128;   // 128 rows of one 128-byte swizzle span: 16 KB
constexpr uint32_t kStArr = 2 * kStSpan;      // a 128 x 128 bf16 tile: 32 KB
constexpr uint32_t kStBop = 2 * kStN * 128;   // a 16 x 128 bf16 operand (two spans): 4 KB
constexpr uint32_t kStTmemCols = 128;         // two buffers of S1 (16), S2 (16), O (16 of 32)
constexpr int kStTopkBlocks = 2048;           // rows up to this many blocks take their top-k here

template <bool ZT>
struct StLayout {
  static constexpr uint32_t kKStage = 2 * kStArr;             // kmean and kvar of a tile
  static constexpr uint32_t kVRing = 2 * kKStage;             // the value means' ring (ZT)
  static constexpr uint32_t kBop = kVRing + (ZT ? 2 * kStArr : 0);   // Q, W_hi, W_lo
  static constexpr uint32_t kP = kBop + 3 * kStBop;           // P of the two buffers
  static constexpr uint32_t kRed = kP + 2 * kStBop;           // [2 groups][4 warps][16 heads][2]
  static constexpr uint32_t kBar = kRed + 2 * 4 * kStN * 2 * 4;
  enum { B_FK = 0, B_EK = 2, B_FV = 4, B_EV = 6, B_SC = 8, B_PR = 10, B_OC = 12, B_TF = 14, B_FIN = 16, NBAR = 17 };
  static constexpr uint32_t kSlot = kBar + 8 * NBAR;          // tmem base, abort flag
  static constexpr uint32_t kScores = kSlot + 16;             // the row's scores (fused top-k)
  static constexpr uint32_t kTopk = kScores + 4 * kStTopkBlocks;   // RadixTopkSmem
  static constexpr size_t bytes() { return 1024 + kTopk + sizeof(RadixTopkSmem); }
};

// Byte offset of element (row h, column c) of a 16 x 128 bf16 operand in the
// K-major 128-byte-swizzled layout: two spans of 64 columns, rows of 128
// bytes, 16-byte chunk index XOR (row mod 8).
__device__ __forceinline__ uint32_t bop_off(int h, int c) {
  return (uint32_t)((c >> 6) * (kStN * 128) + h * 128 + ((((c & 63) >> 3) ^ (h & 7)) << 4) + (c & 7) * 2);
}

__device__ __forceinline__ void st_mma_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
               ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u) : "memory");
}
__device__ __forceinline__ void st_commit_w(uint32_t bar) {
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
               : "memory");
}

// used only on the abort path, where no other role can release the wait
__device__ __forceinline__ void st_wait_bounded(uint32_t bar, uint32_t parity) {
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
    if (done || clock64() - t0 > kWaitCycles) return;
  }
}

// Named barrier of one epilogue group (128 threads, ids 2 and 3) that also
// ANDs `v` over the group: every thread of the group reaches each of these
// barriers, and all of them leave the tile loop together when any failed.
__device__ __forceinline__ bool group_and(int grp, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(2 + grp)
      : "memory");
  return r != 0u;
}

template <bool ZT>
__global__ void __launch_bounds__(kStThreads, 1)
decode_stats_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmVar,
                       const __grid_constant__ CUtensorMap tmV, const __nv_bfloat16* __restrict__ q, int Hq,
                       int Hkv, int nb, float scale, float bias2, int nsegA, int splits, float* __restrict__ scores,
                       float* __restrict__ parta, int topk, int32_t* __restrict__ idx) {
  using L = StLayout<ZT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int g = Hq / Hkv;
  const int pair = blockIdx.x / splits, part = blockIdx.x % splits;
  const int b = pair / Hkv, kh = pair % Hkv;
  const int t_lo = (int)(((long long)nsegA * part) / splits);
  const int T = (int)(((long long)nsegA * (part + 1)) / splits) - t_lo;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlot + 4);
  // with `idx`, the CTA holds the whole row of its pair (one tile range per
  // pair) and selects its top-k at the end
  float* scs = reinterpret_cast<float*>(smem + L::kScores);
  auto bar = [&](int k) { return sb + L::kBar + 8u * k; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_FK + s), 1);
      mbar_init(bar(L::B_EK + s), 1);
      mbar_init(bar(L::B_FV + s), 1);
      mbar_init(bar(L::B_EV + s), 1);
      mbar_init(bar(L::B_SC + s), 1);
      mbar_init(bar(L::B_PR + s), 4);
      mbar_init(bar(L::B_OC + s), 1);
      mbar_init(bar(L::B_TF + s), 4);
    }
    mbar_init(bar(L::B_FIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // the B operands of S1 and S2: q and ½ s² q² (hi + lo) of the group's
  // heads, rows past the group zero
  {
    const float hs = 0.5f * scale * scale;
    for (int x = threadIdx.x; x < kStN * kStD; x += kStThreads) {
      const int h = x / kStD, c = x % kStD;
      const __nv_bfloat16 qb = h < g ? q[((size_t)b * Hq + kh * g + h) * kStD + c] : __float2bfloat16_rn(0.f);
      const float qv = __bfloat162float(qb);
      const float w = hs * qv * qv;
      const __nv_bfloat16 whi = __float2bfloat16_rn(w);
      const __nv_bfloat16 wlo = __float2bfloat16_rn(w - __bfloat162float(whi));
      const uint32_t off = bop_off(h, c);
      *reinterpret_cast<__nv_bfloat16*>(smem + L::kBop + off) = qb;
      *reinterpret_cast<__nv_bfloat16*>(smem + L::kBop + kStBop + off) = whi;
      *reinterpret_cast<__nv_bfloat16*>(smem + L::kBop + 2 * kStBop + off) = wlo;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kStMmaWarp) tmem_alloc(smem_u32(tmem_slot), kStTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kStTmaWarp) {
    // ------------------------------------------------------------ TMA producers
    if (T > 0 && (lane == 0 || (ZT && lane == 1))) {
      const bool kv = lane == 0;   // lane 0: kmean and kvar; lane 1: the value means
      prefetch_tmap(kv ? &tmK : &tmV);
      if (kv) prefetch_tmap(&tmVar);
      const int fb = kv ? L::B_FK : L::B_FV, eb = kv ? L::B_EK : L::B_EV;
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t & 1;
        if (t >= 2 && !mbar_wait(bar(eb + s), ((t >> 1) - 1) & 1, abort_flag)) break;
        const int row = (t_lo + t) * kStTile;
        if (kv) {
          const uint32_t dst = sb + s * L::kKStage;
          mbar_expect_tx(bar(fb + s), L::kKStage);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_3d(dst + h * kStSpan, &tmK, 64 * h, row, pair, bar(fb + s));
            tma_load_3d(dst + kStArr + h * kStSpan, &tmVar, 64 * h, row, pair, bar(fb + s));
          }
        } else {
          const uint32_t dst = sb + L::kVRing + s * kStArr;
          mbar_expect_tx(bar(fb + s), kStArr);
#pragma unroll
          for (int h = 0; h < 2; ++h) tma_load_3d(dst + h * kStSpan, &tmV, 64 * h, row, pair, bar(fb + s));
        }
        issued = t + 1;
      }
      if (*abort_flag) {
        // let the loads already in flight land before the CTA goes away
        for (int t = issued > 2 ? issued - 2 : 0; t < issued; ++t) st_wait_bounded(bar(fb + (t & 1)), (t >> 1) & 1);
      }
    }
  } else if (warp == kStMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (T > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kStTile, kStN, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(kStD, kStN, 1, 0);   // A = V̄ᵀ: the value-mean tile read MN-major
      const uint64_t qd = desc_sw128(sb + L::kBop, 16, 1024);
      const uint64_t whd = desc_sw128(sb + L::kBop + kStBop, 16, 1024);
      const uint64_t wld = desc_sw128(sb + L::kBop + 2 * kStBop, 16, 1024);
      // S1 and S2 of tile t into TMEM buffer t % 2; the kmean/kvar stage is then free
      auto issue_s = [&](int t) -> bool {
        const int s = t & 1, k = t >> 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_FK + s), k & 1, abort_flag))) return false;
        if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(L::B_TF + s), (k - 1) & 1, abort_flag))) return false;
        tc_fence_after();
        const uint32_t stage = sb + s * L::kKStage;
        const uint64_t kd = desc_sw128(stage, 16, 1024), vd = desc_sw128(stage + kStArr, 16, 1024);
        const uint32_t dS1 = tbase + 64u * s, dS2 = dS1 + 16u;
        // K step kk: 16 channels = 32 bytes along the rows, the next span every 4 steps
#pragma unroll
        for (int kk = 0; kk < kStD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * kStSpan + (kk & 3) * 32, bo = (kk >> 2) * (kStN * 128) + (kk & 3) * 32;
          st_mma_w(dS1, desc_adv(kd, ao), desc_adv(qd, bo), idS, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < kStD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * kStSpan + (kk & 3) * 32, bo = (kk >> 2) * (kStN * 128) + (kk & 3) * 32;
          st_mma_w(dS2, desc_adv(vd, ao), desc_adv(whd, bo), idS, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < kStD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * kStSpan + (kk & 3) * 32, bo = (kk >> 2) * (kStN * 128) + (kk & 3) * 32;
          st_mma_w(dS2, desc_adv(vd, ao), desc_adv(wld, bo), idS, 1u);
        }
        st_commit_w(bar(L::B_SC + s));
        st_commit_w(bar(L::B_EK + s));
        return true;
      };
      bool ok = issue_s(0);
      for (int t = 0; ok && t < T; ++t) {
        if (t + 1 < T && !(ok = issue_s(t + 1))) break;
        if (ZT) {
          const int s = t & 1, k = t >> 1;
          if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_PR + s), k & 1, abort_flag))) break;
          if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_FV + s), k & 1, abort_flag))) break;
          tc_fence_after();
          // Oᵀ = V̄ᵀ Pᵀ: K step kk = 16 blocks = 16 rows of the value-mean tile
          const uint64_t ad = desc_sw128(sb + L::kVRing + s * kStArr, kStSpan, 1024);
          const uint64_t pd = desc_sw128(sb + L::kP + s * kStBop, 16, 1024);
          const uint32_t dO = tbase + 64u * s + 32u;
#pragma unroll
          for (int kk = 0; kk < kStTile / 16; ++kk) {
            const uint32_t bo = (kk >> 2) * (kStN * 128) + (kk & 3) * 32;
            st_mma_w(dO, desc_adv(ad, kk * 16 * 128), desc_adv(pd, bo), idO, kk > 0);
          }
          st_commit_w(bar(L::B_OC + s));
          st_commit_w(bar(L::B_EV + s));
        }
      }
      // every MMA issued above has completed before TMEM is released
      st_commit_w(bar(L::B_FIN));
      st_wait_bounded(bar(L::B_FIN), 0);
    }
  } else if (warp >= kStEpiWarp0) {
    // ------------------------------------------------------------ epilogue groups
    const int grp = (warp - kStEpiWarp0) >> 2;   // tiles t with t % 2 == grp
    const int wq = warp & 3;                      // TMEM lane quarter
    const int j = wq * 32 + lane;                 // block row of the tile (ZT: also the channel of Oᵀ)
    const uint32_t lrow = tbase + ((uint32_t)(wq * 32) << 16);
    float* red = reinterpret_cast<float*>(smem + L::kRed) + grp * (4 * kStN * 2);   // [4 warps][16][2]
    const float scale2 = scale * kLog2e;
    bool ok = true;
    for (int t = grp; t < T; t += 2) {
      const int s = t & 1, k = t >> 1;
      const int seg = t_lo + t, j0 = seg * kStTile;
      const bool valid = j0 + j < nb;
      ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(L::B_SC + s), k & 1, abort_flag));
      uint32_t sv[32];
      if (ok) {
        tc_fence_after();
        tmem_ld32(lrow + 64u * s, sv);   // S1 of the 16 heads, then S2
        tmem_wait_ld();
      }
      float x[kStN];
#pragma unroll
      for (int h = 0; h < kStN; ++h)
        x[h] = (ok && valid && h < g) ? __uint_as_float(sv[h]) * scale2 : -INFINITY;   // s log2e q·k̄
      if (ZT) {
        // each head's maximum over the tile of the log2 weight x + log2 B, then
        // P = 2^{x + log2 B − M} into the B operand of Oᵀ = V̄ᵀ Pᵀ (first: the
        // ring slot is freed only after that product)
#pragma unroll
        for (int h = 0; h < kStN; ++h) {
          if (h < g) {
            float m = x[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) red[(wq * kStN + h) * 2] = m;
          }
        }
        // every thread reaches this barrier; all leave the loop together if any failed
        if (!group_and(grp, ok)) break;
        float M[kStN];
        uint8_t* pb = smem + L::kP + s * kStBop;
#pragma unroll
        for (int h = 0; h < kStN; ++h) {
          float p = 0.f;
          M[h] = -INFINITY;
          if (h < g) {
            M[h] = fmaxf(fmaxf(red[(0 * kStN + h) * 2], red[(1 * kStN + h) * 2]),
                         fmaxf(red[(2 * kStN + h) * 2], red[(3 * kStN + h) * 2]));
            p = x[h] == -INFINITY ? 0.f : fast_exp2(x[h] - M[h]);
            float ls = p;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
            if (lane == 0) red[(wq * kStN + h) * 2 + 1] = ls;
          }
          *reinterpret_cast<__nv_bfloat16*>(pb + bop_off(h, j)) = __float2bfloat16_rn(p);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(L::B_PR + s));
        // group score of the block: ln Σ_h e^{s q_h·k̄}(1 + S2_h), from log2 terms
        float mx = -INFINITY;
#pragma unroll
        for (int h = 0; h < kStN; ++h) mx = fmaxf(mx, x[h]);
        float se = 0.f;
#pragma unroll
        for (int h = 0; h < kStN; ++h)
          if (h < g && valid) se += fast_exp2(x[h] - mx) * (1.0f + __uint_as_float(sv[16 + h]));
        if (valid) {
          const float sc = (mx + __log2f(se)) * kLn2;
          scores[(size_t)pair * nb + j0 + j] = sc;
          if (idx) scs[j0 + j] = sc;
        }
        if (!group_and(grp, true)) break;   // the heads' sums are in `red`
        if (j < g) {
          float* out = parta + (((size_t)b * Hq + kh * g + j) * nsegA + seg) * (kStD + 2);
          float Mj = -INFINITY;
#pragma unroll
          for (int h = 0; h < kStN; ++h)
            if (h == j) Mj = M[h];
          out[0] = Mj + bias2;
          out[1] = (red[(0 * kStN + j) * 2 + 1] + red[(1 * kStN + j) * 2 + 1]) +
                   (red[(2 * kStN + j) * 2 + 1] + red[(3 * kStN + j) * 2 + 1]);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_OC + s), k & 1, abort_flag));
        if (ok) {
          tc_fence_after();
          uint32_t ov[32];
          tmem_ld32(lrow + 64u * s + 32u, ov);   // Oᵀ row j = channel j, columns = heads
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kStN; ++h)
            if (h < g)
              parta[(((size_t)b * Hq + kh * g + h) * nsegA + seg) * (kStD + 2) + 2 + j] = __uint_as_float(ov[h]);
        }
      } else {
        if (!ok) break;
        float mx = -INFINITY;
#pragma unroll
        for (int h = 0; h < kStN; ++h) mx = fmaxf(mx, x[h]);
        float se = 0.f;
#pragma unroll
        for (int h = 0; h < kStN; ++h)
          if (h < g && valid) se += fast_exp2(x[h] - mx) * (1.0f + __uint_as_float(sv[16 + h]));
        if (valid) {
          const float sc = (mx + __log2f(se)) * kLn2;
          scores[(size_t)pair * nb + j0 + j] = sc;
          if (idx) scs[j0 + j] = sc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::B_TF + s));   // this TMEM buffer is read out
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kStMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kStTmemCols);
  }
  if (idx && !*abort_flag)
    radix_topk_cta<kStThreads>(scs, nb, topk, idx + (size_t)pair * topk,
                               *reinterpret_cast<RadixTopkSmem*>(smem + L::kTopk));
}

}  // namespace

sa_status decode_stats_tc(const __nv_bfloat16* q, const void* kmean, const void* kvar, const void* vmean, int B,
                          int Hq, int Hkv, int nb, int blk, float scale, int nsegA, bool zt, int sms,
                          float* scores, float* parta, int topk, int32_t* idx, bool* topk_done,
                          cudaStream_t stream) {
  const int npairs = B * Hkv;
  CUtensorMap mk, mvar, mv;
  if (!make_tmap_128x128(&mk, kmean, 2, kStD, (uint64_t)nb, (uint64_t)npairs) ||
      !make_tmap_128x128(&mvar, kvar, 2, kStD, (uint64_t)nb, (uint64_t)npairs) ||
      (zt && !make_tmap_128x128(&mv, vmean, 2, kStD, (uint64_t)nb, (uint64_t)npairs)))
    return fail(SA_ERR_CUDA, "sa_decode_fwd: cuTensorMapEncodeTiled failed for the block statistics");
  if (!zt) mv = mk;
  int splits = npairs < sms ? sms / npairs : 1;
  if (splits > nsegA) splits = nsegA;
  const dim3 grid((unsigned)(npairs * splits));
  // a CTA that holds a whole row of at most kStTopkBlocks blocks selects its top-k
  const bool fuse = splits == 1 && nb <= kStTopkBlocks && topk > 0 && idx != nullptr;
  *topk_done = fuse;
  const size_t smem = zt ? StLayout<true>::bytes() : StLayout<false>::bytes();
  auto kern = zt ? decode_stats_tc_kernel<true> : decode_stats_tc_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(decode_stats_tc_kernel)");
  kern<<<grid, kStThreads, smem, stream>>>(mk, mvar, mv, q, Hq, Hkv, nb, scale, log2f((float)blk), nsegA, splits,
                                           scores, parta, topk, fuse ? idx : nullptr);
  return launch_status("decode_stats_tc_kernel");
}

uint32_t decode_tc_error_take() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, tc::g_device_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return 0u;
  return v;
}

}  // namespace sa
