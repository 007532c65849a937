// dQ of the sparse prefill's backward on the fifth-generation tensor cores
// (tcgen05 MMAs with TMEM accumulators, TMA tiles), bf16 operands, d = 128,
// block 128.  Same gradients as bwd_dq_mma_kernel: the forward is softmax
// attention of query block i to its exact keys (the selected blocks) and, with
// the zero-order tail, one pseudo-key per unselected block (k̄_j, value
// v̄_j = vsum_j / B, logit bias ln B; PISA "Algoritmo Central"), so with
// P = softmax(s Q Kᵀ + bias) and δ_t = dO_t · o_t:
//   dP = dO Vᵀ,  dS = P ⊙ (dP − δ),  dQ = s dS K.
//
// One CTA per 128-row query block, 384 threads:
//   warps 0-7  two element-wise warpgroups; warp w reads TMEM lanes
//              32 (w % 4) .. + 31 (its query rows) and group w / 4 takes keys
//              64 g .. 64 g + 63 of every 128-key tile;
//   warp 8     TMA producer: Q and dO once, then K tiles through a ring of
//              three and V tiles through a ring of two;
//   warp 9     MMA issuer (converged; elect.sync picks the issuing lane).
// Two passes over the row block's tiles (the selected blocks, then the
// centroid tiles): pass 1 forms S = Q Kᵀ and the row's log-sum-exp (skipped
// when the forward's log-sum-exp is given); pass 2
// forms S again, dP = dO Vᵀ, writes dS (bf16) into the S columns, and
// accumulates dQ += dS · K with dS read from TMEM.
// SLA2's linear mix (delta_in non-null): the softmax branch's δ is given, and
// with dq_add the kernel adds its dQ to what dQ already holds (the linear
// branch's term, written first).
// PISA's first-order tail (doff non-null): a pseudo-key's value seen by row t
// is v̄_j + f_t / B (f_t = s H̄ᵀ q_t), so the centroid tiles take
// dS = P (dP − δ + doff_t) with doff_t = dO_t·f_t / B; the kernel also writes
// that row's centroid δ (delta_c = δ − doff) for the centroid dK/dV pass and
// each group's share of λ_t = Σ_{pseudo-keys} P / B (lam[grp · lam_stride + row]).
// TMEM (512 columns): S₀ [0,128), S₁ [128,256) (tile g in S_{g mod 2}),
// dP [256,384), dQ [384,512).  dS of tile g goes to columns [32, 96) of its S
// buffer: group 0 writes [32, 64) and group 1 [64, 96), each inside the
// columns it read itself, so neither overwrites the other's unread S.
#include "attn_simt.cuh"
#include "tc_util.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int TB = 128;                        // rows per tile (queries and keys)
constexpr int TD = 128;                        // head dim
constexpr int kThreads = 384;
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr uint32_t kSpan = TB * 128;           // 128 rows x one 128-byte swizzle span
constexpr uint32_t kTile = 2 * kSpan;          // 128 rows x 256 bytes
constexpr int NK = 3, NV = 2;                  // ring depths
constexpr uint32_t kColDP = 256, kColDQ = 384, kTmemCols = 512;

struct Lay {
  static constexpr uint32_t kQ = 0, kG = kTile, kK = 2 * kTile, kV = kK + NK * kTile;
  static constexpr int B_QG = 0, B_KF = 1, B_KE = B_KF + NK, B_VF = B_KE + NK, B_VE = B_VF + NV,
                       B_SF = B_VE + NV, B_SC = B_SF + 2, B_DPF = B_SC + 2, B_DQ = B_DPF + 1, B_FIN = B_DQ + 1,
                       NBAR = B_FIN + 1;
  static constexpr uint32_t kBarOff = kV + NV * kTile;
  static constexpr uint32_t kSlotOff = kBarOff + 8 * NBAR;   // tmem base, abort flag
  static constexpr uint32_t kMaskOff = kSlotOff + 16;
  static size_t smem_bytes(int nb) { return 1024 + kMaskOff + 4 * (size_t)((nb + 31) / 32 + 4); }
};

__device__ __forceinline__ void mma_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
               ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u) : "memory");
}
__device__ __forceinline__ void mma_ts_w(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
               ::"r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u) : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint32_t bar) {
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
               : "memory");
}
// two consecutive 32-bit TMEM columns of the warp's 32 lanes
__device__ __forceinline__ void tmem_st2(uint32_t taddr, uint32_t a, uint32_t b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t& a, uint32_t& b) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void named_bar_ew() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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

__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                 const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                 const int32_t* __restrict__ block_idx, int N, int topk, int zo, float scale,
                 const float* __restrict__ lse_in, float* __restrict__ lse2, float* __restrict__ delta,
                 float* __restrict__ dQ, const float* __restrict__ doff, float* __restrict__ delta_c,
                 float* __restrict__ lam, size_t lam_stride, const float* __restrict__ delta_in, int dq_add) {
  using L = Lay;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int k) { return sb + L::kBarOff + 8u * (uint32_t)k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlotOff + 4);
  uint32_t* selmask = reinterpret_cast<uint32_t*>(smem + L::kMaskOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = N / TB;
  const int i = blockIdx.x;                    // query block
  const int bh = blockIdx.y;
  const int nwords = (nb + 31) / 32;
  const int ntc = zo ? (nb + TB - 1) / TB : 0;  // centroid tiles
  const int T = topk + ntc;                    // tiles per pass
  // pass-1 tiles: none when the forward's log-sum-exp is given; tile sequence
  // g = 0 .. P1 + T - 1, the last T being pass 2
  const int P1 = lse_in ? 0 : T, G = P1 + T;
  const int32_t* sel = block_idx + ((size_t)bh * nb + i) * (size_t)topk;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_QG), 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(bar(L::B_KF + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bar(L::B_VF + s), 1);
      mbar_init(bar(L::B_VE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_SF + s), 1);
      mbar_init(bar(L::B_SC + s), 256);
    }
    mbar_init(bar(L::B_DPF), 1);
    mbar_init(bar(L::B_DQ), 1);
    mbar_init(bar(L::B_FIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // selection bitmap, padded with 4 zero words so a tile's words never run past it
  for (int w = threadIdx.x; w < nwords + 4; w += kThreads) selmask[w] = 0u;
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && T > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmG);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (zo) {
        prefetch_tmap(&tmKb);
        prefetch_tmap(&tmVb);
      }
      mbar_expect_tx(bar(L::B_QG), 2 * kTile);
      for (int h = 0; h < 2; ++h) {
        tma_load_3d(sb + L::kQ + h * kSpan, &tmQ, 64 * h, i * TB, bh, bar(L::B_QG));
        tma_load_3d(sb + L::kG + h * kSpan, &tmG, 64 * h, i * TB, bh, bar(L::B_QG));
      }
      // K loads n = 0 .. G-1 (tile n, then n - P1 in pass 2); V loads of pass 2 follow their K
      int nk = 0, nv = 0;
      for (int n = 0; n < G; ++n) {
        const int t = n < P1 ? n : n - P1;
        const bool exact = t < topk;
        const int row = exact ? sel[t] * TB : (t - topk) * TB;
        {
          const int s = n % NK;
          if (n >= NK && !mbar_wait(bar(L::B_KE + s), ((n / NK) - 1) & 1, abort_flag)) break;
          mbar_expect_tx(bar(L::B_KF + s), kTile);
          for (int h = 0; h < 2; ++h)
            tma_load_3d(sb + L::kK + s * kTile + h * kSpan, exact ? &tmK : &tmKb, 64 * h, row, bh,
                        bar(L::B_KF + s));
          nk = n + 1;
        }
        if (n >= P1) {
          const int s = t % NV;
          if (t >= NV && !mbar_wait(bar(L::B_VE + s), ((t / NV) - 1) & 1, abort_flag)) break;
          mbar_expect_tx(bar(L::B_VF + s), kTile);
          for (int h = 0; h < 2; ++h)
            tma_load_3d(sb + L::kV + s * kTile + h * kSpan, exact ? &tmV : &tmVb, 64 * h, row, bh,
                        bar(L::B_VF + s));
          nv = t + 1;
        }
      }
      if (*abort_flag) {
        // let the loads already in flight land before the CTA goes away
        wait_bounded(bar(L::B_QG), 0);
        for (int n = nk > NK ? nk - NK : 0; n < nk; ++n) wait_bounded(bar(L::B_KF + n % NK), (n / NK) & 1);
        for (int t = nv > NV ? nv - NV : 0; t < nv; ++t) wait_bounded(bar(L::B_VF + t % NV), (t / NV) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (T > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(TB, TB, 0, 0);    // S, dP: both operands K-major
      constexpr uint32_t idQ = idesc_bf16_f32(TB, TD, 0, 1);    // dQ: K as the MN-major operand
      const uint64_t qd0 = desc_sw128(sb + L::kQ, 16, 1024);
      const uint64_t gd0 = desc_sw128(sb + L::kG, 16, 1024);
      // S(g) = Q K(g)ᵀ into S_{g mod 2}; pass-1 tiles release their K stage here
      auto issue_s = [&](int g) -> bool {
        const int s = g % NK;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_KF + s), (g / NK) & 1, abort_flag))) return false;
        tc_fence_after();
        const uint64_t kd0 = desc_sw128(sb + L::kK + s * kTile, 16, 1024);
        const uint32_t d = tbase + (uint32_t)(g & 1) * TB;
#pragma unroll
        for (int k = 0; k < TD / 16; ++k) {
          const uint32_t koff = (k >> 2) * kSpan + (k & 3) * 32;
          mma_ss_w(d, desc_adv(qd0, koff), desc_adv(kd0, koff), idS, k > 0);
        }
        mma_commit_w(bar(L::B_SF + (g & 1)));
        if (g < P1) mma_commit_w(bar(L::B_KE + s));
        return true;
      };
      // dP(t) = dO V(t)ᵀ; releases the V stage
      auto issue_dp = [&](int t) -> bool {
        const int s = t % NV;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_VF + s), (t / NV) & 1, abort_flag))) return false;
        tc_fence_after();
        const uint64_t vd0 = desc_sw128(sb + L::kV + s * kTile, 16, 1024);
#pragma unroll
        for (int k = 0; k < TD / 16; ++k) {
          const uint32_t koff = (k >> 2) * kSpan + (k & 3) * 32;
          mma_ss_w(tbase + kColDP, desc_adv(gd0, koff), desc_adv(vd0, koff), idS, k > 0);
        }
        mma_commit_w(bar(L::B_DPF));
        mma_commit_w(bar(L::B_VE + s));
        return true;
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_QG), 0, abort_flag));
      if (ok) ok = issue_s(0);
      if (ok && G > 1) ok = issue_s(1);
      // pass 1: S only; a buffer is reissued once its S has been read
      for (int g = 0; ok && g < P1; ++g) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SC + (g & 1)), (g >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (g + 2 < G) ok = issue_s(g + 2);
      }
      // pass 2: dP one tile ahead, dQ += dS K once dS is in TMEM
      if (ok) ok = issue_dp(0);
      for (int g = P1; ok && g < G; ++g) {
        const int t = g - P1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SC + (g & 1)), (g >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (t + 1 < T && !(ok = issue_dp(t + 1))) break;
        const int s = g % NK;
        const uint64_t kd0 = desc_sw128(sb + L::kK + s * kTile, kSpan, 1024);
        const uint32_t a0 = tbase + (uint32_t)(g & 1) * TB + 32;
#pragma unroll
        for (int k = 0; k < TB / 16; ++k)
          // K step k: 16 keys = 16 rows of 128 bytes into K; 8 TMEM columns of dS
          mma_ts_w(tbase + kColDQ, a0 + 8 * k, desc_adv(kd0, k * 16 * 128), idQ, (t > 0 || k > 0));
        mma_commit_w(bar(L::B_KE + s));
        if (g + 2 < G) ok = issue_s(g + 2);
      }
      mma_commit_w(bar(L::B_DQ));
      // every MMA issued above has completed before TMEM is released
      mma_commit_w(bar(L::B_FIN));
      wait_bounded(bar(L::B_FIN), 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ element-wise
    for (int s = threadIdx.x; s < topk; s += 256) {
      const int j = sel[s];
      atomicOr(&selmask[j >> 5], 1u << (j & 31));
    }
    named_bar_ew();                             // the bitmap is complete
    const int grp = warp >> 2;                  // key half of every tile
    const int wq = warp & 3;                    // TMEM lane quarter
    const int r = wq * 32 + lane;               // query row within the block
    const size_t row = (size_t)bh * N + (size_t)i * TB + r;
    const uint32_t lrow = tbase + ((uint32_t)(wq * 32) << 16);
    const float scale2 = scale * kLog2e;
    // δ = dO · O over the row's 128 channels (both groups, from the stored bf16
    // output), or the caller's δ (SLA2's linear mix: the softmax branch's own)
    float dl = 0.f;
    if (delta_in) {
      dl = delta_in[row];
    } else {
      const uint4* go = reinterpret_cast<const uint4*>(dO + row * TD);
      const uint4* oo = reinterpret_cast<const uint4*>(O + row * TD);
#pragma unroll 4
      for (int c = 0; c < TD / 8; ++c) {
        const uint4 a = go[c], b = oo[c];
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
          const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
          dl = fmaf(fa.x, fb.x, dl);
          dl = fmaf(fa.y, fb.y, dl);
        }
      }
    }
    // validity of the thread's 64 keys of tile t (bit c = key 64 grp + c)
    auto valid_bits = [&](int t, uint32_t& v0, uint32_t& v1) {
      if (t < topk) {
        v0 = v1 = 0xffffffffu;
        return;
      }
      const int jb = (t - topk) * TB + 64 * grp;
      const int w0 = jb >> 5;
      const int lim0 = nb - jb, lim1 = nb - (jb + 32);
      const uint32_t r0 = lim0 >= 32 ? 0xffffffffu : (lim0 <= 0 ? 0u : ((1u << lim0) - 1u));
      const uint32_t r1 = lim1 >= 32 ? 0xffffffffu : (lim1 <= 0 ? 0u : ((1u << lim1) - 1u));
      v0 = ~selmask[w0] & r0;
      v1 = ~selmask[w0 + 1] & r1;
    };
    bool ok = true;
    float m = -INFINITY, l = 0.f;
    // ---- pass 1: the row's running max and sum over its 64 keys of every tile
    for (int g = 0; g < P1; ++g) {
      const int b = g & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SF + b), (g >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[64];
      tmem_ld32(lrow + (uint32_t)b * TB + 64 * grp, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld32(lrow + (uint32_t)b * TB + 64 * grp + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::B_SC + b));
      uint32_t vb0, vb1;
      valid_bits(g, vb0, vb1);
      const float bias = g < topk ? 0.f : 7.0f;   // log2 of the block size 128
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const bool ok_c = ((c < 32 ? vb0 : vb1) >> (c & 31)) & 1u;
        const float x = ok_c ? fmaf(__uint_as_float(v[c]), scale2, bias) : -INFINITY;
        v[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      const float mn = fmaxf(m, mx);
      if (mn == -INFINITY) continue;
      float sm = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) sm += fast_exp2(__uint_as_float(v[c]) - mn);
      l = l * (m == -INFINITY ? 0.f : fast_exp2(m - mn)) + sm;
      m = mn;
    }
    // ---- the two groups' (max, sum) through the unused dQ columns
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    float lse = INFINITY;
    if (ok && P1 > 0) {
      tmem_st2(lrow + kColDQ + 2 * grp, __float_as_uint(m), __float_as_uint(l));
      tmem_wait_st();
    }
    tc_fence_before();
    named_bar_ew();
    tc_fence_after();
    const float dof = doff ? doff[row] : 0.f;
    if (ok && grp == 0 && delta_c) delta_c[row] = dl - dof;
    if (ok && P1 == 0) {
      lse = lse_in[row];
      if (grp == 0) {
        lse2[row] = lse;
        delta[row] = dl;
      }
    } else if (ok) {
      uint32_t mo, lo;
      tmem_ld2(lrow + kColDQ + 2 * (1 - grp), mo, lo);
      tmem_wait_ld();
      const float m1 = __uint_as_float(mo), l1 = __uint_as_float(lo);
      const float M = fmaxf(m, m1);
      const float Ls = (M == -INFINITY) ? 0.f
                                        : (m == -INFINITY ? 0.f : l * fast_exp2(m - M)) +
                                              (m1 == -INFINITY ? 0.f : l1 * fast_exp2(m1 - M));
      lse = Ls > 0.f ? M + log2f(Ls) : INFINITY;
      if (grp == 0) {
        lse2[row] = lse;
        delta[row] = dl;
      }
    }
    // both groups have read the exchange before the first dQ MMA overwrites it
    // (that MMA waits for every thread's arrival on the S barrier of tile P1)
    // ---- pass 2: dS = P (dP − δ) into the S columns [32, 96)
    float lam_part = 0.f;   // Σ P over this group's pseudo-keys
    for (int g = P1; ok && g < G; ++g) {
      const int t = g - P1, b = g & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SF + b), (g >> 1) & 1, abort_flag)) ||
          !__all_sync(0xffffffffu, mbar_wait(bar(L::B_DPF), t & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[64], p[64];
      tmem_ld32(lrow + (uint32_t)b * TB + 64 * grp, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld32(lrow + (uint32_t)b * TB + 64 * grp + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_ld32(lrow + kColDP + 64 * grp, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
      tmem_ld32(lrow + kColDP + 64 * grp + 32, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
      tmem_wait_ld();
      uint32_t vb0, vb1;
      valid_bits(t, vb0, vb1);
      const bool cent = t >= topk;
      const float nb2 = (cent ? 7.0f : 0.f) - lse;
      const float dlt = cent ? dl - dof : dl;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int cc = 2 * c + e;
          const bool ok_c = ((cc < 32 ? vb0 : vb1) >> (cc & 31)) & 1u;
          const float pr = ok_c ? fast_exp2(fmaf(__uint_as_float(v[cc]), scale2, nb2)) : 0.f;
          psum += pr;
          ds[e] = pr * (__uint_as_float(p[cc]) - dlt);
        }
        v[c] = pack_bf16(ds[0], ds[1]);
      }
      if (cent) lam_part += psum;
      tmem_st32(lrow + (uint32_t)b * TB + 32 + 32 * grp, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::B_SC + b));
    }
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    if (ok && lam) lam[(size_t)grp * lam_stride + row] = lam_part * (1.0f / TB);   // ÷ B = 128
    if (ok && T > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_DQ), 0, abort_flag));
    float4* out = reinterpret_cast<float4*>(dQ + row * TD + 64 * grp);
    if (ok && T > 0) {
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[32];
        tmem_ld32(lrow + kColDQ + 64 * grp + 32 * h, a);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 y = make_float4(scale * __uint_as_float(a[4 * q]), scale * __uint_as_float(a[4 * q + 1]),
                                 scale * __uint_as_float(a[4 * q + 2]), scale * __uint_as_float(a[4 * q + 3]));
          if (dq_add) {
            const float4 x = out[8 * h + q];
            y.x += x.x;
            y.y += x.y;
            y.z += x.z;
            y.w += x.w;
          }
          out[8 * h + q] = y;
        }
      }
    } else if (T == 0 && !dq_add) {
#pragma unroll
      for (int q = 0; q < 16; ++q) out[q] = make_float4(0.f, 0.f, 0.f, 0.f);
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

// ---- dK, dV of the exact keys --------------------------------------------
// One CTA per 128-key block j, over the query blocks that selected it (the
// transposed index offs/list, ascending), with the keys as the MMA rows:
//   Sᵀ = K Q_cᵀ, dPᵀ = V dO_cᵀ, Pᵀ = 2^(s' Sᵀ − lse2), dSᵀ = Pᵀ ⊙ (dPᵀ − δ),
//   dV += Pᵀ dO_c, dK += dSᵀ Q_c     (dK scaled by s at the end).
// Warps 0-7: element-wise, group h = warp / 4 owns query rows 64 h .. + 63
// of every chunk (its half); warp 8: TMA (K, V once; a ring of two
// (Q, dO, lse2, δ) chunks); warp 9: MMA.  Each half has its own Sᵀ and dPᵀ
// (M = 128 keys, N = 64 rows), so while one group forms its Pᵀ and dSᵀ the
// tensor pipe runs the other half's products: per chunk the MMA warp issues
// dV, dK of half 0, then Sᵀ, dPᵀ of the next chunk's half 0, then the same
// for half 1.  TMEM: half h at [128 h, 128 h + 128) (Sᵀ in the first 64
// columns, dPᵀ in the next 64; Pᵀ and dSᵀ, bf16, overwrite the first 32 of
// each), dV [256,384), dK [384,512).
constexpr int NR = 2;                          // query-chunk ring depth
constexpr uint32_t kColDV = 256, kColDK = 384;

struct KvLay {
  static constexpr uint32_t kK = 0, kV = kTile, kR = 2 * kTile;     // ring stage: Q, dO
  static constexpr uint32_t kLsd = kR + NR * 2 * kTile;             // [NR][lse2 128, δ 128] floats
  static constexpr int B_KV = 0, B_RF = 1, B_RE = B_RF + NR, B_SF = B_RE + NR, B_EW = B_SF + 2,
                       B_ACC = B_EW + 2, B_FIN = B_ACC + 1, NBAR = B_FIN + 1;
  static constexpr uint32_t kBarOff = kLsd + NR * 2 * TB * 4;
  static constexpr uint32_t kSlotOff = kBarOff + 8 * NBAR;
  static constexpr size_t kSmem = 1024 + kSlotOff + 16;
};

__device__ __forceinline__ float4 lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// CENT = false: the keys of block j over the query blocks that selected it;
// dK = s acc + (s / B) dk̄_j and dV = acc + dv̄_j / B, with dk̄_j, dv̄_j the
// block's pseudo-key gradients (cent_k, cent_v; null without the tail).
// CENT = true: 128 pseudo-keys (tmK, tmV over the bf16 centroids, bias
// log2 B) over one of nsplit ranges of the head's query blocks, masked where
// the query block selected the centroid's block; the unscaled sums go to
// part[2][nsplit][BH][nb][d] for bwd_cent_reduce_kernel.
template <bool CENT>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int N, int topk,
                  const int32_t* __restrict__ offs, const int32_t* __restrict__ list,
                  const int32_t* __restrict__ block_idx, int nsplit, float scale, const float* __restrict__ lse2,
                  const float* __restrict__ delta, const float* __restrict__ cent_k,
                  const float* __restrict__ cent_v, float* __restrict__ dK, float* __restrict__ dV,
                  float* __restrict__ part) {
  using L = KvLay;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int k) { return sb + L::kBarOff + 8u * (uint32_t)k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlotOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = N / TB;
  const int bh = blockIdx.y;
  // key tile j (exact: block j; centroids: centroids 128 j ..) and its query chunks
  int j, C, qlo = 0, split = 0;
  const int32_t* lst = nullptr;
  if (CENT) {
    j = blockIdx.x / nsplit;
    split = blockIdx.x % nsplit;
    qlo = (int)(((long)nb * split) / nsplit);
    C = (int)(((long)nb * (split + 1)) / nsplit) - qlo;
  } else {
    j = blockIdx.x;
    const int32_t* off = offs + (size_t)bh * (nb + 1);
    lst = list + (size_t)bh * nb * topk + off[j];
    C = off[j + 1] - off[j];                   // query blocks that selected block j
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_KV), 1);
    for (int s = 0; s < NR; ++s) {
      mbar_init(bar(L::B_RF + s), 1);
      mbar_init(bar(L::B_RE + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(L::B_SF + h), 1);
      mbar_init(bar(L::B_EW + h), 128);
    }
    mbar_init(bar(L::B_ACC), 1);
    mbar_init(bar(L::B_FIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && C > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmG);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(bar(L::B_KV), 2 * kTile);
      for (int h = 0; h < 2; ++h) {
        tma_load_3d(sb + L::kK + h * kSpan, &tmK, 64 * h, j * TB, bh, bar(L::B_KV));
        tma_load_3d(sb + L::kV + h * kSpan, &tmV, 64 * h, j * TB, bh, bar(L::B_KV));
      }
      int issued = 0;
      for (int c = 0; c < C; ++c) {
        const int s = c % NR;
        if (c >= NR && !mbar_wait(bar(L::B_RE + s), ((c / NR) - 1) & 1, abort_flag)) break;
        const int row0 = (CENT ? qlo + c : lst[c]) * TB;
        const uint32_t st = sb + L::kR + s * 2 * kTile;
        mbar_expect_tx(bar(L::B_RF + s), 2 * kTile + 2 * TB * 4);
        for (int h = 0; h < 2; ++h) {
          tma_load_3d(st + h * kSpan, &tmQ, 64 * h, row0, bh, bar(L::B_RF + s));
          tma_load_3d(st + kTile + h * kSpan, &tmG, 64 * h, row0, bh, bar(L::B_RF + s));
        }
        const uint32_t ls = sb + L::kLsd + s * 2 * TB * 4;
        bulk_load(ls, lse2 + (size_t)bh * N + row0, TB * 4, bar(L::B_RF + s));
        bulk_load(ls + TB * 4, delta + (size_t)bh * N + row0, TB * 4, bar(L::B_RF + s));
        issued = c + 1;
      }
      if (*abort_flag) {
        wait_bounded(bar(L::B_KV), 0);
        for (int c = issued > NR ? issued - NR : 0; c < issued; ++c) wait_bounded(bar(L::B_RF + c % NR), (c / NR) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (C > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(TB, 64, 0, 0);    // Sᵀ, dPᵀ of a half: both operands K-major
      constexpr uint32_t idA = idesc_bf16_f32(TB, TD, 0, 1);    // dV, dK: dO / Q as the MN-major operand
      const uint64_t kd0 = desc_sw128(sb + L::kK, 16, 1024);
      const uint64_t vd0 = desc_sw128(sb + L::kV, 16, 1024);
      // Sᵀ and dPᵀ of half h of chunk c (rows 64 h .. + 63 start 8 KB into each span)
      auto issue_s = [&](int c, int h) -> bool {
        const int s = c % NR;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_RF + s), (c / NR) & 1, abort_flag))) return false;
        tc_fence_after();
        const uint32_t st = sb + L::kR + s * 2 * kTile + 8192u * h;
        const uint64_t qd0 = desc_sw128(st, 16, 1024), gd0 = desc_sw128(st + kTile, 16, 1024);
        const uint32_t d = tbase + 128u * h;
#pragma unroll
        for (int k = 0; k < TD / 16; ++k) {
          const uint32_t koff = (k >> 2) * kSpan + (k & 3) * 32;
          mma_ss_w(d, desc_adv(kd0, koff), desc_adv(qd0, koff), idS, k > 0);
        }
#pragma unroll
        for (int k = 0; k < TD / 16; ++k) {
          const uint32_t koff = (k >> 2) * kSpan + (k & 3) * 32;
          mma_ss_w(d + 64, desc_adv(vd0, koff), desc_adv(gd0, koff), idS, k > 0);
        }
        mma_commit_w(bar(L::B_SF + h));
        return true;
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_KV), 0, abort_flag));
      if (ok) ok = issue_s(0, 0);
      if (ok) ok = issue_s(0, 1);
      for (int c = 0; ok && c < C; ++c) {
        const int s = c % NR;
        const uint32_t st = sb + L::kR + s * 2 * kTile;
        const uint64_t qm0 = desc_sw128(st, kSpan, 1024), gm0 = desc_sw128(st + kTile, kSpan, 1024);
        for (int h = 0; ok && h < 2; ++h) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_EW + h), c & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pa = tbase + 128u * h;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            // K step k: 16 query rows (64 h + 16 k ..) of 128 bytes; 8 TMEM columns of Pᵀ
            mma_ts_w(tbase + kColDV, pa + 8 * k, desc_adv(gm0, (4 * h + k) * 16 * 128), idA,
                     (c > 0 || h > 0 || k > 0));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts_w(tbase + kColDK, pa + 64 + 8 * k, desc_adv(qm0, (4 * h + k) * 16 * 128), idA,
                     (c > 0 || h > 0 || k > 0));
          if (h == 1) mma_commit_w(bar(L::B_RE + s));
          if (c + 1 < C) ok = issue_s(c + 1, h);
        }
      }
      mma_commit_w(bar(L::B_ACC));
      mma_commit_w(bar(L::B_FIN));
      wait_bounded(bar(L::B_FIN), 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ element-wise
    const int grp = warp >> 2;                  // query-row half of every chunk (h)
    const int wq = warp & 3;                    // TMEM lane quarter
    const int r = wq * 32 + lane;               // key within the block
    const uint32_t lrow = tbase + ((uint32_t)(wq * 32) << 16);
    const float scale2 = scale * kLog2e;
    bool ok = true;
    for (int c = 0; c < C; ++c) {
      const int s = c % NR;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SF + grp), c & 1, abort_flag)) ||
          !__all_sync(0xffffffffu, mbar_wait(bar(L::B_RF + s), (c / NR) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t hcol = lrow + 128u * grp;
      uint32_t v[64], p[64];
      tmem_ld32(hcol, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld32(hcol + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_ld32(hcol + 64, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
      tmem_ld32(hcol + 96, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
      tmem_wait_ld();
      // the chunk's lse2 and δ of this group's 64 rows (shared-memory addresses)
      const uint32_t ls_a = sb + L::kLsd + (uint32_t)(s * 2 * TB + 64 * grp) * 4u;
      const uint32_t dl_a = ls_a + TB * 4u;
      // pseudo-keys: live unless past the head's blocks or selected by this query block
      bool live = true;
      if (CENT) {
        const int jj = j * TB + r;
        live = jj < nb;
        const int32_t* sq = block_idx + ((size_t)bh * nb + qlo + c) * (size_t)topk;
        for (int x = 0; x < topk; ++x) live &= __ldg(sq + x) != jj;
      }
      const float bias = CENT ? 7.0f : 0.f;   // log2 of the block size 128
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 la = lds4(ls_a + 16u * q), da = lds4(dl_a + 16u * q);
        const float lq[4] = {la.x, la.y, la.z, la.w}, dq[4] = {da.x, da.y, da.z, da.w};
        float pr[4], ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int cc = 4 * q + e;
          pr[e] = live ? fast_exp2(fmaf(__uint_as_float(v[cc]), scale2, bias - lq[e])) : 0.f;
          ds[e] = pr[e] * (__uint_as_float(p[cc]) - dq[e]);
        }
        v[2 * q] = pack_bf16(pr[0], pr[1]);
        v[2 * q + 1] = pack_bf16(pr[2], pr[3]);
        p[2 * q] = pack_bf16(ds[0], ds[1]);
        p[2 * q + 1] = pack_bf16(ds[2], ds[3]);
      }
      tmem_st32(hcol, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_st32(hcol + 64, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::B_EW + grp));
    }
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    if (ok && C > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_ACC), 0, abort_flag));
    // accumulators (zero without chunks), 64 channels of the thread's key
    float acc_v[64], acc_k[64];
    if (ok && C > 0) {
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tmem_ld32(lrow + kColDV + 64 * grp + 32 * h, *reinterpret_cast<uint32_t(*)[32]>(&acc_v[32 * h]));
        tmem_ld32(lrow + kColDK + 64 * grp + 32 * h, *reinterpret_cast<uint32_t(*)[32]>(&acc_k[32 * h]));
      }
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 64; ++e) acc_v[e] = acc_k[e] = 0.f;
    }
    if (ok || C == 0) {
      if (CENT) {
        const int jj = j * TB + r;
        if (jj < nb) {
          const size_t BHn = gridDim.y;
          float4* pk4 = reinterpret_cast<float4*>(part + (((size_t)split * BHn + bh) * nb + jj) * TD + 64 * grp);
          float4* pv4 =
              reinterpret_cast<float4*>(part + (((size_t)(nsplit + split) * BHn + bh) * nb + jj) * TD + 64 * grp);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            pk4[q] = make_float4(acc_k[4 * q], acc_k[4 * q + 1], acc_k[4 * q + 2], acc_k[4 * q + 3]);
            pv4[q] = make_float4(acc_v[4 * q], acc_v[4 * q + 1], acc_v[4 * q + 2], acc_v[4 * q + 3]);
          }
        }
      } else {
        const size_t krow = ((size_t)bh * N + (size_t)j * TB + r) * TD + 64 * grp;
        float4* ok4 = reinterpret_cast<float4*>(dK + krow);
        float4* ov4 = reinterpret_cast<float4*>(dV + krow);
        const size_t crow = ((size_t)bh * nb + j) * TD + 64 * grp;
        const float sk = scale * (1.0f / TB), sv = 1.0f / TB;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float4 a = make_float4(scale * acc_k[4 * q], scale * acc_k[4 * q + 1], scale * acc_k[4 * q + 2],
                                 scale * acc_k[4 * q + 3]);
          float4 b = make_float4(acc_v[4 * q], acc_v[4 * q + 1], acc_v[4 * q + 2], acc_v[4 * q + 3]);
          if (cent_k) {
            const float4 ck = *reinterpret_cast<const float4*>(cent_k + crow + 4 * q);
            const float4 cv = *reinterpret_cast<const float4*>(cent_v + crow + 4 * q);
            a.x = fmaf(sk, ck.x, a.x);
            a.y = fmaf(sk, ck.y, a.y);
            a.z = fmaf(sk, ck.z, a.z);
            a.w = fmaf(sk, ck.w, a.w);
            b.x = fmaf(sv, cv.x, b.x);
            b.y = fmaf(sv, cv.y, b.y);
            b.z = fmaf(sv, cv.z, b.z);
            b.w = fmaf(sv, cv.w, b.w);
          }
          ok4[q] = a;
          ov4[q] = b;
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

// dk̄_j, dv̄_j = the splits' partial sums in order, written over split 0
// (one CTA per (centroid, head), thread = channel).
__global__ void __launch_bounds__(TD)
bwd_cent_reduce_kernel(float* __restrict__ part, int nb, int nsplit) {
  const int j = blockIdx.x, c = threadIdx.x;
  const size_t bh = blockIdx.y, BHn = gridDim.y;
  for (int slot = 0; slot < 2; ++slot) {
    float acc = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) acc += part[(((size_t)(slot * nsplit + sp) * BHn + bh) * nb + j) * TD + c];
    part[(((size_t)(slot * nsplit) * BHn + bh) * nb + j) * TD + c] = acc;
  }
}

}  // namespace

sa_status bwd_dq_tc(const void* Q, const void* K, const void* V, const void* O, const void* dO, const sa_shape& s,
                    const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st, float scale,
                    const float* lse_in, float* lse2, float* delta, float* dQ, cudaStream_t stream,
                    const BwdTailTerms* fo) {
  const int nb = s.N / TB;
  const uint64_t BH = (uint64_t)s.B * s.H;
  alignas(64) CUtensorMap mq, mg, mk, mv, mkb, mvb;
  if (!make_tmap_128x128(&mq, Q, 2, TD, s.N, BH) || !make_tmap_128x128(&mg, dO, 2, TD, s.N, BH) ||
      !make_tmap_128x128(&mk, K, 2, TD, s.N, BH) || !make_tmap_128x128(&mv, V, 2, TD, s.N, BH))
    return fail(SA_ERR_CUDA, "sa_sparse_attn_bwd: cuTensorMapEncodeTiled failed for Q/dO/K/V");
  if (zo) {
    if (!make_tmap_128x128(&mkb, st.kmean_bf16, 2, TD, nb, BH) ||
        !make_tmap_128x128(&mvb, st.vmean_bf16, 2, TD, nb, BH))
      return fail(SA_ERR_CUDA, "sa_sparse_attn_bwd: cuTensorMapEncodeTiled failed for the block centroids");
  } else {
    mkb = mk;
    mvb = mv;
  }
  const size_t smem = Lay::smem_bytes(nb);
  if (cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(bwd_dq_tc_kernel)");
  bwd_dq_tc_kernel<<<dim3(nb, (unsigned)BH), kThreads, smem, stream>>>(
      mq, mg, mk, mv, mkb, mvb, static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO),
      block_idx, s.N, topk, zo ? 1 : 0, scale, lse_in, lse2, delta, dQ, fo ? fo->doff : nullptr,
      fo ? fo->delta_c : nullptr, fo ? fo->lam : nullptr, (size_t)BH * s.N, fo ? fo->delta_in : nullptr,
      fo && fo->dq_add ? 1 : 0);
  return launch_status("bwd_dq_tc_kernel");
}

sa_status bwd_dkv_tc(const void* Q, const void* K, const void* V, const void* dO, const sa_shape& s,
                     const int32_t* block_idx, int topk, bool zo, const sa_block_stats& st, const int32_t* offs,
                     const int32_t* list, float scale, const float* lse2, const float* delta, float* dK, float* dV,
                     float* part, int nsplit, cudaStream_t stream, const float* delta_cent) {
  const int nb = s.N / TB;
  const uint64_t BH = (uint64_t)s.B * s.H;
  alignas(64) CUtensorMap mq, mg, mk, mv;
  if (!make_tmap_128x128(&mq, Q, 2, TD, s.N, BH) || !make_tmap_128x128(&mg, dO, 2, TD, s.N, BH) ||
      !make_tmap_128x128(&mk, K, 2, TD, s.N, BH) || !make_tmap_128x128(&mv, V, 2, TD, s.N, BH))
    return fail(SA_ERR_CUDA, "sa_sparse_attn_bwd: cuTensorMapEncodeTiled failed for Q/dO/K/V");
  const float* cent_k = nullptr;
  const float* cent_v = nullptr;
  if (zo) {
    // the pseudo-keys first: partial sums per query-block range, reduced in order
    alignas(64) CUtensorMap mkb, mvb;
    if (!make_tmap_128x128(&mkb, st.kmean_bf16, 2, TD, nb, BH) ||
        !make_tmap_128x128(&mvb, st.vmean_bf16, 2, TD, nb, BH))
      return fail(SA_ERR_CUDA, "sa_sparse_attn_bwd: cuTensorMapEncodeTiled failed for the block centroids");
    auto kc = bwd_dkv_tc_kernel<true>;
    if (cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KvLay::kSmem) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(bwd_dkv_tc_kernel)");
    const int ntc = (nb + TB - 1) / TB;
    kc<<<dim3(ntc * nsplit, (unsigned)BH), kThreads, KvLay::kSmem, stream>>>(
        mq, mg, mkb, mvb, s.N, topk, offs, list, block_idx, nsplit, scale, lse2, delta_cent ? delta_cent : delta,
        nullptr, nullptr, dK, dV, part);
    sa_status r = launch_status("bwd_dkv_tc_kernel(centroids)");
    if (r != SA_OK) return r;
    bwd_cent_reduce_kernel<<<dim3(nb, (unsigned)BH), TD, 0, stream>>>(part, nb, nsplit);
    r = launch_status("bwd_cent_reduce_kernel");
    if (r != SA_OK) return r;
    cent_k = part;
    cent_v = part + (size_t)nsplit * BH * nb * TD;
  }
  auto ke = bwd_dkv_tc_kernel<false>;
  if (cudaFuncSetAttribute(ke, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KvLay::kSmem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(bwd_dkv_tc_kernel)");
  ke<<<dim3(nb, (unsigned)BH), kThreads, KvLay::kSmem, stream>>>(mq, mg, mk, mv, s.N, topk, offs, list, block_idx,
                                                                 nsplit, scale, lse2, delta, cent_k, cent_v, dK, dV,
                                                                 part);
  return launch_status("bwd_dkv_tc_kernel");
}

uint32_t bwd_error_take() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, tc::g_device_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return 0u;
  return v;
}

}  // namespace sa
