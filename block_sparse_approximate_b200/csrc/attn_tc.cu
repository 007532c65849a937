// Sparse prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// 128-token blocks, d = 128, tails drop and zero-order, with bf16 operands
// (kind::f16) or per-block-scaled e4m3 operands (kind::f8f6f4, SLA2 §2C's
// low-precision sparse branch).
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
//   warp 9     MMA issuer (the whole warp runs the loop, one elected lane
//              issues): S = Q·Kᵀ (both operands K-major in shared memory)
//              into the stream's S, and O_s += P·V with P read from TMEM and V
//              as an MN-major shared-memory operand, alternating the streams
//              so one group's softmax overlaps the other group's MMAs.
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
//
// e4m3 variant: Q, K, V (and the centroid tiles) are e4m3 codes with one
// scale per 128-row block; S = σ_Q σ_K (Q̂·K̂ᵀ).  P is quantised to e4m3 as
// P · 112 · σ_V(tile) / σ_Vmax (P ≤ 4: the running max is applied lazily,
// once it has grown by more than a factor 4, and 4 · 112 = 448 is the e4m3
// maximum), so the MMA accumulates Σ P σ_V V̂ · 112 / σ_Vmax across tiles of
// different V scales; the row sum uses the unquantised P.  σ_Vmax is the
// largest V scale of the head (exact and centroid tiles).
#include <mutex>

#include "attn_simt.cuh"
#include <cuda_fp8.h>

#include "tc_util.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int TB = 128;                        // rows per tile (queries and keys)
constexpr int TD = 128;                        // head dim
constexpr int kTcThreads = 384;
constexpr int kTmaWarp = 8, kMmaWarp = 9;
// register split: 256 softmax threads x 216 + 128 producer threads x 40 =
// 60416 <= 384 x (launch registers); build.py checks ptxas reports >= 158
constexpr int kSoftmaxRegs = 216, kProducerRegs = 40;
constexpr uint32_t kSpan = TB * 128;           // 128 rows x one 128-byte swizzle span = 16 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
// bf16 softmax: pair n of a row's 64 exponential pairs runs on the FMA pipe
// (exp2_poly2) when bit n % 8 is set, else on MUFU.  Three of eight was the
// fastest split measured on B200 for d = 128 tiles.
constexpr uint32_t kExpFma = 0x49u;
// e4m3 softmax: quad n of a row's 32 exponential quads runs on the FMA pipe
// when bit n % 8 is set.  The e4m3 packing already loads the FMA pipe, so
// only one quad in four moves there (measured on B200: 0, 1, 3, 4, 5 and 6 of
// eight; 2 was the fastest, and 4 or more slower than none).
constexpr uint32_t kExpFmaF8 = 0x11u;

// Operand format of the kernel: spans per 128x128 tile, pipeline depth, MMA
// K step (in elements), lazy-rescale threshold.
template <bool F8>
struct Fmt;
template <>
struct Fmt<false> {   // bf16
  static constexpr int kSpans = 2;             // 256 bytes per row
  static constexpr int NS = 3;
  static constexpr int kK = 16;                // K per MMA instruction
  static constexpr float kLazy = 8.0f;
  static constexpr float kPScale = 1.0f;       // unused
};
template <>
struct Fmt<true> {    // e4m3
  static constexpr int kSpans = 1;             // 128 bytes per row
  static constexpr int NS = 6;
  static constexpr int kK = 32;
  // lazy rescale by up to 2^kLazy: P <= 2^kLazy, so P is quantised as
  // P · kPScale with kPScale = 448 · 2^-kLazy (the e4m3 maximum is 448)
  static constexpr float kLazy = 2.0f;
  static constexpr float kPScale = 112.0f;
};

template <bool F8>
struct Layout {
  static constexpr int NS = Fmt<F8>::NS;
  static constexpr uint32_t kTile = kSpan * Fmt<F8>::kSpans;
  static constexpr int B_Q = 0, B_KF = 1, B_VF = B_KF + NS, B_KE = B_VF + NS, B_SF = B_KE + NS,
                       B_PR = B_SF + 2, B_OD = B_PR + 2, B_FIN = B_OD + 2, NBAR = B_FIN + 1;
  static constexpr uint32_t kBarOff = kTile * (1 + 2 * NS);
  static constexpr uint32_t kSlotOff = kBarOff + 8 * NBAR;   // tmem base, abort flag
  static constexpr uint32_t kMaskOff = kSlotOff + 16;
  static size_t smem_bytes(int nb) { return 1024 + kMaskOff + 4 * (size_t)((nb + 31) / 32 + 4); }
};

// Scales of the e4m3 operands (all null for bf16).
struct F8Scales {
  const float* q;       // [BH][nqb]
  const float* k;       // [BH][nb]
  const float* v;       // [BH][nb]
  const float* v_max;   // [BH]  max over the head's V blocks
  const float* kbar;    // [BH][ceil(nb/128)]  centroid key tiles
  const float* vbar;    // [BH][ceil(nb/128)]  centroid value tiles
};

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

// MMA issue from a converged warp: the whole MMA warp runs the issue loop
// (its descriptors and addresses are warp-uniform) and elect.sync picks the
// one lane that issues each tcgen05 instruction.  The same loop run by lane
// 0 alone issued its instructions much more slowly while the softmax warps
// kept the FMA pipes of its sub-partition busy (measured on B200: 7% of the
// whole kernel).
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
__device__ __forceinline__ void mma_ss_f8_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
               ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u) : "memory");
}
__device__ __forceinline__ void mma_ts_f8_w(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
               ::"r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u) : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint32_t bar) {
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}

// Instruction descriptor of kind::f8f6f4 with e4m3 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, int b_mn_major) {
  return (1u << 4) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// L2 prefetch of the Q tile and the first `ntiles` selected K/V tiles of
// the CTA one SM count further in launch order (grid x = query block,
// y = batch·head), the one most likely to take this SM next.
template <int kSpans>
__device__ __forceinline__ void prefetch_next_cta(const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                                  const CUtensorMap* tmV, const int32_t* block_idx, int nb,
                                                  int topk, int ntiles) {
  const uint32_t nl = blockIdx.y * gridDim.x + blockIdx.x + sm_count_reg();
  if (nl >= gridDim.x * gridDim.y) return;
  const int ni = (int)(nl % gridDim.x), nbh = (int)(nl / gridDim.x);
#pragma unroll
  for (int h = 0; h < kSpans; ++h) tma_prefetch_3d(tmQ, 64 * h, ni * TB, nbh);
  const int32_t* nsel = block_idx + ((size_t)nbh * nb + ni) * topk;
  for (int u = 0; u < ntiles && u < topk; ++u) {
    const int nr = nsel[u] * TB;
#pragma unroll
    for (int h = 0; h < kSpans; ++h) {
      tma_prefetch_3d(tmK, 64 * h, nr, nbh);
      tma_prefetch_3d(tmV, 64 * h, nr, nbh);
    }
  }
}

template <bool ZO, bool F8, bool FO>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
               const __grid_constant__ CUtensorMap tmVb, const __grid_constant__ CUtensorMap tmHb,
               const int32_t* __restrict__ block_idx, int nb, int topk, float scale2, F8Scales f8,
               __nv_bfloat16* __restrict__ O, int N, float* __restrict__ lse_out) {
  static_assert(!FO || (ZO && !F8), "the first-order tail extends the bf16 zero-order tail");
  // launched with programmatic stream serialization: the block indices and
  // statistics come from the previous launches on the stream
  pdl_wait();
  pdl_trigger();
  using L = Layout<F8>;
  constexpr int NS = L::NS;
  constexpr uint32_t kTile = L::kTile;
  constexpr int kSpans = Fmt<F8>::kSpans;
  constexpr int kK = Fmt<F8>::kK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int i = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlotOff + 4);
  uint32_t* selmask = reinterpret_cast<uint32_t*>(smem + L::kMaskOff);
  auto bar = [&](int k) { return sb + L::kBarOff + 8u * k; };

  const int nwords = (nb + 31) >> 5;
  const int ntail = (ZO && topk < nb) ? (nb + TB - 1) / TB : 0;
  const int T = topk + ntail;
  // first-order tail: one more S MMA, S' = Q H̄ (tile T, K slot only), into
  // the S columns of stream T % 2 once that stream's last P has been read
  const bool fo = FO && ntail > 0;
  const int Tx = T + (fo ? 1 : 0);
  const int32_t* sel = block_idx + ((size_t)bh * nb + i) * topk;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_Q), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::B_KF + s), 1);
      mbar_init(bar(L::B_VF + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_SF + s), 1);
      mbar_init(bar(L::B_PR + s), 128);
      mbar_init(bar(L::B_OD + s), 1);
    }
    mbar_init(bar(L::B_FIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // selection bitmap, padded with 4 zero words so a tile's 4 words never run past it
  for (int w = threadIdx.x; w < nwords + 4; w += kTcThreads) selmask[w] = 0u;
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // The producer and MMA warps start at once; the softmax warps fill the
  // bitmap (read only by them, at the centroid tiles) under their own barrier.

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
      if (FO) prefetch_tmap(&tmHb);
      mbar_expect_tx(bar(L::B_Q), kTile);
#pragma unroll
      for (int h = 0; h < kSpans; ++h) tma_load_3d(sb + h * kSpan, &tmQ, 64 * h, i * TB, bh, bar(L::B_Q));
      int issued = 0;
      for (int t = 0; t < Tx; ++t) {
        const int s = t % NS;
        if (t >= NS && !mbar_wait(bar(L::B_KE + s), ((t / NS) - 1) & 1, abort_flag)) break;
        if (FO && t == T) {
          // H̄ᵀ of this head [d rows = output channel e][d cols = c] as a K tile
          const uint32_t ka = sb + kTile * (1 + 2 * s);
          mbar_expect_tx(bar(L::B_KF + s), kTile);
#pragma unroll
          for (int h = 0; h < kSpans; ++h) tma_load_3d(ka + h * kSpan, &tmHb, 64 * h, 0, bh, bar(L::B_KF + s));
          issued = t + 1;
          break;
        }
        const bool exact = t < topk;
        const CUtensorMap* mk = exact ? &tmK : &tmKb;
        const CUtensorMap* mv = exact ? &tmV : &tmVb;
        const int row = exact ? sel[t] * TB : (t - topk) * TB;
        const uint32_t ka = sb + kTile * (1 + 2 * s), va = ka + kTile;
        mbar_expect_tx(bar(L::B_KF + s), kTile);
#pragma unroll
        for (int h = 0; h < kSpans; ++h) tma_load_3d(ka + h * kSpan, mk, 64 * h, row, bh, bar(L::B_KF + s));
        mbar_expect_tx(bar(L::B_VF + s), kTile);
#pragma unroll
        for (int h = 0; h < kSpans; ++h) tma_load_3d(va + h * kSpan, mv, 64 * h, row, bh, bar(L::B_VF + s));
        issued = t + 1;
      }
      // every load of this CTA is issued: warm L2 for the CTA that most
      // likely takes this SM next, so its prologue reads L2, not HBM
      prefetch_next_cta<kSpans>(&tmQ, &tmK, &tmV, block_idx, nb, topk, NS);
      if (*abort_flag) {
        // let the loads already in flight land before the CTA goes away
        wait_bounded(bar(L::B_Q), 0);
        for (int t = issued > NS ? issued - NS : 0; t < issued; ++t) {
          wait_bounded(bar(L::B_KF + t % NS), (t / NS) & 1);
          if (t < T) wait_bounded(bar(L::B_VF + t % NS), (t / NS) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kProducerRegs>();
    if (T > 0) {
      constexpr uint32_t idS = F8 ? idesc_e4m3_f32(TB, TB, 0) : idesc_bf16_f32(TB, TB, 0, 0);
      constexpr uint32_t idO = F8 ? idesc_e4m3_f32(TB, TD, 1) : idesc_bf16_f32(TB, TD, 0, 1);
      // descriptors are built once per operand tile and advanced per K step
      const uint64_t qd0 = desc_sw128(sb, 16, 1024);
      // S(t) = Q K_tᵀ into the S columns of stream t % 2
      auto issue_s = [&](int t) -> bool {
        const int s = t % NS;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_KF + s), (t / NS) & 1, abort_flag))) return false;
        tc_fence_after();
        const uint64_t kd0 = desc_sw128(sb + kTile * (1 + 2 * s), 16, 1024);
        const uint32_t d = tbase + (uint32_t)(t & 1) * TB;
#pragma unroll
        for (int k = 0; k < TD / kK; ++k) {
          // K step k: 32 bytes further along the row, next span every 4 steps
          const uint32_t koff = (k >> 2) * kSpan + (k & 3) * 32;
          const uint64_t a = desc_adv(qd0, koff), b = desc_adv(kd0, koff);
          if (F8) mma_ss_f8_w(d, a, b, idS, k > 0);
          else mma_ss_w(d, a, b, idS, k > 0);
        }
        mma_commit_w(bar(L::B_SF + (t & 1)));
        return true;
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_Q), 0, abort_flag));
      if (ok) ok = issue_s(0);
      if (ok && Tx > 1) ok = issue_s(1);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t & 1, u = t >> 1, su = t % NS;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_PR + st), u & 1, abort_flag))) break;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_VF + su), (t / NS) & 1, abort_flag))) break;
        tc_fence_after();
        const uint64_t vd0 = desc_sw128(sb + kTile * (2 + 2 * su), kSpan, 1024);
        const uint32_t pa = tbase + (uint32_t)st * TB;
        const uint32_t od = tbase + kColO + (uint32_t)st * TD;
#pragma unroll
        for (int k = 0; k < TB / kK; ++k) {
          // K step k: kK keys = kK rows of 128 bytes further into V; 8 TMEM columns of P
          const uint64_t b = desc_adv(vd0, k * kK * 128);
          if (F8) mma_ts_f8_w(od, pa + k * 8, b, idO, (u > 0 || k > 0));
          else mma_ts_w(od, pa + k * 8, b, idO, (u > 0 || k > 0));
        }
        mma_commit_w(bar(L::B_KE + su));
        mma_commit_w(bar(L::B_OD + st));
        if (t + 2 < Tx && !issue_s(t + 2)) break;
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit_w(bar(L::B_FIN));
      wait_bounded(bar(L::B_FIN), 0);
    }
  } else if (warp >= 8) {
    regs_dec<kProducerRegs>();                  // idle warps of the producer warpgroup
  } else {
    // ------------------------------------------------------------ softmax
    regs_inc<kSoftmaxRegs>();
    for (int s = threadIdx.x; s < topk; s += 256) {
      const int j = sel[s];
      atomicOr(&selmask[j >> 5], 1u << (j & 31));
    }
    named_bar_softmax();                        // the bitmap is complete
    const int st = warp >> 2;                   // stream
    const int wq = warp & 3;                    // TMEM lane quarter
    const int r = wq * 32 + lane;               // query row
    const uint32_t lrow = tbase + ((uint32_t)(wq * 32) << 16);
    const uint32_t s_col = (uint32_t)st * TB;
    const uint32_t o_col = kColO + (uint32_t)st * TD;
    const int U = T > st ? (T - st + 1) / 2 : 0;   // tiles of this stream
    // e4m3: the head's largest V scale and this query block's Q scale
    float vmax = 1.f, qs = 1.f;
    if (F8) {
      const int ntiles = (nb + TB - 1) / TB;
      vmax = f8.v_max[bh];
      if (ZO)
        for (int c = 0; c < ntiles; ++c) vmax = fmaxf(vmax, f8.vbar[(size_t)bh * ntiles + c]);
      qs = f8.q[(size_t)bh * nb + i];
    }
    const float inv_vmax = 1.0f / vmax;
    // e4m3: the K and V scales of tile t (the block index, then the block's
    // scales: two dependent loads), fetched one tile of this stream ahead so
    // that they arrive during the previous tile's softmax
    auto tile_scales = [&](int t, float& ks, float& vs) {
      if (!F8 || t >= T) return;
      const int ntiles = (nb + TB - 1) / TB;
      if (t >= topk) {
        ks = f8.kbar[(size_t)bh * ntiles + (t - topk)];
        vs = f8.vbar[(size_t)bh * ntiles + (t - topk)];
      } else {
        const int j = sel[t];
        ks = f8.k[(size_t)bh * nb + j];
        vs = f8.v[(size_t)bh * nb + j];
      }
    };
    float ks_cur = 1.f, vs_cur = 1.f;
    if (F8 && U > 0) tile_scales(st, ks_cur, vs_cur);
    float m_used = -INFINITY, l = 0.f;
    float lc = 0.f;   // first-order: the centroid tiles' share of l
    bool ok = true;
    for (int u = 0; u < U; ++u) {
      const int t = 2 * u + st;
      float ks_nxt = 1.f, vs_nxt = 1.f;
      if (F8) tile_scales(t + 2, ks_nxt, vs_nxt);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SF + st), u & 1, abort_flag))) {
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
      float tscale = scale2, pscale = 1.f;
      if (F8) {
        tscale = scale2 * qs * ks_cur;
        pscale = Fmt<true>::kPScale * vs_cur * inv_vmax;
        ks_cur = ks_nxt;
        vs_cur = vs_nxt;
      }
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
      const float m_tile = mx == -INFINITY ? -INFINITY : fmaf(mx, tscale, bias);
      const float m_new = fmaxf(m_used, m_tile);
      const bool need = m_new > m_used + Fmt<F8>::kLazy;
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
      const float sc2 = live ? tscale : 0.f, ng = live ? neg : -INFINITY;   // dead row: p = 0
      float sum_scale = 1.f;
      if (F8) {
        // the exponentials come out already scaled for the e4m3 store,
        // p' = p·pscale = 2^(a + log2 pscale), and the row sum takes Σp'/pscale.
        // pscale is floored at 2^-100: below it every p' rounds to e4m3 zero
        // either way, and p' stays a normal fp32 number for the sum.
        const float pse = fmaxf(pscale, 0x1p-100f);
        const float ngp = ng + __log2f(pse);
        sum_scale = 1.0f / pse;
#pragma unroll
        for (int n = 0; n < TB / 4; ++n) {
          float a0, a1, a2, a3;
          ffma2(a0, a1, __uint_as_float(v[4 * n]), __uint_as_float(v[4 * n + 1]), sc2, sc2, ngp, ngp);
          ffma2(a2, a3, __uint_as_float(v[4 * n + 2]), __uint_as_float(v[4 * n + 3]), sc2, sc2, ngp, ngp);
          float p0, p1, p2, p3;
          if ((kExpFmaF8 >> (n & 7)) & 1u) {
            exp2_poly2(a0, a1, p0, p1);
            exp2_poly2(a2, a3, p2, p3);
          } else {
            p0 = fast_exp2(a0); p1 = fast_exp2(a1); p2 = fast_exp2(a2); p3 = fast_exp2(a3);
          }
          fadd2(sm8[2 * (n & 3)], sm8[2 * (n & 3) + 1], p0 + p2, p1 + p3);
          v[n] = pack_e4m3x4(p0, p1, p2, p3);
        }
      } else {
#pragma unroll
        for (int n = 0; n < TB / 2; ++n) {
          float a0, a1;
          ffma2(a0, a1, __uint_as_float(v[2 * n]), __uint_as_float(v[2 * n + 1]), sc2, sc2, ng, ng);
          float p0, p1;
          if ((kExpFma >> (n & 7)) & 1u) exp2_poly2(a0, a1, p0, p1);
          else { p0 = fast_exp2(a0); p1 = fast_exp2(a1); }
          fadd2(sm8[2 * (n & 3)], sm8[2 * (n & 3) + 1], p0, p1);
          v[n] = pack_bf16(p0, p1);
        }
      }
      const float sum =
          (((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]))) * sum_scale;
      l = l * factor + sum;
      if (FO) lc = lc * factor + (centroid ? sum : 0.f);
      tmem_st32(lrow + s_col, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      if (!F8) tmem_st32(lrow + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_st();
      if (u >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_OD + st), (u - 1) & 1, abort_flag))) {
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
      mbar_arrive(bar(L::B_PR + st));
    }
    if (ok && U > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_OD + st), (U - 1) & 1, abort_flag));
    // both groups past their last PV: every MMA that reads Q has completed,
    // so the Q tile's shared memory can carry the (max, sum) exchange
    named_bar_softmax();
    constexpr int kEx = FO ? 384 : 256;
    float* ex = reinterpret_cast<float*>(smem);   // [2 streams][2 or 3][128]
    ex[st * kEx + r] = (U > 0) ? m_used : -INFINITY;
    ex[st * kEx + 128 + r] = l;
    if (FO) ex[st * kEx + 256 + r] = lc;
    named_bar_softmax();
    const float m0 = ex[r], l0 = ex[128 + r], m1 = ex[kEx + r], l1 = ex[kEx + 128 + r];
    const int U0 = T > 0 ? (T + 1) / 2 : 0, U1 = T > 1 ? T / 2 : 0;
    const float M = fmaxf(m0, m1);
    const float f0 = (U0 > 0 && m0 != -INFINITY) ? fast_exp2(m0 - M) : 0.f;
    const float f1 = (U1 > 0 && m1 != -INFINITY) ? fast_exp2(m1 - M) : 0.f;
    const float L_ = l0 * f0 + l1 * f1;
    // e4m3: O accumulated Σ P σ_V V̂ · kPScale / σ_Vmax
    const float inv = L_ > 0.f ? (F8 ? vmax / Fmt<true>::kPScale : 1.0f) / L_ : 0.f;
    // the row's log-sum-exp of its logits in log2 units (for the backward)
    if (lse_out && st == 0) lse_out[(size_t)bh * N + (size_t)i * TB + r] = L_ > 0.f ? M + log2f(L_) : INFINITY;
    // first-order: + Λ_t (s q_t)ᵀ H̄ with Λ_t = Σ_U e^{s q·k̄_j} on the merged
    // maximum (the centroid tiles' sums carry the factor 128 = e^{ln 128})
    float wfo = 0.f;
    const uint32_t sp_col = (uint32_t)(T & 1) * TB + 64u * st;
    if (FO && fo) {
      const float lc0 = ex[256 + r], lc1 = ex[kEx + 256 + r];
      wfo = scale2 * 0.6931471805599453f * (1.0f / 128.0f) * (lc0 * f0 + lc1 * f1);
      // S' = Q H̄ is the (U_b + 1)-th completion of stream b = T % 2's S barrier
      const int Ub = (T & 1) ? U1 : U0;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_SF + (T & 1)), Ub & 1, abort_flag));
    }
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
        uint32_t sp[32];
        if (FO && fo) tmem_ld32(lrow + sp_col + 32 * c, sp);
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
          for (int e = 0; e < 8; ++e) {
            float acc = __uint_as_float(a[8 * q + e]) * f0 + __uint_as_float(b[8 * q + e]) * f1;
            if (FO && fo) acc = fmaf(wfo, __uint_as_float(sp[8 * q + e]), acc);
            y[e] = acc * inv;
          }
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

// 3-D tensor map [outer][rows][cols] (cols innermost) with a box of
// {128 bytes, 128 rows, 1} and 128-byte swizzle; elem = 2 (bf16) or 1 (e4m3).
bool make_tmap_3d(CUtensorMap* map, const void* base, int elem, uint64_t cols, uint64_t rows, uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * elem, cols * rows * elem};
  cuuint32_t box[3] = {128u / (cuuint32_t)elem, (cuuint32_t)TB, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
            const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool F8>
sa_status launch_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mkb,
                    const CUtensorMap& mvb, const CUtensorMap& mhb, bool zo, bool fo, const sa_shape& s,
                    const int32_t* block_idx, int topk, float scale, const F8Scales& f8, void* O,
                    float* lse_out, cudaStream_t stream) {
  const int nb = s.N / TB;
  const size_t smem = Layout<F8>::smem_bytes(nb);
  auto kern = zo ? attn_tc_kernel<true, F8, false> : attn_tc_kernel<false, F8, false>;
  if constexpr (!F8) {
    if (fo) kern = attn_tc_kernel<true, false, true>;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(attn_tc_kernel)");
  dim3 grid(nb, (unsigned)((uint64_t)s.B * s.H));
  const cudaError_t le = launch_pdl(kern, grid, dim3(kTcThreads), smem, stream, mq, mk, mv, mkb, mvb, mhb, block_idx,
                                    nb, topk, scale * kLog2e, f8, static_cast<__nv_bfloat16*>(O), s.N, lse_out);
  if (le != cudaSuccess) return fail(SA_ERR_CUDA, std::string("attn_tc_kernel: ") + cudaGetErrorString(le));
  return launch_status("attn_tc_kernel");
}

// ---------------------------------------------------------------- linear mix
// SLA2 §2A mixture O = α⊙O_s + (1−α)⊙O_l on the tensor cores.  O_s is the
// exact softmax over the selected blocks; O_l is the ReLU linear attention
// (SALAD §2) over the unselected blocks in SPLA §2.2's subtraction form:
//   O_l = relu(q)ᵀ (H_tot − A_i) / (relu(q)·(z_tot − ζ_i) + eps),
//   A_i = Σ_{j∈S_i} relu(K_j)ᵀ V_j,  ζ_i = Σ_{j∈S_i} z_j,
// with A_i accumulated by the MMA warp from the K/V tiles already in shared
// memory (unselected blocks are never read).  TMEM (512 columns): S0, S1 (the
// double-buffered score tile), O (the softmax accumulator), A (A_i, d×d).
// Warps 0-3 run the softmax of every tile; warps 4-7 apply ReLU in place to
// each K tile once its S MMA has finished with it, then build the epilogue's
// operands (relu(Q) in place, D = H_tot − A_i as a bf16 tile, ζ_i); warp 8 is
// the TMA producer, warp 9 the MMA issuer.
struct LinLayout {
  static constexpr int NS = 3;
  static constexpr uint32_t kTile = 2 * kSpan;
  static constexpr int B_Q = 0, B_KF = 1, B_VF = B_KF + NS, B_KE = B_VF + NS, B_SF = B_KE + NS,
                       B_PR = B_SF + 2, B_RL = B_PR + 2, B_OD = B_RL + 2, B_LAST = B_OD + 1,
                       B_EPI_IN = B_LAST + 1, B_EPI = B_EPI_IN + 1, B_FIN = B_EPI + 1, NBAR = B_FIN + 1;
  static constexpr uint32_t kBarOff = kTile * (1 + 2 * NS);
  static constexpr uint32_t kSlotOff = kBarOff + 8 * NBAR;   // tmem base, abort flag
  static constexpr uint32_t kZetaOff = kSlotOff + 16;        // ζ_i: TD floats
  static constexpr uint32_t kEnd = kZetaOff + TD * 4;
  static size_t smem_bytes() { return 1024 + kEnd; }
};
constexpr uint32_t kColA = 384;
// register split: 128 softmax threads x 216 + 128 ReLU threads x 96 + 128
// producer threads x 56 = 47104.  The producer warpgroup (TMA lane, MMA
// issuer) keeps 56 registers here: at 40 the kernel spilled (280 bytes of
// spill loads) and ran 3% slower (7.65 against 7.40 ms on sla2_mix, same box)
constexpr int kReluRegs = 96, kLinProducerRegs = 56;

__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_linmix_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ block_idx, int nb,
                      int topk, float scale2, const float* __restrict__ alpha, const float* __restrict__ zrelu,
                      const float* __restrict__ htot, const float* __restrict__ ztot, int H,
                      __nv_bfloat16* __restrict__ O, int N) {
  pdl_wait();                                   // the block indices and statistics of the previous launches
  pdl_trigger();
  using L = LinLayout;
  constexpr int NS = L::NS;
  constexpr uint32_t kTile = L::kTile;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int i = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlotOff + 4);
  float* zeta = reinterpret_cast<float*>(smem + L::kZetaOff);
  auto bar = [&](int k) { return sb + L::kBarOff + 8u * k; };
  const int T = topk;
  const int32_t* sel = block_idx + ((size_t)bh * nb + i) * topk;

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_Q), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::B_KF + s), 1);
      mbar_init(bar(L::B_VF + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::B_SF + s), 1);
      mbar_init(bar(L::B_PR + s), 128);
      mbar_init(bar(L::B_RL + s), 128);
    }
    mbar_init(bar(L::B_OD), 1);
    mbar_init(bar(L::B_LAST), 1);
    mbar_init(bar(L::B_EPI_IN), 256);
    mbar_init(bar(L::B_EPI), 1);
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
    regs_dec<kLinProducerRegs>();
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(bar(L::B_Q), kTile);
      tma_load_3d(sb, &tmQ, 0, i * TB, bh, bar(L::B_Q));
      tma_load_3d(sb + kSpan, &tmQ, 64, i * TB, bh, bar(L::B_Q));
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % NS;
        if (t >= NS && !mbar_wait(bar(L::B_KE + s), ((t / NS) - 1) & 1, abort_flag)) break;
        const int row = sel[t] * TB;
        const uint32_t ka = sb + kTile * (1 + 2 * s), va = ka + kTile;
        mbar_expect_tx(bar(L::B_KF + s), kTile);
        tma_load_3d(ka, &tmK, 0, row, bh, bar(L::B_KF + s));
        tma_load_3d(ka + kSpan, &tmK, 64, row, bh, bar(L::B_KF + s));
        mbar_expect_tx(bar(L::B_VF + s), kTile);
        tma_load_3d(va, &tmV, 0, row, bh, bar(L::B_VF + s));
        tma_load_3d(va + kSpan, &tmV, 64, row, bh, bar(L::B_VF + s));
        issued = t + 1;
      }
      prefetch_next_cta<2>(&tmQ, &tmK, &tmV, block_idx, nb, topk, NS);
      if (*abort_flag) {
        wait_bounded(bar(L::B_Q), 0);
        for (int t = issued > NS ? issued - NS : 0; t < issued; ++t) {
          wait_bounded(bar(L::B_KF + t % NS), (t / NS) & 1);
          wait_bounded(bar(L::B_VF + t % NS), (t / NS) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kLinProducerRegs>();
    {   // the whole warp runs the loop; elect.sync picks the issuing lane
      constexpr uint32_t idS = idesc_bf16_f32(TB, TB, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(TB, TD, 0, 1);
      constexpr uint32_t idA = idesc_bf16_f32(TD, TD, 1, 1);   // relu(K)ᵀ (MN-major) · V (MN-major)
      const uint32_t colO = tbase + 256, colA = tbase + kColA;
      const uint64_t qd0 = desc_sw128(sb, 16, 1024);
      auto issue_s = [&](int t) -> bool {
        const int s = t % NS;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_KF + s), (t / NS) & 1, abort_flag))) return false;
        tc_fence_after();
        const uint64_t kd0 = desc_sw128(sb + kTile * (1 + 2 * s), 16, 1024);
        const uint32_t d = tbase + (uint32_t)(t & 1) * TB;
#pragma unroll
        for (int k = 0; k < TD / 16; ++k) {
          const uint32_t koff = (k >> 2) * kSpan + (k & 3) * 32;
          mma_ss_w(d, desc_adv(qd0, koff), desc_adv(kd0, koff), idS, k > 0);
        }
        mma_commit_w(bar(L::B_SF + (t & 1)));
        return true;
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar(L::B_Q), 0, abort_flag));
      if (ok && T > 0) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int t = 0; ok && t < T; ++t) {
        const int su = t % NS, b2 = t & 1;
        const uint64_t kd0 = desc_sw128(sb + kTile * (1 + 2 * su), kSpan, 1024);
        const uint64_t vd0 = desc_sw128(sb + kTile * (2 + 2 * su), kSpan, 1024);
        // A_i += relu(K_t)ᵀ V_t once warps 4-7 have applied the ReLU
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_RL + b2), (t >> 1) & 1, abort_flag))) break;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_VF + su), (t / NS) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < TB / 16; ++k)
          mma_ss_w(colA, desc_adv(kd0, k * 16 * 128), desc_adv(vd0, k * 16 * 128), idA, (t > 0 || k > 0));
        // O += P_t V_t
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_PR + b2), (t >> 1) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < TB / 16; ++k)
          mma_ts_w(colO, tbase + (uint32_t)b2 * TB + k * 8, desc_adv(vd0, k * 16 * 128), idO, (t > 0 || k > 0));
        mma_commit_w(bar(L::B_KE + su));
        mma_commit_w(bar(L::B_OD));
        if (t + 2 < T && !issue_s(t + 2)) break;
      }
      mma_commit_w(bar(L::B_LAST));   // every MMA of the tile loop (or none) has completed
      // epilogue: S0 = relu(Q) · (H_tot − A_i), operands prepared by warps 0-7
      if (__all_sync(0xffffffffu, ok && mbar_wait(bar(L::B_EPI_IN), 0, abort_flag))) {
        tc_fence_after();
        const uint32_t dbase = sb + kTile;   // D tile in stage 0's K slot
#pragma unroll
        for (int k = 0; k < TD / 16; ++k) {
          const uint32_t koff = (k >> 2) * kSpan + (k & 3) * 32;
          mma_ss_w(tbase, desc_sw128(sb + koff, 16, 1024), desc_sw128(dbase + k * 16 * 128, kSpan, 1024),
                   idO, k > 0);
        }
        mma_commit_w(bar(L::B_EPI));
      }
      mma_commit_w(bar(L::B_FIN));
      wait_bounded(bar(L::B_FIN), 0);
    }
  } else if (warp >= 8) {
    regs_dec<kLinProducerRegs>();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ ReLU warps
    regs_dec<kReluRegs>();
    const int tr = threadIdx.x - 128;          // 0..127
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SF + (t & 1)), (t >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      // the S MMA has read K_t: replace it by relu(K_t) in place (layout-free)
      uint4* kt = reinterpret_cast<uint4*>(smem + kTile * (1 + 2 * (t % NS)));
      const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
#pragma unroll 4
      for (int x = tr; x < (int)(kTile / 16); x += 128) {
        uint4 u = kt[x];
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __hmax2(h[e], zero);
        kt[x] = u;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(bar(L::B_RL + (t & 1)));
    }
    // ζ_i = Σ_{j∈S_i} z_j (channel tr)
    float z = 0.f;
    for (int s2 = 0; s2 < T; ++s2) z += zrelu[((size_t)bh * nb + sel[s2]) * TD + tr];
    zeta[tr] = z;
    // after the last MMA reading Q: relu(Q) in place
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(L::B_LAST), 0, abort_flag));
    if (ok) {
      uint4* qt = reinterpret_cast<uint4*>(smem);
      const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
      for (int x = tr; x < (int)(kTile / 16); x += 128) {
        uint4 u = qt[x];
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __hmax2(h[e], zero);
        qt[x] = u;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    named_bar_softmax();          // zeta visible to warps 0-3
    mbar_arrive(bar(L::B_EPI_IN));
  } else {
    // ------------------------------------------------------------ softmax
    regs_inc<kSoftmaxRegs>();
    const int r = warp * 32 + lane;
    const uint32_t lrow = tbase + ((uint32_t)(warp * 32) << 16);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int b2 = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_SF + b2), (t >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lrow + b2 * TB + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
      tmem_wait_ld();
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
      for (int n = 0; n < TB / 2; ++n)
        mx8[n & 7] = fmax3(mx8[n & 7], __uint_as_float(v[2 * n]), __uint_as_float(v[2 * n + 1]));
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                             fmaxf(mx8[6], mx8[7]));
      const float m_tile = mx * scale2;
      const float m_new = fmaxf(m_used, m_tile);
      const bool need = m_new > m_used + Fmt<false>::kLazy;
      float factor = 1.f;
      if (need) {
        factor = fast_exp2(m_used - m_new);
        m_used = m_new;
      }
      const float neg = -m_used;
      float sm8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) sm8[k] = 0.f;
#pragma unroll
      for (int n = 0; n < TB / 2; ++n) {
        float a0, a1;
        ffma2(a0, a1, __uint_as_float(v[2 * n]), __uint_as_float(v[2 * n + 1]), scale2, scale2, neg, neg);
        const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
        fadd2(sm8[2 * (n & 3)], sm8[2 * (n & 3) + 1], p0, p1);
        v[n] = pack_bf16(p0, p1);
      }
      l = l * factor + (((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7])));
      tmem_st32(lrow + b2 * TB, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_st32(lrow + b2 * TB + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_st();
      if (t >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_OD), (t - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (__any_sync(0xffffffffu, need)) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(lrow + 256 + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(lrow + 256 + 32 * c, o);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(bar(L::B_PR + b2));
    }
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(L::B_LAST), 0, abort_flag));
    // D = H_tot − A_i (row c = this thread's TMEM lane) as a bf16 MN-major tile
    // in stage 0's K slot: span e/64, row c, 16-byte chunk (e%64)/8 xor (c%8)
    if (ok) {
      tc_fence_after();
      const float* hrow = htot + ((size_t)bh * TD + r) * TD;
      uint8_t* dt = smem + kTile;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t a[32];
        if (T > 0) {
          tmem_ld32(lrow + kColA + 32 * c, a);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = 0u;
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int e0 = 32 * c + 8 * q4;                  // first of 8 output channels
          uint4 w;
          w.x = pack_bf16(hrow[e0 + 0] - __uint_as_float(a[8 * q4 + 0]), hrow[e0 + 1] - __uint_as_float(a[8 * q4 + 1]));
          w.y = pack_bf16(hrow[e0 + 2] - __uint_as_float(a[8 * q4 + 2]), hrow[e0 + 3] - __uint_as_float(a[8 * q4 + 3]));
          w.z = pack_bf16(hrow[e0 + 4] - __uint_as_float(a[8 * q4 + 4]), hrow[e0 + 5] - __uint_as_float(a[8 * q4 + 5]));
          w.w = pack_bf16(hrow[e0 + 6] - __uint_as_float(a[8 * q4 + 6]), hrow[e0 + 7] - __uint_as_float(a[8 * q4 + 7]));
          const int span = e0 >> 6, chunk = (e0 & 63) >> 3;
          *reinterpret_cast<uint4*>(dt + span * kSpan + r * 128 + ((chunk ^ (r & 7)) << 4)) = w;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    named_bar_softmax();          // zeta ready (warps 4-7)
    mbar_arrive(bar(L::B_EPI_IN));
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(L::B_EPI), 0, abort_flag)) && !*abort_flag;
    if (ok) {
      tc_fence_after();
      // relu(q_r)·(z_tot − ζ_i) from this row of the (now relu'd) Q tile
      float den = kLinearEps;
      const float* zt = ztot + (size_t)bh * TD;
#pragma unroll 4
      for (int ch = 0; ch < 16; ++ch) {            // 16-byte chunks of the 128 channels
        const int span = ch >> 3, cc = ch & 7;
        const uint4 u = *reinterpret_cast<const uint4*>(smem + span * kSpan + r * 128 + ((cc ^ (r & 7)) << 4));
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          const int c0 = ch * 8 + 2 * e;
          den = fmaf(f.x, zt[c0] - zeta[c0], den);
          den = fmaf(f.y, zt[c0 + 1] - zeta[c0 + 1], den);
        }
      }
      const bool u_empty = (topk == nb);            // no unselected block: O_l = 0
      const float inv_den = u_empty ? 0.f : 1.0f / den;
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const float* al = alpha + (size_t)(bh % H) * TD;
      uint4* orow = reinterpret_cast<uint4*>(O + ((size_t)bh * N + (size_t)i * TB + r) * TD);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t os[32], ol[32];
        if (T > 0) tmem_ld32(lrow + 256 + 32 * c, os);
        tmem_ld32(lrow + 32 * c, ol);
        tmem_wait_ld();
        if (T == 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) os[e] = 0u;
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ee = 32 * c + 8 * q4 + e;
            const float a = al[ee];
            y[e] = a * __uint_as_float(os[8 * q4 + e]) * inv_l + (1.0f - a) * __uint_as_float(ol[8 * q4 + e]) * inv_den;
          }
          uint4 w;
          w.x = pack_bf16(y[0], y[1]);
          w.y = pack_bf16(y[2], y[3]);
          w.z = pack_bf16(y[4], y[5]);
          w.w = pack_bf16(y[6], y[7]);
          orow[4 * c + q4] = w;
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

// ---------------------------------------------------------------- H_tot, H̄
// d×d outer-product sums Σ_n f(k_n) v_nᵀ of one head on the tensor cores:
//   kKvRelu:   f = relu, H_tot (the total of SLA2's ReLU linear branch,
//              SALAD §2);
//   kKvCentre: f(k_n) = k_n − k̄_j with k̄_j the centroid of the 128-token
//              block that holds n, each chunk's sum scaled by oscale (1/nb):
//              PISA's mean first-order statistic H̄ (§2).  The MMAs
//              accumulate the raw Kᵀ V of the chunk (bf16 products are exact
//              in fp32) and the epilogue subtracts Σ_j k̄_j vsum_jᵀ over the
//              chunk's blocks in fp32, which equals Σ_j Σ_n (k_n − k̄_j) v_nᵀ
//              without rounding the deviations to bf16;
//   kKvExp:    f = φ = phi_exp rounded to bf16: SPLA's residual linear state
//              Σ_n φ(k_n) v_nᵀ over all tokens (§2.2).
// A CTA takes a chunk of 128-token tiles of one head, warps 2-5 apply f in
// place to each K tile (relu, exp), warp 1 accumulates f(K)ᵀ V in TMEM
// (MN-major × MN-major MMA), and the chunk's d×d sum is added to `out`
// with vector atomics.  Warp 0 is the TMA producer.
constexpr int kHtThreads = 192;
constexpr int kHtMinTiles = 4;        // fewest tiles (of 128 tokens) per CTA
struct HtLayout {
  static constexpr int NS = 3;
  static constexpr uint32_t kTile = 2 * kSpan;
  static constexpr int B_KF = 0, B_VF = B_KF + NS, B_KE = B_VF + NS, B_RL = B_KE + NS, B_DONE = B_RL + NS,
                       NBAR = B_DONE + 1;
  static constexpr uint32_t kBarOff = 2 * kTile * NS;
  static constexpr uint32_t kSlotOff = kBarOff + 8 * NBAR;
  static size_t smem_bytes() { return 1024 + kSlotOff + 16; }
};

__global__ void __launch_bounds__(kHtThreads, 1)
htot_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int N,
               int tiles_per_cta, int feature, const float* __restrict__ kmean, const float* __restrict__ vsum,
               float oscale, float* __restrict__ htot) {
  using L = HtLayout;
  constexpr int NS = L::NS;
  constexpr uint32_t kTile = L::kTile;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlotOff + 4);
  auto bar = [&](int k) { return sb + L::kBarOff + 8u * k; };
  const int ntile_head = N / TB;
  const int t0 = chunk * tiles_per_cta;
  const int T = min(tiles_per_cta, ntile_head - t0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(L::B_KF + s), 1);
      mbar_init(bar(L::B_VF + s), 1);
      mbar_init(bar(L::B_KE + s), 1);
      mbar_init(bar(L::B_RL + s), 128);
    }
    mbar_init(bar(L::B_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % NS;
        if (t >= NS && !mbar_wait(bar(L::B_KE + s), ((t / NS) - 1) & 1, abort_flag)) break;
        const int row = (t0 + t) * TB;
        const uint32_t ka = sb + 2 * kTile * s, va = ka + kTile;
        mbar_expect_tx(bar(L::B_KF + s), kTile);
        tma_load_3d(ka, &tmK, 0, row, bh, bar(L::B_KF + s));
        tma_load_3d(ka + kSpan, &tmK, 64, row, bh, bar(L::B_KF + s));
        mbar_expect_tx(bar(L::B_VF + s), kTile);
        tma_load_3d(va, &tmV, 0, row, bh, bar(L::B_VF + s));
        tma_load_3d(va + kSpan, &tmV, 64, row, bh, bar(L::B_VF + s));
        issued = t + 1;
      }
      if (*abort_flag)
        for (int t = issued > NS ? issued - NS : 0; t < issued; ++t) {
          wait_bounded(bar(L::B_KF + t % NS), (t / NS) & 1);
          wait_bounded(bar(L::B_VF + t % NS), (t / NS) & 1);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idA = idesc_bf16_f32(TD, TD, 1, 1);
      for (int t = 0; t < T; ++t) {
        const int s = t % NS;
        if (!mbar_wait(bar(L::B_RL + s), (t / NS) & 1, abort_flag)) break;
        if (!mbar_wait(bar(L::B_VF + s), (t / NS) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t ka = sb + 2 * kTile * s, va = ka + kTile;
#pragma unroll
        for (int k = 0; k < TB / 16; ++k)
          mma_ss(tbase, desc_sw128(ka + k * 16 * 128, kSpan, 1024), desc_sw128(va + k * 16 * 128, kSpan, 1024),
                 idA, (t > 0 || k > 0));
        mma_commit(bar(L::B_KE + s));
      }
      mma_commit(bar(L::B_DONE));
      wait_bounded(bar(L::B_DONE), 0);
    }
  } else {
    // warps 2-5: ReLU of each K tile (H_tot), then the epilogue (TMEM lane
    // quarter w % 4)
    const int tr = threadIdx.x - 64;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::B_KF + s), (t / NS) & 1, abort_flag))) {
        ok = false;
        break;
      }
      if (feature == kKvRelu) {
        uint4* kt = reinterpret_cast<uint4*>(smem + 2 * kTile * s);
        const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
#pragma unroll 4
        for (int x = tr; x < (int)(kTile / 16); x += 128) {
          uint4 u = kt[x];
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) h[e] = __hmax2(h[e], zero);
          kt[x] = u;
        }
      } else if (feature == kKvExp) {
        uint4* kt = reinterpret_cast<uint4*>(smem + 2 * kTile * s);
#pragma unroll 4
        for (int x = tr; x < (int)(kTile / 16); x += 128) {
          uint4 u = kt[x];
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            h[e] = __floats2bfloat162_rn(phi_exp(f.x), phi_exp(f.y));
          }
          kt[x] = u;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(bar(L::B_RL + s));
    }
    ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(L::B_DONE), 0, abort_flag)) && !*abort_flag;
    if (ok && T > 0) {
      tc_fence_after();
      const int wq = warp & 3;
      const int c = wq * 32 + lane;                  // row c of relu(K)ᵀ V
      const uint32_t lrow = tbase + ((uint32_t)(wq * 32) << 16);
      float4* hrow = reinterpret_cast<float4*>(htot + ((size_t)bh * TD + c) * TD);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t a[32];
        tmem_ld32(lrow + 32 * cc, a);
        tmem_wait_ld();
        if (feature == kKvCentre) {
          // − Σ_j k̄_j[c] vsum_j[e] over the chunk's blocks
          float* f = reinterpret_cast<float*>(a);
          for (int t = 0; t < T; ++t) {
            const size_t blk = (size_t)bh * ntile_head + t0 + t;
            const float kc = kmean[blk * TD + c];
            const float4* vs4 = reinterpret_cast<const float4*>(vsum + blk * TD + 32 * cc);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const float4 v = vs4[q4];
              f[4 * q4] = fmaf(-kc, v.x, f[4 * q4]);
              f[4 * q4 + 1] = fmaf(-kc, v.y, f[4 * q4 + 1]);
              f[4 * q4 + 2] = fmaf(-kc, v.z, f[4 * q4 + 2]);
              f[4 * q4 + 3] = fmaf(-kc, v.w, f[4 * q4 + 3]);
            }
          }
        }
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          atomicAdd(hrow + 8 * cc + q4,
                    make_float4(__uint_as_float(a[4 * q4]) * oscale, __uint_as_float(a[4 * q4 + 1]) * oscale,
                                __uint_as_float(a[4 * q4 + 2]) * oscale, __uint_as_float(a[4 * q4 + 3]) * oscale));
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
  }
}

}  // namespace

bool make_tmap_128x128(void* map, const void* base, int elem, uint64_t cols, uint64_t rows, uint64_t outer) {
  return make_tmap_3d(static_cast<CUtensorMap*>(map), base, elem, cols, rows, outer);
}

sa_status kv_outer_tc(const void* K, const void* V, const sa_shape& s, int feature, const float* kmean,
                      const float* vsum, float oscale, float* out, cudaStream_t stream) {
  if (s.d != TD || (s.N % TB) || (feature == kKvCentre && s.block != TB)) return SA_ERR_UNSUPPORTED;
  const uint64_t BH = (uint64_t)s.B * s.H;
  CUtensorMap mk, mv;
  if (!make_tmap_3d(&mk, K, 2, TD, s.N, BH) || !make_tmap_3d(&mv, V, 2, TD, s.N, BH))
    return fail(SA_ERR_CUDA, "sa_block_pool: cuTensorMapEncodeTiled failed for K/V");
  const size_t smem = HtLayout::smem_bytes();
  if (cudaFuncSetAttribute(htot_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(htot_tc_kernel)");
  const int nt = s.N / TB;
  // tiles per CTA: one CTA per SM (three 64 KB stages), so a wave of CTAs of
  // c tiles takes about c + 2 tile-times (ring fill, the d×d atomic flush);
  // pick the c with the fewest tile-times over all waves, at least
  // kHtMinTiles
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  int tpc = kHtMinTiles;
  long best = -1;
  for (int c = kHtMinTiles; c <= std::max(kHtMinTiles, nt); ++c) {
    const long ctas = (long)((nt + c - 1) / c) * (long)BH;
    const long cost = ((ctas + sms - 1) / sms) * (long)(c + 2);
    if (best < 0 || cost < best) {
      best = cost;
      tpc = c;
    }
    if (ctas <= sms) break;   // one wave: more tiles per CTA only add time
  }
  dim3 grid((nt + tpc - 1) / tpc, (unsigned)BH);
  htot_tc_kernel<<<grid, kHtThreads, smem, stream>>>(mk, mv, s.N, tpc, feature, kmean, vsum, oscale, out);
  return launch_status("htot_tc_kernel");
}

bool attn_tc_supports(sa_dtype dtype, const sa_shape& s, sa_tail_mode tail) {
  return dtype == SA_BF16 && s.block == TB && s.d == TD &&
         (tail == SA_TAIL_DROP || tail == SA_TAIL_ZERO_ORDER || tail == SA_TAIL_LINEAR_MIX ||
          tail == SA_TAIL_FIRST_ORDER);
}

sa_status attn_tc(const void* Q, const void* K, const void* V, const sa_shape& s, const int32_t* block_idx,
                  int topk, sa_tail_mode tail, const float* alpha, const sa_block_stats& st, float scale,
                  void* O, float* lse_out, cudaStream_t stream) {
  const int nb = s.N / TB;
  const uint64_t BH = (uint64_t)s.B * s.H;
  CUtensorMap mq, mk, mv, mkb, mvb;
  if (!make_tmap_3d(&mq, Q, 2, TD, s.N, BH) || !make_tmap_3d(&mk, K, 2, TD, s.N, BH) ||
      !make_tmap_3d(&mv, V, 2, TD, s.N, BH))
    return fail(SA_ERR_CUDA, "sa_sparse_attn_fwd: cuTensorMapEncodeTiled failed for Q/K/V");
  if (tail == SA_TAIL_LINEAR_MIX) {
    const size_t smem = LinLayout::smem_bytes();
    if (cudaFuncSetAttribute(attn_tc_linmix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return launch_status("cudaFuncSetAttribute(attn_tc_linmix_kernel)");
    dim3 grid(nb, (unsigned)BH);
    const cudaError_t le = launch_pdl(attn_tc_linmix_kernel, grid, dim3(kTcThreads), smem, stream, mq, mk, mv,
                                      block_idx, nb, topk, scale * kLog2e, alpha, st.zrelu, st.htot, st.ztot, s.H,
                                      static_cast<__nv_bfloat16*>(O), s.N);
    if (le != cudaSuccess)
      return fail(SA_ERR_CUDA, std::string("attn_tc_linmix_kernel: ") + cudaGetErrorString(le));
    return launch_status("attn_tc_linmix_kernel");
  }
  const bool fo = tail == SA_TAIL_FIRST_ORDER;
  const bool zo = tail == SA_TAIL_ZERO_ORDER || fo;
  CUtensorMap mhb = mk;
  if (zo) {
    if (!make_tmap_3d(&mkb, st.kmean_bf16, 2, TD, nb, BH) || !make_tmap_3d(&mvb, st.vmean_bf16, 2, TD, nb, BH))
      return fail(SA_ERR_CUDA, "sa_sparse_attn_fwd: cuTensorMapEncodeTiled failed for the block centroids");
  } else {
    mkb = mk;
    mvb = mv;
  }
  if (fo && !make_tmap_3d(&mhb, st.hbarT_bf16, 2, TD, TD, BH))
    return fail(SA_ERR_CUDA, "sa_sparse_attn_fwd: cuTensorMapEncodeTiled failed for H̄ᵀ");
  return launch_tc<false>(mq, mk, mv, mkb, mvb, mhb, zo, fo, s, block_idx, topk, scale, F8Scales{}, O, lse_out,
                          stream);
}

}  // namespace sa

extern "C" sa_status sa_sparse_attn_fwd_fp8(const sa_fp8_operands* ops, sa_shape shape,
                                            const int32_t* block_idx, int32_t topk, sa_tail_mode tail,
                                            float scale, void* O, void* stream) {
  using namespace sa;
  sa_status r = check_shape(shape, "sa_sparse_attn_fwd_fp8");
  if (r != SA_OK) return r;
  if (shape.d != TD || shape.block != TB)
    return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd_fp8: d and block must be 128");
  if (tail != SA_TAIL_DROP && tail != SA_TAIL_ZERO_ORDER)
    return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd_fp8: tail must be SA_TAIL_DROP or SA_TAIL_ZERO_ORDER");
  if (shape.B == 0 || shape.H == 0 || shape.N == 0) return SA_OK;
  const int nb = shape.N / TB;
  if (!ops || !ops->q || !ops->k || !ops->v || !ops->q_scale || !ops->k_scale || !ops->v_scale ||
      !ops->v_scale_max || !O)
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd_fp8: codes, scales, v_scale_max and O are required");
  const bool zo = tail == SA_TAIL_ZERO_ORDER;
  if (zo && (!ops->kbar || !ops->vbar || !ops->kbar_scale || !ops->vbar_scale))
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd_fp8: SA_TAIL_ZERO_ORDER needs the centroid codes and scales");
  if (topk < 0 || topk > nb) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd_fp8: topk must be in [0, N/block]");
  if (topk > 0 && !block_idx) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_fwd_fp8: block_idx is required");
  if (nb > kMaxAttnBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_sparse_attn_fwd_fp8: at most 4096 blocks per head");
  const void* ptrs[] = {ops->q, ops->k, ops->v, ops->kbar, ops->vbar, O, block_idx};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_sparse_attn_fwd_fp8: pointers must be 16-byte aligned");
  const uint64_t BH = (uint64_t)shape.B * shape.H;
  CUtensorMap mq, mk, mv, mkb, mvb;
  if (!make_tmap_3d(&mq, ops->q, 1, TD, shape.N, BH) || !make_tmap_3d(&mk, ops->k, 1, TD, shape.N, BH) ||
      !make_tmap_3d(&mv, ops->v, 1, TD, shape.N, BH))
    return fail(SA_ERR_CUDA, "sa_sparse_attn_fwd_fp8: cuTensorMapEncodeTiled failed for Q/K/V");
  if (zo) {
    if (!make_tmap_3d(&mkb, ops->kbar, 1, TD, nb, BH) || !make_tmap_3d(&mvb, ops->vbar, 1, TD, nb, BH))
      return fail(SA_ERR_CUDA, "sa_sparse_attn_fwd_fp8: cuTensorMapEncodeTiled failed for the centroids");
  } else {
    mkb = mk;
    mvb = mv;
  }
  F8Scales f8{ops->q_scale, ops->k_scale, ops->v_scale, ops->v_scale_max, ops->kbar_scale, ops->vbar_scale};
  return launch_tc<true>(mq, mk, mv, mkb, mvb, mk, zo, false, shape, block_idx, topk, scale, f8, O, nullptr,
                         as_stream(stream));
}

extern "C" sa_status sa_device_error(uint32_t* code) {
  using namespace sa;
  if (!code) return fail(SA_ERR_INVALID_ARG, "sa_device_error: code is required");
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, tc::g_device_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return launch_status("sa_device_error");
  *code = v | decode_error_take() | covnorm_error_take() | bwd_error_take() | decode_tc_error_take();
  return SA_OK;
}
