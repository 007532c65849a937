// PISA's covariance-aware routing statistic ("Roteamento Consciente de
// Covariância"): M_j = ‖H_j − H̄‖₂, the spectral norm of block j's
// first-order matrix H_j = Σ_{n∈j} (k_n − k̄_j) v_nᵀ minus the head's mean H̄,
// on the tensor cores for bf16 with d = block = 128.  One CTA per block:
//   1. TMA brings the block's K and V tiles; one MMA chain accumulates Kᵀ V
//      (128×128 fp32 in TMEM; both operands MN-major).  bf16 products are
//      exact in fp32, so nothing is rounded before step 2.
//   2. Warps 2-5 (thread = row c of the matrix) form
//      A = Kᵀ V − k̄_j vsum_jᵀ − H̄ = H_j − H̄ in fp32 and store it as a pair of
//      bf16 operand tiles A = A_hi + A_lo (K-major, 128-byte swizzle) over
//      the K and V tiles' shared memory.
//   3. Three MMA chains accumulate G = A Aᵀ ≈ A_hi A_hiᵀ + A_hi A_loᵀ +
//      A_lo A_hiᵀ into the same TMEM columns (the dropped A_lo A_loᵀ is
//      ~2^-16 of G).
//   4. Power iteration on G (symmetric positive semi-definite): y = G x with
//      each thread's row of G read from TMEM, one reduction of ‖y‖², xᵀy and
//      ‖x‖² across the four warps per step; it stops when the Rayleigh
//      quotient xᵀGx / xᵀx changes by less than 1e-6 (relative) or after 256
//      steps, and M_j = sqrt(λ_max(G)) = σ_max(A).
// Every mbarrier wait is bounded; a give-up sets this unit's device error
// word (read through sa_device_error) and the CTA skips the rest.
#include "attn_simt.cuh"
#include "tc_util.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int kCvThreads = 192;
constexpr int kCvD = 128;                      // head dim = tokens per block
constexpr uint32_t kCvSpan = 128 * 128;        // 128 rows of one 128-byte swizzle span
constexpr uint32_t kCvTile = 2 * kCvSpan;      // one 128×128 bf16 tile
constexpr int kCvMaxSteps = 256;
constexpr float kCvTol = 1e-6f;

struct CvLayout {
  static constexpr uint32_t kK = 0, kV = kCvTile;
  static constexpr uint32_t kX = 2 * kCvTile;              // float x[2][128]
  static constexpr uint32_t kRed = kX + 2 * 128 * 4;       // float red[2][4 warps][4]
  static constexpr uint32_t kBar = kRed + 2 * 4 * 4 * 4;
  enum { B_KF = 0, B_VF, B_H, B_A, B_G, B_FIN, NBAR };
  static constexpr uint32_t kSlot = kBar + 8 * NBAR;
  static size_t smem_bytes() { return 1024 + kSlot + 16; }
};

__device__ __forceinline__ bool cv_wait_bounded(uint32_t bar, uint32_t parity) {
  // abort path only: the copy or MMA being waited for is already in flight
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

__device__ __forceinline__ void bar_math() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kCvThreads, 3)
covnorm_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int nb,
                  const float* __restrict__ kmean, const float* __restrict__ vsum,
                  const float* __restrict__ hbar, float* __restrict__ covnorm) {
  using L = CvLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int j = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kSlot + 4);
  auto bar = [&](int k) { return sb + L::kBar + 8u * k; };

  if (threadIdx.x == 0) {
    mbar_init(bar(L::B_KF), 1);
    mbar_init(bar(L::B_VF), 1);
    mbar_init(bar(L::B_H), 1);
    mbar_init(bar(L::B_A), 128);
    mbar_init(bar(L::B_G), 1);
    mbar_init(bar(L::B_FIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      mbar_expect_tx(bar(L::B_KF), kCvTile);
      tma_load_3d(sb + L::kK, &tmK, 0, j * kCvD, bh, bar(L::B_KF));
      tma_load_3d(sb + L::kK + kCvSpan, &tmK, 64, j * kCvD, bh, bar(L::B_KF));
      mbar_expect_tx(bar(L::B_VF), kCvTile);
      tma_load_3d(sb + L::kV, &tmV, 0, j * kCvD, bh, bar(L::B_VF));
      tma_load_3d(sb + L::kV + kCvSpan, &tmV, 64, j * kCvD, bh, bar(L::B_VF));
      // the copies land before the CTA can leave, whatever the other roles do
      cv_wait_bounded(bar(L::B_KF), 0);
      cv_wait_bounded(bar(L::B_VF), 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      bool ok = mbar_wait(bar(L::B_KF), 0, abort_flag) && mbar_wait(bar(L::B_VF), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        // Kᵀ V: M = key channel c, N = value channel e, K = the 128 tokens
        constexpr uint32_t idH = idesc_bf16_f32(kCvD, kCvD, 1, 1);
#pragma unroll
        for (int k = 0; k < kCvD / 16; ++k)
          mma_ss(tbase, desc_sw128(sb + L::kK + k * 16 * 128, kCvSpan, 1024),
                 desc_sw128(sb + L::kV + k * 16 * 128, kCvSpan, 1024), idH, k > 0);
        mma_commit(bar(L::B_H));
        ok = mbar_wait(bar(L::B_A), 0, abort_flag);
      }
      if (ok) {
        tc_fence_after();
        // G = A Aᵀ: both operands are A's rows (K-major, 32 bytes per K step,
        // next 64-column span every four steps)
        constexpr uint32_t idG = idesc_bf16_f32(kCvD, kCvD, 0, 0);
        const uint64_t dhi = desc_sw128(sb + L::kK, 16, 1024), dlo = desc_sw128(sb + L::kV, 16, 1024);
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          const uint64_t da = p == 2 ? dlo : dhi, db = p == 1 ? dlo : dhi;
#pragma unroll
          for (int k = 0; k < kCvD / 16; ++k) {
            const uint32_t koff = (k >> 2) * kCvSpan + (k & 3) * 32;
            mma_ss(tbase, desc_adv(da, koff), desc_adv(db, koff), idG, (p > 0 || k > 0));
          }
        }
        mma_commit(bar(L::B_G));
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(bar(L::B_FIN));
      cv_wait_bounded(bar(L::B_FIN), 0);
    }
  } else {
    // ------------------------------------------------------------ math (warps 2-5)
    const int wq = warp & 3;                        // TMEM lane quarter
    const int c = wq * 32 + lane;                   // matrix row
    const uint32_t lrow = tbase + ((uint32_t)(wq * 32) << 16);
    float* xs = reinterpret_cast<float*>(smem + L::kX);
    float* red = reinterpret_cast<float*>(smem + L::kRed);
    const bool okh = __all_sync(0xffffffffu, mbar_wait(bar(L::B_H), 0, abort_flag));
    if (okh) {
      tc_fence_after();
      const size_t blk = (size_t)bh * nb + j;
      const float kc = kmean[blk * kCvD + c];
      const float4* vs4 = reinterpret_cast<const float4*>(vsum + blk * kCvD);
      const float4* hb4 = reinterpret_cast<const float4*>(hbar + ((size_t)bh * kCvD + c) * kCvD);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t a[32];
        tmem_ld32(lrow + 32 * cc, a);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float val[8];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 v = vs4[8 * cc + 2 * q + h];
            const float4 hb = hb4[8 * cc + 2 * q + h];
            const float* t = reinterpret_cast<const float*>(&a[8 * q + 4 * h]);
            val[4 * h + 0] = fmaf(-kc, v.x, t[0]) - hb.x;
            val[4 * h + 1] = fmaf(-kc, v.y, t[1]) - hb.y;
            val[4 * h + 2] = fmaf(-kc, v.z, t[2]) - hb.z;
            val[4 * h + 3] = fmaf(-kc, v.w, t[3]) - hb.w;
          }
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(val[2 * e]), h1 = __float2bfloat16_rn(val[2 * e + 1]);
            hi[e] = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
            lo[e] = pack_bf16(val[2 * e] - __bfloat162float(h0), val[2 * e + 1] - __bfloat162float(h1));
          }
          // 16-byte chunk k16 of row c: span k16 / 8, position (k16 % 8) ^ (c % 8)
          const int k16 = 4 * cc + q;
          const uint32_t off = (uint32_t)(k16 >> 3) * kCvSpan + (uint32_t)c * 128u +
                               ((uint32_t)((k16 & 7) ^ (c & 7)) << 4);
          *reinterpret_cast<uint4*>(smem + L::kK + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(smem + L::kV + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
    }
    mbar_arrive(bar(L::B_A));
    if (okh) mbar_wait(bar(L::B_G), 0, abort_flag);
    // one decision for the four warps: a give-up anywhere sets the flag
    // before this barrier, and nothing sets it after
    bar_math();
    if (!*abort_flag) {
      tc_fence_after();
      // positive start vector with no structure
      float xo = 0.5f + (float)((((uint32_t)c * 2654435761u) >> 24) & 0xffu) * (1.0f / 256.0f);
      xs[c] = xo;
      bar_math();
      float inv = 1.f, lam = 0.f, lam_prev = -1.f;
      int b = 0;
      for (int it = 0; it < kCvMaxSteps; ++it) {
        // y_c = (G[c] · x_raw) · inv, x = x_raw · inv of unit norm after step 0
        const float4* x4 = reinterpret_cast<const float4*>(xs + 128 * b);
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t g0[32], g1[32];
          tmem_ld32(lrow + 64 * h, g0);
          tmem_ld32(lrow + 64 * h + 32, g1);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 u = x4[16 * h + q];
            acc[q] = fmaf(__uint_as_float(g0[4 * q]), u.x, acc[q]);
            acc[q] = fmaf(__uint_as_float(g0[4 * q + 1]), u.y, acc[q]);
            acc[q] = fmaf(__uint_as_float(g0[4 * q + 2]), u.z, acc[q]);
            acc[q] = fmaf(__uint_as_float(g0[4 * q + 3]), u.w, acc[q]);
            const float4 w = x4[16 * h + 8 + q];
            acc[q] = fmaf(__uint_as_float(g1[4 * q]), w.x, acc[q]);
            acc[q] = fmaf(__uint_as_float(g1[4 * q + 1]), w.y, acc[q]);
            acc[q] = fmaf(__uint_as_float(g1[4 * q + 2]), w.z, acc[q]);
            acc[q] = fmaf(__uint_as_float(g1[4 * q + 3]), w.w, acc[q]);
          }
        }
        const float y = (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]))) * inv;
        const float xc = xo * inv;
        const float p1 = warp_sum_f(y * y), p2 = warp_sum_f(xc * y), p3 = warp_sum_f(xc * xc);
        if (lane == 0) {
          red[(b * 4 + wq) * 4 + 0] = p1;
          red[(b * 4 + wq) * 4 + 1] = p2;
          red[(b * 4 + wq) * 4 + 2] = p3;
        }
        xs[128 * (b ^ 1) + c] = y;
        bar_math();
        float S1 = 0.f, S2 = 0.f, S3 = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          S1 += red[(b * 4 + w) * 4 + 0];
          S2 += red[(b * 4 + w) * 4 + 1];
          S3 += red[(b * 4 + w) * 4 + 2];
        }
        lam = S3 > 0.f ? S2 / S3 : 0.f;
        xo = y;
        inv = S1 > 0.f ? rsqrtf(S1) : 0.f;
        b ^= 1;
        // every thread takes the same decision from the same shared sums
        if (!(S1 > 0.f) || fabsf(lam - lam_prev) <= kCvTol * lam) break;
        lam_prev = lam;
      }
      if (c == 0) covnorm[(size_t)bh * nb + j] = sqrtf(fmaxf(lam, 0.f));
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

sa_status covnorm_tc(const void* K, const void* V, const sa_shape& s, const float* kmean, const float* vsum,
                     const float* hbar, float* covnorm, cudaStream_t stream) {
  if (s.d != kCvD || s.block != kCvD || (s.N % kCvD)) return SA_ERR_UNSUPPORTED;
  const uint64_t BH = (uint64_t)s.B * s.H;
  const int nb = s.N / kCvD;
  CUtensorMap mk, mv;
  if (!make_tmap_128x128(&mk, K, 2, kCvD, s.N, BH) || !make_tmap_128x128(&mv, V, 2, kCvD, s.N, BH))
    return fail(SA_ERR_CUDA, "sa_block_pool: cuTensorMapEncodeTiled failed for K/V");
  const size_t smem = CvLayout::smem_bytes();
  if (cudaFuncSetAttribute(covnorm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return launch_status("cudaFuncSetAttribute(covnorm_tc_kernel)");
  dim3 grid(nb, (unsigned)BH);
  covnorm_tc_kernel<<<grid, kCvThreads, smem, stream>>>(mk, mv, nb, kmean, vsum, hbar, covnorm);
  return launch_status("covnorm_tc_kernel");
}

uint32_t covnorm_error_take() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, tc::g_device_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(tc::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return 0u;
  return v;
}

}  // namespace sa
