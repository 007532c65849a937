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
//   4. Lanczos on G (symmetric positive semi-definite) from a fixed positive
//      start vector: each step one product w = G v (each thread's row of G
//      read from TMEM in 32-column pieces, which leaves room for three CTAs
//      per SM) and two reductions across the four warps
//      (α = vᵀw, then β = ‖w − α v − β_prev v_prev‖).  After 8, 10, 12, ...
//      steps one warp finds the largest eigenvalue θ of the tridiagonal T (α
//      on the diagonal, β off it) by Sturm-count multisection (32 points per
//      round, 5 rounds: 33^-5 of the Gershgorin interval) and shares it; the
//      iteration stops when θ moved by less than 1e-6 (relative) since the
//      last check, when β vanishes (the Krylov space is invariant), or after
//      32 steps.  M_j = sqrt(θ) = σ_max(A).  Blocks of the smooth video
//      workloads converge in 8-10 steps; Gaussian blocks, whose top
//      eigenvalues crowd, in 20-24.
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
constexpr int kCvMaxSteps = 32;               // Lanczos steps at most
constexpr float kCvTol = 1e-6f;

struct CvLayout {
  static constexpr uint32_t kK = 0, kV = kCvTile;
  static constexpr uint32_t kX = 2 * kCvTile;              // float x[2][128]
  static constexpr uint32_t kRed = kX + 2 * 128 * 4;       // float red[2][4 warps][2]
  static constexpr uint32_t kT = kRed + 2 * 4 * 2 * 4;     // float alpha[32], beta[32]
  static constexpr uint32_t kTheta = kT + 2 * kCvMaxSteps * 4;   // float θ, 3 spare
  static constexpr uint32_t kBar = kTheta + 16;
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

// Largest eigenvalue of the symmetric tridiagonal T (diagonal al[0..n),
// off-diagonal be[0..n-1)) by multisection on Sturm counts: the number of
// negative pivots of T − x I is the number of eigenvalues below x.  `prev`
// is the value for a leading block of T (or <= 0): by interlacing it bounds
// the answer from below, and the first round tests prev (1 + tol) on lane 0,
// so a converged θ costs one round.  All 32 lanes return the same value.
__device__ __forceinline__ float tridiag_max_eig(const float* al, const float* be, int n, int lane, float prev,
                                                 float tol) {
  float lo = al[0], hi = -INFINITY;
#pragma unroll 4
  for (int i = 0; i < n; ++i) {
    const float bl = i > 0 ? fabsf(be[i - 1]) : 0.f, br = i + 1 < n ? fabsf(be[i]) : 0.f;
    lo = fmaxf(lo, al[i]);                 // a Rayleigh quotient: λ_max >= α_i
    hi = fmaxf(hi, al[i] + bl + br);       // Gershgorin
  }
  lo = fmaxf(lo, fminf(prev, hi));
  const bool probe = prev > 0.f && prev * (1.f + tol) < hi;
  const float tiny = 1e-30f;
  for (int round = 0; round < 5; ++round) {
    float x;
    if (round == 0 && probe) {
      const float xc = prev * (1.f + tol);
      x = lane == 0 ? xc : xc + (hi - xc) * (float)lane * (1.0f / 32.0f);
    } else {
      x = lo + (hi - lo) * (float)(lane + 1) * (1.0f / 33.0f);
    }
    int below = 0;
    float d = 1.f;
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
      const float b2 = i > 0 ? be[i - 1] * be[i - 1] : 0.f;
      d = (al[i] - x) - (i > 0 ? __fdividef(b2, d) : 0.f);
      if (fabsf(d) < tiny) d = -tiny;
      below += d < 0.f;
    }
    // λ_max > x exactly where fewer than n eigenvalues lie below x; the
    // points increase with the lane, so those lanes form a prefix
    const unsigned above = __ballot_sync(0xffffffffu, below < n);
    const int p = __popc(above);
    const float xl = __shfl_sync(0xffffffffu, x, p > 0 ? p - 1 : 0);
    const float xh = __shfl_sync(0xffffffffu, x, p < 32 ? p : 31);
    const float nlo = p > 0 ? xl : lo, nhi = p < 32 ? xh : hi;
    lo = nlo;
    hi = nhi;
    if (round == 0 && probe && p == 0) break;   // θ within tol of prev
  }
  return 0.5f * (lo + hi);
}

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
      // 16-byte chunk k16 of a row of the K or V tile: span k16 / 8,
      // position (k16 % 8) ^ (row % 8) (the 128-byte swizzle)
      auto chunk_off = [](int row, int k16) -> uint32_t {
        return (uint32_t)(k16 >> 3) * kCvSpan + (uint32_t)row * 128u + ((uint32_t)((k16 & 7) ^ (row & 7)) << 4);
      };
      // H̄ rows of this warp, staged through the bytes the A tiles will take:
      // the 32 floats of row R, columns [32 cc, 32 cc + 32) go to chunks
      // 4 cc .. 4 cc + 3 of row R in the K tile (floats 0-15) and the V tile
      // (floats 16-31).  Global reads are whole 128-byte row segments.
      const float4* hbh = reinterpret_cast<const float4*>(hbar + ((size_t)bh * kCvD + wq * 32) * kCvD);
#pragma unroll 2
      for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int r = 4 * it + (lane >> 3), f = lane & 7;
          const float4 hv = hbh[(size_t)r * (kCvD / 4) + 8 * cc + f];
          const uint32_t base = f < 4 ? L::kK : L::kV;
          *reinterpret_cast<float4*>(smem + base + chunk_off(wq * 32 + r, 4 * cc + (f & 3))) = hv;
        }
      }
      __syncwarp();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t a[32];
        tmem_ld32(lrow + 32 * cc, a);
        float hbv[32];
#pragma unroll
        for (int f = 0; f < 8; ++f) {
          const float4 hv = *reinterpret_cast<const float4*>(smem + (f < 4 ? L::kK : L::kV) + chunk_off(c, 4 * cc + (f & 3)));
          hbv[4 * f] = hv.x;
          hbv[4 * f + 1] = hv.y;
          hbv[4 * f + 2] = hv.z;
          hbv[4 * f + 3] = hv.w;
        }
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float val[8];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 v = vs4[8 * cc + 2 * q + h];
            const float* t = reinterpret_cast<const float*>(&a[8 * q + 4 * h]);
            const float* hb = hbv + 8 * q + 4 * h;
            val[4 * h + 0] = fmaf(-kc, v.x, t[0]) - hb[0];
            val[4 * h + 1] = fmaf(-kc, v.y, t[1]) - hb[1];
            val[4 * h + 2] = fmaf(-kc, v.z, t[2]) - hb[2];
            val[4 * h + 3] = fmaf(-kc, v.w, t[3]) - hb[3];
          }
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(val[2 * e]), h1 = __float2bfloat16_rn(val[2 * e + 1]);
            hi[e] = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
            lo[e] = pack_bf16(val[2 * e] - __bfloat162float(h0), val[2 * e + 1] - __bfloat162float(h1));
          }
          // this row's chunk 4 cc + q: its staged H̄ floats are already in registers
          const uint32_t off = chunk_off(c, 4 * cc + q);
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
      // positive start vector with no structure; every thread knows its norm
      auto start = [](int i) {
        return 0.5f + (float)((((uint32_t)i * 2654435761u) >> 24) & 0xffu) * (1.0f / 256.0f);
      };
      float own = start(c);                      // this thread's entry of the unnormalised vector
      float n2 = 0.f;
      for (int i = 0; i < kCvD; ++i) n2 = fmaf(start(i), start(i), n2);
      xs[c] = own;
      float* al_s = reinterpret_cast<float*>(smem + L::kT);
      float* be_s = al_s + kCvMaxSteps;
      float* theta_s = reinterpret_cast<float*>(smem + L::kTheta);
      bar_math();
      float inv = rsqrtf(n2), vp = 0.f, bp = 0.f, theta = 0.f, theta_prev = -1.f;
      int b = 0;
      for (int k = 0; k < kCvMaxSteps; ++k) {
        // w = G v with v = xs[b] · inv
        const float4* x4 = reinterpret_cast<const float4*>(xs + 128 * b);
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t g[32];
          tmem_ld32(lrow + 32 * h, g);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 u = x4[8 * h + q];
            acc[q] = fmaf(__uint_as_float(g[4 * q]), u.x, acc[q]);
            acc[q] = fmaf(__uint_as_float(g[4 * q + 1]), u.y, acc[q]);
            acc[q] = fmaf(__uint_as_float(g[4 * q + 2]), u.z, acc[q]);
            acc[q] = fmaf(__uint_as_float(g[4 * q + 3]), u.w, acc[q]);
          }
        }
        float wv = (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]))) * inv;
        const float v = own * inv;
        const float pa = warp_sum_f(v * wv);
        if (lane == 0) red[(b * 4 + wq) * 2] = pa;
        bar_math();
        float alpha = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) alpha += red[(b * 4 + w) * 2];
        if (c == 0) al_s[k] = alpha;
        wv = wv - alpha * v - bp * vp;
        xs[128 * (b ^ 1) + c] = wv;
        const float pb = warp_sum_f(wv * wv);
        if (lane == 0) red[(b * 4 + wq) * 2 + 1] = pb;
        bar_math();
        float b2 = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) b2 += red[(b * 4 + w) * 2 + 1];
        const float beta = sqrtf(b2);
        if (c == 0) be_s[k] = beta;            // read from step k + 1 on
        vp = v;
        own = wv;
        bp = beta;
        inv = beta > 0.f ? 1.0f / beta : 0.f;
        b ^= 1;
        // every thread takes the same decisions from the same shared values;
        // warp 0 of the group finds θ and shares it
        const int n = k + 1;
        const bool invariant = !(beta > 1e-7f * fabsf(alpha));
        if (invariant || n == kCvMaxSteps || (n >= 8 && (n & 1) == 0)) {
          if (wq == 0) {
            const float t = tridiag_max_eig(al_s, be_s, n, lane, theta_prev, 0.5f * kCvTol);
            if (lane == 0) theta_s[0] = t;
          }
          bar_math();
          theta = theta_s[0];
          if (invariant || n == kCvMaxSteps || fabsf(theta - theta_prev) <= kCvTol * theta) break;
          theta_prev = theta;
        }
      }
      const float lam = theta;
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
