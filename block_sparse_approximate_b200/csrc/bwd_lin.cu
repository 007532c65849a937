// Backward of SLA2's mixture (§2A) O = α⊙O_s + (1−α)⊙O_l: O_s is softmax
// attention over the selected blocks S_i (the drop output), O_l the ReLU
// linear attention over the unselected ones (SALAD §2),
//   O_l,t = φ(q_t)ᵀ H_U / (φ(q_t)·z_U + ε),  H_U = H_tot − Σ_{j∈S_i} h_j,
//   z_U = z_tot − Σ_{j∈S_i} z_j,  h_j = Σ_{n∈j} φ(k_n) v_nᵀ,  φ = ReLU
// (O_l = 0 when every block is selected).  With g = dO_t and g_l = (1−α)⊙g:
//   softmax branch: the drop backward with the cotangent α⊙g and
//     δ_s = (α⊙g)·O_s = g·O − g_l·O_l (no division by α);
//   linear branch:  dnum = g_l / den,  dden = −(g_l·O_l) / den,
//     dq += 1[q > 0] ⊙ (H_U dnum + z_U dden),
//     dH_U,i = Σ_{t∈i} φ(q_t) dnumᵀ,  dz_U,i = Σ_{t∈i} φ(q_t) dden,
//     and each key block j collects dh_j = Σ_{i: j∉S_i} dH_U,i (formed as
//     the total over query blocks minus the query blocks that selected j,
//     SPLA §2.2's subtraction form again), dz_j likewise:
//     dk_n += 1[k_n > 0] ⊙ (dh_j v_n + dz_j),  dv_n += dh_jᵀ φ(k_n).
// Kernels (mma.sync products on the tiles of mma_tile.cuh):
//   lin_hblk_kernel  h_j of every block, bf16 (the query blocks read
//                    Σ_{j∈S_i} h_j from them, a head's h_j staying in L2);
//   lin_q_kernel     per query block: H_U, O_l, then δ_s, α⊙g, dH_U,i,
//                    dz_U,i and the dq term, written to dQ (the softmax
//                    branch's dQ kernel then adds its own);
//   lin_tot_kernel   Σ_i dH_U,i and Σ_i dz_U,i per head, in order;
//   lin_kv_kernel    per key block: dh_j, dz_j and the dk, dv terms.
// No atomics: every sum runs in a fixed order.
#include "mma_tile.cuh"

namespace sa {
namespace {

using namespace mt;

constexpr float kLinEps = 1e-6f;   // the linear branch's denominator term (SLA2 §2A reading)

__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t x) {
  const __nv_bfloat162 z = __float2bfloat162_rn(0.f);
  const __nv_bfloat162 r = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&x), z);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// a[e] (e < 64) = init[e] − Σ_{s < n} M_{ids[s]}[64 tid + e]: the thread's 64
// entries of a sum of bf16 d x d matrices M_i = base + i d², the indices in
// shared memory; two matrices' loads in flight at a time
__device__ __forceinline__ void sub_matrices(float (&a)[64], const float* init, const __nv_bfloat16* base,
                                             const int* ids, int n, int tid) {
#pragma unroll
  for (int e = 0; e < 64; e += 4) {
    const float4 x = *reinterpret_cast<const float4*>(init + 64 * tid + e);
    a[e] = x.x;
    a[e + 1] = x.y;
    a[e + 2] = x.z;
    a[e + 3] = x.w;
  }
  auto sub8 = [&](const uint4 (&x)[8]) {
#pragma unroll
    for (int e8 = 0; e8 < 8; ++e8) {
      const uint32_t xv[4] = {x[e8].x, x[e8].y, x[e8].z, x[e8].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv[u]));
        a[8 * e8 + 2 * u] -= f.x;
        a[8 * e8 + 2 * u + 1] -= f.y;
      }
    }
  };
  int s = 0;
  for (; s + 2 <= n; s += 2) {
    const uint4* m0 = reinterpret_cast<const uint4*>(base + (size_t)ids[s] * FD * FD + 64 * tid);
    const uint4* m1 = reinterpret_cast<const uint4*>(base + (size_t)ids[s + 1] * FD * FD + 64 * tid);
    uint4 x0[8], x1[8];
#pragma unroll
    for (int e8 = 0; e8 < 8; ++e8) x0[e8] = m0[e8];
#pragma unroll
    for (int e8 = 0; e8 < 8; ++e8) x1[e8] = m1[e8];
    sub8(x0);
    sub8(x1);
  }
  if (s < n) {
    const uint4* m0 = reinterpret_cast<const uint4*>(base + (size_t)ids[s] * FD * FD + 64 * tid);
    uint4 x0[8];
#pragma unroll
    for (int e8 = 0; e8 < 8; ++e8) x0[e8] = m0[e8];
    sub8(x0);
  }
}

// the thread's 64 entries (row tid / 2, columns 64 (tid & 1) ..) as a bf16 tile
__device__ __forceinline__ void store_entries(uint8_t* tile, const float (&a)[64], int tid) {
  const int r = tid >> 1;
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    const int c = 8 * (tid & 1) + c8;
    *reinterpret_cast<uint4*>(tile + swz(r, c)) =
        make_uint4(fo_pack2(a[8 * c8], a[8 * c8 + 1]), fo_pack2(a[8 * c8 + 2], a[8 * c8 + 3]),
                   fo_pack2(a[8 * c8 + 4], a[8 * c8 + 5]), fo_pack2(a[8 * c8 + 6], a[8 * c8 + 7]));
  }
}

// a bf16 [128][128] tile of rows with ReLU applied, into shared memory
__device__ __forceinline__ void stage_relu(uint8_t* dst, const __nv_bfloat16* src) {
  for (int o = threadIdx.x; o < FT * 16; o += kFoThreads) {
    const int r = o >> 4, c = o & 15;
    const uint4 x = *reinterpret_cast<const uint4*>(src + (size_t)r * FD + 8 * c);
    *reinterpret_cast<uint4*>(dst + swz(r, c)) =
        make_uint4(relu_bf16x2(x.x), relu_bf16x2(x.y), relu_bf16x2(x.z), relu_bf16x2(x.w));
  }
}

// the warp's accumulator tile as bf16 rows of a [128][128] array in global memory
__device__ __forceinline__ void store_acc_bf16(__nv_bfloat16* base, const float (&acc)[16][4], int ra, int rb,
                                               int lane) {
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int c = 8 * nt + 2 * (lane & 3);
    *reinterpret_cast<uint32_t*>(base + (size_t)ra * FD + c) = fo_pack2(acc[nt][0], acc[nt][1]);
    *reinterpret_cast<uint32_t*>(base + (size_t)rb * FD + c) = fo_pack2(acc[nt][2], acc[nt][3]);
  }
}

// h_j = Σ_{n∈j} φ(k_n) v_nᵀ (row c, column e), bf16
__global__ void __launch_bounds__(kFoThreads)
lin_hblk_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V, int N,
                __nv_bfloat16* __restrict__ hblk) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int j = blockIdx.x, bh = blockIdx.y, nb = N / FT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t row0 = (size_t)bh * N + (size_t)j * FT;
  uint8_t* kt = fsm;                 // φ(K) [n][c]
  uint8_t* vt = fsm + kTileB;        // V [n][e]
  stage_bf16(vt, V + row0 * FD);
  stage_relu(kt, K + row0 * FD);
  fo_cp_wait_all();
  __syncthreads();
  float acc[16][4];
  zero_acc(acc);
  // h[c][e] = Σ_n φk[n][c] v[n][e]: A[c][n] stored [n][c], B[n][e] stored [n][e]
  warp_gemm<kRowsKM, kRowsKM>(acc, (uint32_t)__cvta_generic_to_shared(kt), (uint32_t)__cvta_generic_to_shared(vt),
                              16 * warp, lane);
  const int ra = 16 * warp + (lane >> 2), rb = ra + 8;
  store_acc_bf16(hblk + ((size_t)bh * nb + j) * FD * FD, acc, ra, rb, lane);
}

// Per query block i: H_U = H_tot − Σ_{j∈S_i} h_j (fp32, used as a bf16 tile),
// O_l, then δ_s, α⊙g, dH_U,i, dz_U,i and the linear branch's dq, written to dQ
// (the softmax branch's dQ kernel adds its own term afterwards).
__global__ void __launch_bounds__(kFoThreads)
lin_q_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ O,
             const __nv_bfloat16* __restrict__ dO, const float* __restrict__ alpha, int H, int N,
             const int32_t* __restrict__ block_idx, int topk, const float* __restrict__ htot,
             const float* __restrict__ ztot, const float* __restrict__ zrelu, const __nv_bfloat16* __restrict__ hblk,
             float* __restrict__ delta_s, __nv_bfloat16* __restrict__ dOs, __nv_bfloat16* __restrict__ dHU,
             float* __restrict__ dzU, float* __restrict__ dQ) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int i = blockIdx.x, bh = blockIdx.y, h = bh % H, nb = N / FT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t row0 = (size_t)bh * N + (size_t)i * FT;
  const int32_t* sel = block_idx + ((size_t)bh * nb + i) * topk;
  uint8_t* hu = fsm;                          // H_U [c][e]
  uint8_t* pq = fsm + kTileB;                 // φ(Q) [t][c]
  uint8_t* dn = fsm + 2 * kTileB;             // dnum [t][e]
  float* zu = reinterpret_cast<float*>(fsm + 3 * kTileB);   // z_U [d]
  float* den = zu + FD;                       // [128]
  float* dden = den + FT;                     // [128]
  int* ids = reinterpret_cast<int*>(dden + FT);             // [topk] the selected blocks
  const float* al = alpha + (size_t)h * FD;
  const int ra = 16 * warp + (lane >> 2), rb = ra + 8;
  const bool lin = topk < nb;                 // U_i is not empty
  if (!lin) {
    // O_l = 0: δ_s = g·O, the cotangent α⊙g, no linear-branch terms
    for (int r = warp; r < FT; r += kFoThreads / 32) {
      const __nv_bfloat16* gr = dO + (row0 + r) * FD;
      const __nv_bfloat16* orow = O + (row0 + r) * FD;
      float d = 0.f;
      for (int c = lane; c < FD; c += 32) {
        const float g = __bfloat162float(gr[c]);
        d = fmaf(g, __bfloat162float(orow[c]), d);
        dOs[(row0 + r) * FD + c] = __float2bfloat16_rn(al[c] * g);
        dQ[(row0 + r) * FD + c] = 0.f;
      }
      d = warp_sum(d);
      if (lane == 0) delta_s[row0 + r] = d;
    }
    for (int x = tid; x < FD * FD; x += kFoThreads) dHU[((size_t)bh * nb + i) * FD * FD + x] = __float2bfloat16_rn(0.f);
    for (int x = tid; x < FD; x += kFoThreads) dzU[((size_t)bh * nb + i) * FD + x] = 0.f;
    return;
  }
  for (int x = tid; x < topk; x += kFoThreads) ids[x] = sel[x];
  __syncthreads();
  // ---- H_U and z_U
  {
    float a[64];
    sub_matrices(a, htot + (size_t)bh * FD * FD, hblk + (size_t)bh * nb * FD * FD, ids, topk, tid);
    store_entries(hu, a, tid);
    if (tid < FD) {
      float z = ztot[(size_t)bh * FD + tid];
      for (int s2 = 0; s2 < topk; ++s2) z -= zrelu[((size_t)bh * nb + ids[s2]) * FD + tid];
      zu[tid] = z;
    }
  }
  stage_relu(pq, Q + row0 * FD);
  __syncthreads();
  // den_t = φ(q_t)·z_U + ε
  if (tid < FT) {
    float d = 0.f;
#pragma unroll 4
    for (int c8 = 0; c8 < 16; ++c8) {
      const uint4 x = *reinterpret_cast<const uint4*>(pq + swz(tid, c8));
      const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv[u]));
        d = fmaf(f.x, zu[8 * c8 + 2 * u], fmaf(f.y, zu[8 * c8 + 2 * u + 1], d));
      }
    }
    den[tid] = d + kLinEps;
  }
  __syncthreads();
  float acc[16][4];
  zero_acc(acc);
  // num[t][e] = Σ_c φq[t][c] H_U[c][e]: A = φQ [t][c], B[c][e] stored [c][e] (k rows)
  const uint32_t hu_s = (uint32_t)__cvta_generic_to_shared(hu), pq_s = (uint32_t)__cvta_generic_to_shared(pq),
                 dn_s = (uint32_t)__cvta_generic_to_shared(dn);
  warp_gemm<kRowsMK, kRowsKM>(acc, pq_s, hu_s, 16 * warp, lane);
  // O_l, g_l, dnum (into the dn tile), the rows' g_l·O_l and g·O, α⊙g
  const float ia = 1.0f / den[ra], ib = 1.0f / den[rb];
  float ga = 0.f, gb = 0.f, oa = 0.f, ob = 0.f;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int c = 8 * nt + 2 * (lane & 3);
    const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dO + (row0 + ra) * FD + c));
    const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dO + (row0 + rb) * FD + c));
    const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(O + (row0 + ra) * FD + c));
    const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(O + (row0 + rb) * FD + c));
    const float w0 = 1.0f - al[c], w1 = 1.0f - al[c + 1];
    const float la0 = acc[nt][0] * ia, la1 = acc[nt][1] * ia, lb0 = acc[nt][2] * ib, lb1 = acc[nt][3] * ib;
    const float gla0 = w0 * g0.x, gla1 = w1 * g0.y, glb0 = w0 * g1.x, glb1 = w1 * g1.y;
    ga = fmaf(gla0, la0, fmaf(gla1, la1, ga));
    gb = fmaf(glb0, lb0, fmaf(glb1, lb1, gb));
    oa = fmaf(g0.x, o0.x, fmaf(g0.y, o0.y, oa));
    ob = fmaf(g1.x, o1.x, fmaf(g1.y, o1.y, ob));
    // dnum[t][e] at chunk c / 8, element c % 8
    const int ch = c >> 3, el = c & 7;
    *reinterpret_cast<uint32_t*>(dn + swz(ra, ch) + 2 * el) = fo_pack2(gla0 * ia, gla1 * ia);
    *reinterpret_cast<uint32_t*>(dn + swz(rb, ch) + 2 * el) = fo_pack2(glb0 * ib, glb1 * ib);
    *reinterpret_cast<uint32_t*>(dOs + (row0 + ra) * FD + c) = fo_pack2(al[c] * g0.x, al[c + 1] * g0.y);
    *reinterpret_cast<uint32_t*>(dOs + (row0 + rb) * FD + c) = fo_pack2(al[c] * g1.x, al[c + 1] * g1.y);
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    ga += __shfl_xor_sync(0xffffffffu, ga, o);
    gb += __shfl_xor_sync(0xffffffffu, gb, o);
    oa += __shfl_xor_sync(0xffffffffu, oa, o);
    ob += __shfl_xor_sync(0xffffffffu, ob, o);
  }
  if ((lane & 3) == 0) {
    dden[ra] = -ga * ia;
    dden[rb] = -gb * ib;
    delta_s[row0 + ra] = oa - ga;   // g·O − g_l·O_l
    delta_s[row0 + rb] = ob - gb;
  }
  __syncthreads();
  // dH_U,i[c][e] = Σ_t φq[t][c] dnum[t][e]: A[c][t] stored [t][c], B[t][e] stored [t][e]
  zero_acc(acc);
  warp_gemm<kRowsKM, kRowsKM>(acc, pq_s, dn_s, 16 * warp, lane);
  store_acc_bf16(dHU + ((size_t)bh * nb + i) * FD * FD, acc, ra, rb, lane);
  // dz_U,i[c] = Σ_t φq[t][c] dden_t
  if (tid < FD) {
    float z = 0.f;
    const int ch = tid >> 3, el = tid & 7;
    for (int t = 0; t < FT; ++t)
      z = fmaf(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(pq + swz(t, ch) + 2 * el)), dden[t], z);
    dzU[((size_t)bh * nb + i) * FD + tid] = z;
  }
  // dφq[t][c] = Σ_e dnum[t][e] H_U[c][e] + z_U[c] dden_t: A = dnum [t][e], B[e][c] = H_U[c][e] stored [c][e]
  zero_acc(acc);
  warp_gemm<kRowsMK, kRowsMK>(acc, dn_s, hu_s, 16 * warp, lane);
  const float da = dden[ra], db = dden[rb];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int c = 8 * nt + 2 * (lane & 3);
    const float2 q0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Q + (row0 + ra) * FD + c));
    const float2 q1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Q + (row0 + rb) * FD + c));
    *reinterpret_cast<float2*>(dQ + (row0 + ra) * FD + c) =
        make_float2(q0.x > 0.f ? fmaf(zu[c], da, acc[nt][0]) : 0.f, q0.y > 0.f ? fmaf(zu[c + 1], da, acc[nt][1]) : 0.f);
    *reinterpret_cast<float2*>(dQ + (row0 + rb) * FD + c) =
        make_float2(q1.x > 0.f ? fmaf(zu[c], db, acc[nt][2]) : 0.f, q1.y > 0.f ? fmaf(zu[c + 1], db, acc[nt][3]) : 0.f);
  }
}

// dH_tot[bh] = Σ_i dH_U,i and dz_tot[bh] = Σ_i dz_U,i, in query-block order
__global__ void lin_tot_kernel(const __nv_bfloat16* __restrict__ dHU, const float* __restrict__ dzU, int nqb,
                               float* __restrict__ dHtot, float* __restrict__ dztot) {
  const int bh = blockIdx.y;
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x < FD * FD) {
    float s = 0.f;
    for (int i = 0; i < nqb; ++i) s += __bfloat162float(dHU[((size_t)bh * nqb + i) * FD * FD + x]);
    dHtot[(size_t)bh * FD * FD + x] = s;
  }
  if (x < FD) {
    float z = 0.f;
    for (int i = 0; i < nqb; ++i) z += dzU[((size_t)bh * nqb + i) * FD + x];
    dztot[(size_t)bh * FD + x] = z;
  }
}

// Per key block j: dh_j = dH_tot − Σ_{i selected j} dH_U,i, dz_j likewise;
// dK += 1[k > 0] ⊙ (dh_j v + dz_j), dV += dh_jᵀ φ(k).
__global__ void __launch_bounds__(kFoThreads)
lin_kv_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V, int N,
              const int32_t* __restrict__ offs, const int32_t* __restrict__ list, int topk,
              const __nv_bfloat16* __restrict__ dHU, const float* __restrict__ dzU, const float* __restrict__ dHtot,
              const float* __restrict__ dztot, float* __restrict__ dK, float* __restrict__ dV) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const int j = blockIdx.x, bh = blockIdx.y, nb = N / FT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t row0 = (size_t)bh * N + (size_t)j * FT;
  const int32_t* off = offs + (size_t)bh * (nb + 1);
  const int32_t* lst = list + (size_t)bh * nb * (topk > 0 ? topk : 1);
  const int i0 = off[j], i1 = off[j + 1];
  uint8_t* dh = fsm;                          // dh_j [c][e]
  uint8_t* at = fsm + kTileB;                 // V, then φ(K)
  float* dz = reinterpret_cast<float*>(fsm + 2 * kTileB);
  int* ids = reinterpret_cast<int*>(dz + FD);   // [i1 - i0] the query blocks that selected j
  stage_bf16(at, V + row0 * FD);
  for (int x = tid; x < i1 - i0; x += kFoThreads) ids[x] = lst[i0 + x];
  __syncthreads();
  {
    float a[64];
    sub_matrices(a, dHtot + (size_t)bh * FD * FD, dHU + (size_t)bh * nb * FD * FD, ids, i1 - i0, tid);
    store_entries(dh, a, tid);
    if (tid < FD) {
      float z = dztot[(size_t)bh * FD + tid];
      for (int s2 = 0; s2 < i1 - i0; ++s2) z -= dzU[((size_t)bh * nb + ids[s2]) * FD + tid];
      dz[tid] = z;
    }
  }
  fo_cp_wait_all();
  __syncthreads();
  const uint32_t dh_s = (uint32_t)__cvta_generic_to_shared(dh), at_s = (uint32_t)__cvta_generic_to_shared(at);
  const int ra = 16 * warp + (lane >> 2), rb = ra + 8;
  float acc[16][4];
  zero_acc(acc);
  // dφk[n][c] = Σ_e v[n][e] dh[c][e] + dz[c]: A = V [n][e], B[e][c] = dh[c][e] stored [c][e]
  warp_gemm<kRowsMK, kRowsMK>(acc, at_s, dh_s, 16 * warp, lane);
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int c = 8 * nt + 2 * (lane & 3);
    const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(K + (row0 + ra) * FD + c));
    const float2 k1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(K + (row0 + rb) * FD + c));
    float2* pa = reinterpret_cast<float2*>(dK + (row0 + ra) * FD + c);
    float2* pb = reinterpret_cast<float2*>(dK + (row0 + rb) * FD + c);
    float2 xa = *pa, xb = *pb;
    xa.x += k0.x > 0.f ? acc[nt][0] + dz[c] : 0.f;
    xa.y += k0.y > 0.f ? acc[nt][1] + dz[c + 1] : 0.f;
    xb.x += k1.x > 0.f ? acc[nt][2] + dz[c] : 0.f;
    xb.y += k1.y > 0.f ? acc[nt][3] + dz[c + 1] : 0.f;
    *pa = xa;
    *pb = xb;
  }
  __syncthreads();
  stage_relu(at, K + row0 * FD);
  __syncthreads();
  zero_acc(acc);
  // dv[n][e] = Σ_c φk[n][c] dh[c][e]: A = φK [n][c], B[c][e] stored [c][e] (k rows)
  warp_gemm<kRowsMK, kRowsKM>(acc, at_s, dh_s, 16 * warp, lane);
  add_rows(dV + row0 * FD, acc, ra, rb, lane, 1.0f, 1.0f);
}

}  // namespace

size_t bwd_lin_bytes(const sa_shape& s) {
  const size_t BH = (size_t)s.B * s.H, nb = (size_t)(s.N / FT);
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return a256(BH * nb * FD * FD * 2) +            // h_j (bf16)
         a256(BH * nb * FD * FD * 2) +            // dH_U,i (bf16)
         a256(BH * nb * FD * 4) +                 // dz_U,i
         a256(BH * s.N * 4) +                     // δ_s
         a256(BH * s.N * FD * 2) +                // α⊙dO (bf16)
         a256(BH * FD * FD * 4) + a256(BH * FD * 4);   // Σ_i dH_U,i, Σ_i dz_U,i
}

sa_status bwd_linear_mix(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                         const sa_shape& s, const int32_t* block_idx, int topk, const float* alpha,
                         const sa_block_stats& st, float scale, float* dQ, float* dK, float* dV, float* lse2,
                         float* delta, const int32_t* offs, const int32_t* list, float* part, char* lin_ws,
                         cudaStream_t stream) {
  typedef __nv_bfloat16 bf;
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t BH = (size_t)s.B * s.H, nb = (size_t)(s.N / FT);
  char* p = lin_ws;
  bf* hblk = reinterpret_cast<bf*>(p);
  p += a256(BH * nb * FD * FD * 2);
  bf* dHU = reinterpret_cast<bf*>(p);
  p += a256(BH * nb * FD * FD * 2);
  float* dzU = reinterpret_cast<float*>(p);
  p += a256(BH * nb * FD * 4);
  float* delta_s = reinterpret_cast<float*>(p);
  p += a256(BH * s.N * 4);
  bf* dOs = reinterpret_cast<bf*>(p);
  p += a256(BH * s.N * FD * 2);
  float* dHtot = reinterpret_cast<float*>(p);
  p += a256(BH * FD * FD * 4);
  float* dztot = reinterpret_cast<float*>(p);
  const bf* q = static_cast<const bf*>(Q);
  const bf* k = static_cast<const bf*>(K);
  const bf* v = static_cast<const bf*>(V);
  const bf* o = static_cast<const bf*>(O);
  const bf* g = static_cast<const bf*>(dO);
  const dim3 grid((unsigned)nb, (unsigned)BH);
  const size_t smem2 = 2 * kTileB, smemq = 3 * kTileB + sizeof(float) * (FD + 2 * FT) + sizeof(int) * nb,
               smemkv = 2 * kTileB + sizeof(float) * FD + sizeof(int) * nb;
  if (cudaFuncSetAttribute(lin_hblk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) !=
          cudaSuccess ||
      cudaFuncSetAttribute(lin_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemq) != cudaSuccess ||
      cudaFuncSetAttribute(lin_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemkv) != cudaSuccess)
    return launch_status("cudaFuncSetAttribute(linear-mix backward kernels)");
  const bool lin = topk < (int)nb;
  if (lin) {
    lin_hblk_kernel<<<grid, kFoThreads, smem2, stream>>>(k, v, s.N, hblk);
    sa_status r = launch_status("lin_hblk_kernel");
    if (r != SA_OK) return r;
  }
  lin_q_kernel<<<grid, kFoThreads, smemq, stream>>>(q, o, g, alpha, s.H, s.N, block_idx, topk, st.htot, st.ztot,
                                                    st.zrelu, hblk, delta_s, dOs, dHU, dzU, dQ);
  sa_status r = launch_status("lin_q_kernel");
  if (r != SA_OK) return r;
  // the softmax branch: the drop backward of α⊙dO with δ_s, its dQ added to the
  // linear branch's (without a selected block it has no keys and no gradients)
  if (topk > 0) {
    const BwdTailTerms tt{nullptr, nullptr, nullptr, delta_s, true};
    r = bwd_tc(Q, K, V, O, dOs, s, block_idx, topk, false, st, scale, dQ, dK, dV, nullptr, lse2, delta, offs, list,
               part, stream, &tt);
  } else {
    const size_t bytes = BH * s.N * FD * sizeof(float);
    r = (cudaMemsetAsync(dK, 0, bytes, stream) == cudaSuccess && cudaMemsetAsync(dV, 0, bytes, stream) == cudaSuccess)
            ? SA_OK
            : launch_status("cudaMemsetAsync(dK, dV)");
  }
  if (r != SA_OK || !lin) return r;
  lin_tot_kernel<<<dim3(FD * FD / 256, (unsigned)BH), 256, 0, stream>>>(dHU, dzU, (int)nb, dHtot, dztot);
  r = launch_status("lin_tot_kernel");
  if (r != SA_OK) return r;
  lin_kv_kernel<<<grid, kFoThreads, smemkv, stream>>>(k, v, s.N, offs, list, topk, dHU, dzU, dHtot, dztot, dK, dV);
  return launch_status("lin_kv_kernel");
}

}  // namespace sa
