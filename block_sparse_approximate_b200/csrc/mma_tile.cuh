// 128 x 128 x 128 contractions on mma.sync (m16n8k16, bf16 operands, fp32
// accumulation) over tiles staged in shared memory, for the small products of
// the backward (bwd_fo.cu, bwd_lin.cu).  A tile is 128 rows of 128 bf16 (256
// bytes) with the 16-byte chunk c of row r stored at chunk c ^ (r & 7), so
// the eight rows an ldmatrix reads fall in different banks.  A CTA has 8
// warps; warp w owns output rows 16 w .. 16 w + 15 and all 128 columns.
#pragma once

#include "attn_simt.cuh"

namespace sa {
namespace mt {

constexpr int FT = 128;                      // rows per tile (= block)
constexpr int FD = 128;                      // head dim
constexpr int kFoThreads = 256;              // 8 warps, 16 output rows each
constexpr uint32_t kRowB = FD * 2;           // bytes of a bf16 row
constexpr uint32_t kTileB = FT * kRowB;      // one bf16 128 x 128 tile
constexpr int kGramRows = 2048;              // rows of one partial G

__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)r * kRowB + ((uint32_t)(c ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t fo_pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void fo_cp16(uint8_t* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void fo_cp_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
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
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Layout of an operand tile in shared memory: kRows = rows indexed by the
// product's M (or N) dimension, kCols = by its K dimension; kT = the
// transpose (rows indexed by K).
enum Lay { kRowsMK, kRowsKM };

// acc[nt] (rows m0 .. m0 + 15 of the warp, columns 8 nt .. 8 nt + 7) +=
// A (rows m0.., K = 128) · B (K = 128 x N = 128).
//   A: kRowsMK = smem [m][k] (plain ldmatrix), kRowsKM = smem [k][m] (.trans);
//   B: kRowsMK = smem [n][k] (plain), kRowsKM = smem [k][n] (.trans).
template <Lay LA, Lay LB>
__device__ __forceinline__ void warp_gemm(float (&acc)[16][4], uint32_t a_s, uint32_t b_s, int m0, int lane) {
#pragma unroll 2
  for (int ks = 0; ks < FD / 16; ++ks) {
    uint32_t a[4];
    if (LA == kRowsMK) {
      ldsm4(a, a_s + swz(m0 + (lane & 15), 2 * ks + (lane >> 4)));
    } else {
      ldsm4t(a, a_s + swz(16 * ks + (lane & 7) + 8 * ((lane >> 4) & 1), m0 / 8 + ((lane >> 3) & 1)));
    }
#pragma unroll
    for (int np = 0; np < 8; ++np) {   // n-tiles 2 np, 2 np + 1
      uint32_t b[4];
      if (LB == kRowsMK) {
        ldsm4(b, b_s + swz(16 * np + (lane & 7) + 8 * (lane >> 4), 2 * ks + ((lane >> 3) & 1)));
      } else {
        ldsm4t(b, b_s + swz(16 * ks + (lane & 15), 2 * np + (lane >> 4)));
      }
      mma16816(acc[2 * np], a, b[0], b[1]);
      mma16816(acc[2 * np + 1], a, b[2], b[3]);
    }
  }
}

__device__ __forceinline__ void zero_acc(float (&acc)[16][4]) {
#pragma unroll
  for (int nt = 0; nt < 16; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
}

// bf16 tile rows [r0, r0 + 128) of a [rows][128] array into shared memory (cp.async)
__device__ __forceinline__ void stage_bf16(uint8_t* dst, const __nv_bfloat16* src) {
  for (int o = threadIdx.x; o < FT * 16; o += kFoThreads) {
    const int r = o >> 4, c = o & 15;
    fo_cp16(dst + swz(r, c), src + (size_t)r * FD + 8 * c);
  }
}
// a float32 [128][128] matrix into a bf16 tile
__device__ __forceinline__ void stage_f32(uint8_t* dst, const float* src) {
  for (int o = threadIdx.x; o < FT * 16; o += kFoThreads) {
    const int r = o >> 4, c = o & 15;
    const float4 a = *reinterpret_cast<const float4*>(src + (size_t)r * FD + 8 * c);
    const float4 b = *reinterpret_cast<const float4*>(src + (size_t)r * FD + 8 * c + 4);
    *reinterpret_cast<uint4*>(dst + swz(r, c)) =
        make_uint4(fo_pack2(a.x, a.y), fo_pack2(a.z, a.w), fo_pack2(b.x, b.y), fo_pack2(b.z, b.w));
  }
}
// bf16 rows x_r minus the float32 row m (the block's mean), as a bf16 tile
__device__ __forceinline__ void stage_centred(uint8_t* dst, const __nv_bfloat16* src, const float* m, float mscale) {
  for (int o = threadIdx.x; o < FT * 16; o += kFoThreads) {
    const int r = o >> 4, c = o & 15;
    const uint4 x = *reinterpret_cast<const uint4*>(src + (size_t)r * FD + 8 * c);
    const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv[e]));
      w[e] = fo_pack2(f.x - mscale * m[8 * c + 2 * e], f.y - mscale * m[8 * c + 2 * e + 1]);
    }
    *reinterpret_cast<uint4*>(dst + swz(r, c)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// out[row][col] += f(row) · acc for the warp's accumulator layout
__device__ __forceinline__ void add_rows(float* base, const float (&acc)[16][4], int ra, int rb, int lane, float fa,
                                         float fb) {
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int c = 8 * nt + 2 * (lane & 3);
    float2* pa = reinterpret_cast<float2*>(base + (size_t)ra * FD + c);
    float2* pb = reinterpret_cast<float2*>(base + (size_t)rb * FD + c);
    float2 xa = *pa, xb = *pb;
    xa.x = fmaf(fa, acc[nt][0], xa.x);
    xa.y = fmaf(fa, acc[nt][1], xa.y);
    xb.x = fmaf(fb, acc[nt][2], xb.x);
    xb.y = fmaf(fb, acc[nt][3], xb.y);
    *pa = xa;
    *pb = xb;
  }
}

}  // namespace mt
}  // namespace sa
