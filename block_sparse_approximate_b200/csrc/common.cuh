// Shared helpers of libsparseattn's kernels and host entry points.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/sparseattn.h"

namespace sa {

// ---------------------------------------------------------------- host side

void set_error(const std::string& msg);

inline sa_status fail(sa_status st, const std::string& msg) {
  set_error(msg);
  return st;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline sa_status launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(SA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return SA_OK;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous launch on the stream drains, so it must call pdl_wait()
// before it reads or writes anything that launch touches.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) cudaGetLastError();   // reported by the caller's status, not left pending
  return e;
}

inline size_t dtype_size(sa_dtype t) { return t == SA_FP32 ? 4 : 2; }

// Host-side validation of a prefill shape; returns SA_OK or sets the error.
sa_status check_shape(const sa_shape& s, const char* fn);

// Reads and clears the decode kernels' device error word (decode.cu).
uint32_t decode_error_take();

// The decode path's statistics pass on the tensor cores (decode_tc.cu): bf16
// kmean, kvar (and, with the zero-order tail, value means) [B·Hkv][nb][128],
// q bf16 [B][Hq][128] with Hq / Hkv <= 16; writes the group scores
// [B·Hkv][nb] and the zero-order partial states [B][Hq][nsegA][130] (one per
// 128 blocks); when each CTA holds a whole row it also writes the row's top
// `topk` indices to idx and sets *topk_done.  decode_tc_error_take() reads
// and clears its device error word.
sa_status decode_stats_tc(const __nv_bfloat16* q, const void* kmean, const void* kvar, const void* vmean, int B,
                          int Hq, int Hkv, int nb, int blk, float scale, int nsegA, bool zt, int sms,
                          float* scores, float* parta, int topk, int32_t* idx, bool* topk_done,
                          cudaStream_t stream);
uint32_t decode_tc_error_take();

// ---------------------------------------------------------------- device side

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// 2^x on the MUFU unit (PTX ex2.approx; flushes subnormal results to zero).
// Programmatic dependent launch: a kernel launched by launch_pdl() may start
// while its predecessor drains; it waits here before touching anything the
// predecessor reads or writes (a no-op for a kernel launched without it).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next launch on the stream start its CTAs (up to their pdl_wait())
// once every CTA of this grid has passed here; all of them are then resident,
// so the waiting successors cannot hold back a CTA of this grid.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// SPLA's exponential feature map φ(x) = e^x (§2.3).  Every kernel that forms
// Σ φ(k) vᵀ or φ(q)·φ(k) calls this one function, so the all-token state
// and the selected blocks' correction that is subtracted from it use the
// same values.
__device__ __forceinline__ float phi_exp(float x) { return __expf(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 8 consecutive elements of T starting at p (16-byte load for bf16, two for fp32).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float out[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float out[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float out[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

// Float -> unsigned key whose unsigned order is the float order (-0 == +0).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLinearEps = 1e-6f;

}  // namespace sa
