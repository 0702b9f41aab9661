// common.cuh -- device helpers shared by the libssmscan kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---- MUFU approximations (hardware special-function unit) ------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float tanh_approx(float x) {
  float r;
  asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// softplus(s) = log(1 + e^s).
//  * s > 20: s (the remainder is below 3e-9 relative);
//  * s < -2: e = e^s < 0.136 and log1p(e) is the alternating series
//    e - e^2/2 + e^3/3 - ... truncated after e^9 (next term < 1.2e-9 e);
//    this keeps full relative accuracy for small steps, which the MUFU
//    logarithm near 1 would lose;
//  * otherwise: ln2 * log2(1 + e) with 1 + e >= 1.135, where the MUFU
//    logarithm's absolute error is small against the result.
__device__ __forceinline__ float softplus_f(float s) {
  const float e = ex2_approx(s * kLog2e);
  float series = 1.0f / 9.0f;
  series = fmaf(series, e, -1.0f / 8.0f);
  series = fmaf(series, e, 1.0f / 7.0f);
  series = fmaf(series, e, -1.0f / 6.0f);
  series = fmaf(series, e, 1.0f / 5.0f);
  series = fmaf(series, e, -1.0f / 4.0f);
  series = fmaf(series, e, 1.0f / 3.0f);
  series = fmaf(series, e, -1.0f / 2.0f);
  series = fmaf(series, e, 1.0f);
  series *= e;
  const float logv = kLn2 * lg2_approx(1.0f + e);
  const float r = s < -2.0f ? series : logv;
  return s > 20.0f ? s : r;
}

// silu(z) = z / (1 + e^{-z}); e^{-z} overflowing to +inf gives 0, as it should.
__device__ __forceinline__ float silu_f(float z) {
  return z * rcp_approx(1.0f + ex2_approx(-z * kLog2e));
}

__host__ __device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// ---- element types -----------------------------------------------------------
template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ---- asynchronous global -> shared copies (16 bytes, zero-filled tail) ------
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, int src_bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

}  // namespace ssm
