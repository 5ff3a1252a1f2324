// ssm_math.cuh -- fp32 device math for the selective-scan kernels (sm_100a).
//
// Transcendentals go to the SFU through the PTX approximations ex2.approx and
// rcp.approx (relative error ~2^-22). Where those lose accuracy near a
// cancellation, the functions below use series written from the mathematics:
//  - log1p on [0, 1] via log(1 + e) = 2 atanh(s), s = e / (2 + e) <= 1/3,
//    with the odd Taylor series of atanh through s^15 (truncation < 2e-9 rel.);
//  - expm1 near 0 via its Taylor series through x^5 (|x| < 1/8: < 5e-8 rel.).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// sigmoid(v) = 1 / (1 + e^-v); saturates cleanly to 0 / 1 at the extremes.
__device__ __forceinline__ float sigmoid(float v) { return rcp_approx(1.0f + ex2_approx(-v * kLog2e)); }

// SiLU(v) = v * sigmoid(v).
__device__ __forceinline__ float silu(float v) { return v * sigmoid(v); }

// log(1 + e) for e in [0, 1]: 2 * atanh(e / (2 + e)) as an odd series.
__device__ __forceinline__ float log1p_unit(float e) {
  const float s = e * rcp_approx(2.0f + e);
  const float s2 = s * s;
  float p = fmaf(s2, 1.0f / 15.0f, 1.0f / 13.0f);
  p = fmaf(s2, p, 1.0f / 11.0f);
  p = fmaf(s2, p, 1.0f / 9.0f);
  p = fmaf(s2, p, 1.0f / 7.0f);
  p = fmaf(s2, p, 1.0f / 5.0f);
  p = fmaf(s2, p, 1.0f / 3.0f);
  p = fmaf(s2, p, 1.0f);
  return 2.0f * s * p;
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(e^-|v|), overflow-free.
__device__ __forceinline__ float softplus(float v) {
  const float e = ex2_approx(-fabsf(v) * kLog2e);
  return fmaxf(v, 0.0f) + log1p_unit(e);
}

// dt = clip(softplus(v), lo, hi).
__device__ __forceinline__ float dt_of(float v, float lo, float hi) { return fminf(fmaxf(softplus(v), lo), hi); }

// e^x - 1 for x <= 0, given ex = e^x: Taylor series near 0, ex - 1 elsewhere.
__device__ __forceinline__ float expm1_nonpos(float x, float ex) {
  float p = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
  p = fmaf(x, p, 1.0f / 6.0f);
  p = fmaf(x, p, 0.5f);
  p = fmaf(x, p, 1.0f);
  const float series = x * p;
  return x > -0.125f ? series : ex - 1.0f;
}

template <typename T>
struct IO;

template <>
struct IO<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};

template <>
struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

}  // namespace ssm
