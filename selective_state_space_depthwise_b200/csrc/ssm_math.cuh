// ssm_math.cuh -- fp32 device math for the selective-scan kernels (sm_100a).
//
// Transcendentals go to the SFU through the PTX approximations ex2.approx and
// rcp.approx (relative error ~2^-22). Where those lose accuracy near a
// cancellation, the functions below use polynomials and series instead:
//  - log1p on [0, 1] as e * Q(e), Q a degree-8 polynomial whose maximum
//    relative error on [0, 1] was minimised by the Remez exchange algorithm
//    (fit_log1p_poly.py; 1.8e-7 in float32), FMA pipe only;
//  - the zero-order-hold input scale (e^x - 1)/A near 0 as dt times the
//    Taylor series of expm1(x)/x through x^4 (|x| < 1/8: < 5e-8 rel.).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

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

// Coefficients of Q, highest degree first (fit_log1p_poly.py, degree 8):
// log(1 + e) ~ e * Q(e) on [0, 1].
constexpr int kLog1pDeg = 8;
__host__ __device__ constexpr float log1p_q(int k) {
  return k == 0   ? 5.232694093e-03f
         : k == 1 ? -2.950523980e-02f
         : k == 2 ? 7.822595537e-02f
         : k == 3 ? -1.366324574e-01f
         : k == 4 ? 1.910600662e-01f
         : k == 5 ? -2.484298199e-01f
         : k == 6 ? 3.331909776e-01f
         : k == 7 ? -4.999949336e-01f
                  : 9.999999404e-01f;
}

// log(1 + e) for e in [0, 1]: e * Q(e) by Horner. No division, so no SFU work.
__device__ __forceinline__ float log1p_unit(float e) {
  float q = fmaf(e, log1p_q(0), log1p_q(1));
#pragma unroll
  for (int k = 2; k <= kLog1pDeg; ++k) q = fmaf(e, q, log1p_q(k));
  return e * q;
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(e^-|v|), overflow-free.
__device__ __forceinline__ float softplus(float v) {
  const float e = ex2_approx(-fabsf(v) * kLog2e);
  return fmaxf(v, 0.0f) + log1p_unit(e);
}

// dt = clip(softplus(v), lo, hi).
__device__ __forceinline__ float dt_of(float v, float lo, float hi) { return fminf(fmaxf(softplus(v), lo), hi); }

// The zero-order-hold input scale (e^x - 1) / A for x = dt A <= 0, given
// ex = e^x and rA = 1 / A: near 0 as dt (e^x - 1) / x by its Taylor series
// (dt (1 + x/2 + x^2/6 + x^3/24 + x^4/120), no cancellation, no division),
// elsewhere (ex - 1) * rA.
__device__ __forceinline__ float zoh_scale(float x, float dt, float ex, float rA) {
  float p = fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f);
  p = fmaf(x, p, 1.0f / 6.0f);
  p = fmaf(x, p, 0.5f);
  p = fmaf(x, p, 1.0f);
  return x > -0.125f ? dt * p : (ex - 1.0f) * rA;
}

// zoh_scale of two states at once (packed f32x2; each half rounds as the
// scalar form does).
__device__ __forceinline__ uint64_t zoh_scale_pair(uint64_t x, uint64_t dt2, uint64_t ex, uint64_t rA) {
  uint64_t p = ffma2(x, pk2(1.0f / 120.0f, 1.0f / 120.0f), pk2(1.0f / 24.0f, 1.0f / 24.0f));
  p = ffma2(x, p, pk2(1.0f / 6.0f, 1.0f / 6.0f));
  p = ffma2(x, p, pk2(0.5f, 0.5f));
  p = ffma2(x, p, pk2(1.0f, 1.0f));
  float s0, s1, l0, l1, x0, x1;
  upk2(fmul2(dt2, p), s0, s1);
  upk2(fmul2(fadd2(ex, pk2(-1.0f, -1.0f)), rA), l0, l1);
  upk2(x, x0, x1);
  return pk2(x0 > -0.125f ? s0 : l0, x1 > -0.125f ? s1 : l1);
}

// 2^x for x <= 0 on the FMA pipe, for a pair of arguments (packed f32x2):
// x = n + f with n = round(x), f in [-1/2, 1/2]; 2^f by a degree-5 polynomial
// whose maximum relative error on [-1/2, 1/2] was minimised by the Remez
// exchange algorithm (fit_exp2_poly.py; 2.4e-7 in float32, on par with
// ex2.approx); 2^n is added to the exponent field. Arguments below -125 are
// clamped there (2^-125 ~ 2e-38, where the SFU version flushes to zero).
__device__ __forceinline__ uint64_t ex2_poly2(float x0, float x1) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer in the low bits
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  uint64_t x;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(x0), "f"(x1));
  uint64_t sh, t, n, f, p;
  asm("mov.b64 %0, {%1, %1};" : "=l"(sh) : "f"(kShift));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(x), "l"(sh));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(n) : "l"(t), "l"(sh));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f) : "l"(x), "l"(n));
  uint64_t c;
  asm("mov.b64 %0, {%1, %1};" : "=l"(p) : "f"(1.327647245e-03f));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(9.675540961e-03f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(5.550713092e-02f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(2.402212024e-01f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(6.931469440e-01f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(1.000000119e+00f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c));
  uint32_t t0, t1, p0, p1;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(t0), "=r"(t1) : "l"(t));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(p0), "=r"(p1) : "l"(p));
  p0 += t0 << 23;  // t's low mantissa bits hold n; shifted, they add n to p's exponent
  p1 += t1 << 23;
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(p0), "r"(p1));
  return r;
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
