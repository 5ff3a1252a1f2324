// decode.cu -- one-token step of the selective scan for sm_100a.
//
// "Axon-SSM: selective state space model", "Autoregressive decoding": the new
// token is appended to conv_cache (the last K-1 raw x rows), the conv yields
// one output, and exactly one scan step runs from the carried ssm_state; both
// caches are updated in place.
//
// The step is bound by the fp32 state stream: 64 B read + 64 B written per
// channel against ~12 B of everything else. One thread owns a channel: it
// issues its four 16-byte state loads first, so every thread has its whole
// state in flight while the per-channel work (conv, SiLU, dt, SiLU(z)) runs,
// then advances the 16 states with packed f32x2 arithmetic and writes them
// back as four 16-byte stores. Across a warp the state accesses cover 32
// consecutive channels (2 KB) and x, z, y, the cache rows 64 contiguous bytes.
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "ssm_internal.h"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kDecodeThreads = 128;

template <typename T, bool ZOH>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const KernelArgs a) {
  const int64_t ch = static_cast<int64_t>(blockIdx.x) * kDecodeThreads + threadIdx.x;  // seq * E + e
  if (ch >= a.batch * a.E) return;
  const int64_t seq = ch / a.E;
  const int64_t e = ch - seq * a.E;

  float4* hp = reinterpret_cast<float4*>(a.ssm_state_out + ch * 16);
  float4 hv[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) hv[q] = hp[q];

  T* cache = static_cast<T*>(a.conv_cache_out);  // in-out
  const T c0 = cache[(seq * 3 + 0) * a.E + e];
  const T c1 = cache[(seq * 3 + 1) * a.E + e];
  const T c2 = cache[(seq * 3 + 2) * a.E + e];
  const T xt = static_cast<const T*>(a.x)[seq * a.s.x_seq + e];
  const float zt = IO<T>::to_f(static_cast<const T*>(a.z)[seq * a.s.z_seq + e]);
  const float4 cw = *reinterpret_cast<const float4*>(a.conv_w + e * 4);
  const float4* Al = reinterpret_cast<const float4*>(a.A_log + e * 16);
  const float4* Bq = reinterpret_cast<const float4*>(a.B + seq * a.s.bc_seq);
  const float4* Cq = reinterpret_cast<const float4*>(a.C + seq * a.s.bc_seq);

  const float conv = fmaf(cw.w, IO<T>::to_f(xt),
                          fmaf(cw.z, IO<T>::to_f(c2), fmaf(cw.y, IO<T>::to_f(c1), fmaf(cw.x, IO<T>::to_f(c0), a.conv_b[e]))));
  const float u = silu(conv);
  const float dt = dt_of(fmaf(a.dt_raw[seq * a.s.dt_seq], a.w_dt[e], a.dt_bias[e]), a.dt_min, a.dt_max);
  const float zg = silu(zt);

  float yl = 0.0f, yh = 0.0f;
  if constexpr (ZOH) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 al = Al[q], b = Bq[q], cc = Cq[q];
      const float alv[4] = {al.x, al.y, al.z, al.w}, bv[4] = {b.x, b.y, b.z, b.w}, cv[4] = {cc.x, cc.y, cc.z, cc.w};
      float hs[4] = {hv[q].x, hv[q].y, hv[q].z, hv[q].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float A = -expf(alv[i]);
        const float xa = dt * A;
        const float dA = ex2_approx(xa * kLog2e);
        hs[i] = fmaf(dA, hs[i], expm1_nonpos(xa, dA) / A * u * bv[i]);
        yl = fmaf(cv[i], hs[i], yl);
      }
      hv[q] = make_float4(hs[0], hs[1], hs[2], hs[3]);
    }
  } else {
    const uint64_t dt2 = pk2(dt, dt), dtu2 = pk2(dt * u, dt * u);
    uint64_t acc = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 al = Al[q], b = Bq[q], cc = Cq[q];
      // a2 = A * log2(e) = -exp(A_log) * log2(e)
      const float a0 = -expf(al.x) * kLog2e, a1 = -expf(al.y) * kLog2e;
      const float a2v = -expf(al.z) * kLog2e, a3 = -expf(al.w) * kLog2e;
      float x0, x1, x2, x3;
      upk2(fmul2(dt2, pk2(a0, a1)), x0, x1);
      upk2(fmul2(dt2, pk2(a2v, a3)), x2, x3);
      const uint64_t h01 = ffma2(pk2(ex2_approx(x0), ex2_approx(x1)), pk2(hv[q].x, hv[q].y), fmul2(dtu2, pk2(b.x, b.y)));
      const uint64_t h23 = ffma2(pk2(ex2_approx(x2), ex2_approx(x3)), pk2(hv[q].z, hv[q].w), fmul2(dtu2, pk2(b.z, b.w)));
      acc = q == 0 ? fmul2(pk2(cc.x, cc.y), h01) : ffma2(pk2(cc.x, cc.y), h01, acc);
      acc = ffma2(pk2(cc.z, cc.w), h23, acc);
      upk2(h01, hv[q].x, hv[q].y);
      upk2(h23, hv[q].z, hv[q].w);
    }
    upk2(acc, yl, yh);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) hp[q] = hv[q];
  static_cast<T*>(a.y)[seq * a.s.y_seq + e] = IO<T>::from_f((yl + yh + a.D[e] * u) * zg);
  cache[(seq * 3 + 0) * a.E + e] = c1;
  cache[(seq * 3 + 1) * a.E + e] = c2;
  cache[(seq * 3 + 2) * a.E + e] = xt;
}

template <typename T, bool ZOH>
cudaError_t launch(const KernelArgs& a, cudaStream_t st) {
  const int64_t blocks = (a.batch * a.E + kDecodeThreads - 1) / kDecodeThreads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  decode_kernel<T, ZOH><<<static_cast<unsigned>(blocks), kDecodeThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const KernelArgs& a, bool io_bf16, bool zoh, cudaStream_t st) {
  if (io_bf16) return zoh ? launch<__nv_bfloat16, true>(a, st) : launch<__nv_bfloat16, false>(a, st);
  return zoh ? launch<float, true>(a, st) : launch<float, false>(a, st);
}

}  // namespace ssm
