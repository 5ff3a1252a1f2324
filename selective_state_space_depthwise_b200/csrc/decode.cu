// decode.cu -- one-token step of the selective scan for sm_100a.
//
// "Axon-SSM: selective state space model", "Autoregressive decoding": the new
// token is appended to conv_cache (the last K-1 raw x rows), the conv yields
// one output, and exactly one scan step runs from the carried ssm_state; both
// caches are updated in place.
//
// The step is bound by the fp32 state stream: 64 B read + 64 B written per
// channel against ~12 B of everything else, so what matters is how many bytes
// each thread keeps in flight. One thread owns a channel and issues its four
// 16-byte state loads (and the A_log row) before any arithmetic; across a
// warp the state accesses cover 32 consecutive channels (2 KB). The grid's y
// dimension is the sequence, so no thread divides a flat index.
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "ssm_internal.h"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kDecodeThreads = 128;

template <typename T, bool ZOH>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const KernelArgs a, int64_t seq0) {
  const int64_t e = static_cast<int64_t>(blockIdx.x) * kDecodeThreads + threadIdx.x;
  if (e >= a.E) return;
  const int64_t seq = seq0 + blockIdx.y;
  const int64_t ch = seq * a.E + e;

  float4* hp = reinterpret_cast<float4*>(a.ssm_state_out) + ch * 4;
  float4 hv[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) hv[q] = hp[q];
  const float4* Al = reinterpret_cast<const float4*>(a.A_log) + e * 4;
  float4 al[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) al[q] = Al[q];

  T* cache = static_cast<T*>(a.conv_cache_out) + seq * 3 * a.E + e;  // in-out
  const T c0 = cache[0], c1 = cache[a.E], c2 = cache[2 * a.E];
  const T xt = static_cast<const T*>(a.x)[seq * a.s.x_seq + e];
  const float zt = IO<T>::to_f(static_cast<const T*>(a.z)[seq * a.s.z_seq + e]);
  const float4 cw = reinterpret_cast<const float4*>(a.conv_w)[e];
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
      const float4 b = Bq[q], cc = Cq[q];
      const float alv[4] = {al[q].x, al[q].y, al[q].z, al[q].w};
      const float bv[4] = {b.x, b.y, b.z, b.w}, cv[4] = {cc.x, cc.y, cc.z, cc.w};
      float hs[4] = {hv[q].x, hv[q].y, hv[q].z, hv[q].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float A = -ex2_approx(alv[i] * kLog2e);  // A = -exp(A_log)
        const float xa = dt * A;
        const float dA = ex2_approx(xa * kLog2e);
        hs[i] = fmaf(dA, hs[i], expm1_nonpos(xa, dA) / A * u * bv[i]);
        yl = fmaf(cv[i], hs[i], yl);
      }
      hv[q] = make_float4(hs[0], hs[1], hs[2], hs[3]);
    }
  } else {
    // exp(dt*A) = 2^(dt * A * log2e) with A * log2e = -2^(A_log * log2e) * log2e
    const uint64_t dt2 = pk2(-dt * kLog2e, -dt * kLog2e), dtu2 = pk2(dt * u, dt * u);
    uint64_t acc = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 b = Bq[q], cc = Cq[q];
      float x0, x1, x2, x3;
      upk2(fmul2(dt2, pk2(ex2_approx(al[q].x * kLog2e), ex2_approx(al[q].y * kLog2e))), x0, x1);
      upk2(fmul2(dt2, pk2(ex2_approx(al[q].z * kLog2e), ex2_approx(al[q].w * kLog2e))), x2, x3);
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
  cache[0] = c1;
  cache[a.E] = c2;
  cache[2 * a.E] = xt;
}

template <typename T, bool ZOH>
cudaError_t launch(const KernelArgs& a, cudaStream_t st) {
  const int64_t bx = (a.E + kDecodeThreads - 1) / kDecodeThreads;
  if (bx > 0x7fffffff) return cudaErrorInvalidConfiguration;
  for (int64_t s0 = 0; s0 < a.batch; s0 += 65535) {  // grid.y is limited to 65535
    const unsigned by = static_cast<unsigned>(a.batch - s0 < 65535 ? a.batch - s0 : 65535);
    decode_kernel<T, ZOH><<<dim3(static_cast<unsigned>(bx), by), kDecodeThreads, 0, st>>>(a, s0);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const KernelArgs& a, bool io_bf16, bool zoh, cudaStream_t st) {
  if (io_bf16) return zoh ? launch<__nv_bfloat16, true>(a, st) : launch<__nv_bfloat16, false>(a, st);
  return zoh ? launch<float, true>(a, st) : launch<float, false>(a, st);
}

}  // namespace ssm
