// decode.cu -- one-token step of the selective scan for sm_100a.
//
// "Axon-SSM: selective state space model", "Autoregressive decoding": the new
// token is appended to conv_cache (the last K-1 raw x rows), the conv yields
// one output, and exactly one scan step runs from the carried ssm_state; both
// caches are updated in place.
//
// The step is bound by the fp32 state stream (64 B read + 64 B written per
// channel). Four lanes share a channel and each moves a 16-byte quarter of its
// state, so a warp covers 8 channels x 64 B = 512 contiguous bytes per access.
// The per-channel scalar work (conv, SiLU, dt, SiLU(z)) is repeated by the
// four lanes rather than exchanged: the SM has ample ALU slack at this
// arithmetic intensity.
#include <cuda_bf16.h>

#include "ssm_internal.h"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kDecodeThreads = 256;

template <typename T, bool ZOH>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const KernelArgs a) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * kDecodeThreads + threadIdx.x;
  const int q = static_cast<int>(gid & 3);  // state quarter
  const int64_t ch = gid >> 2;              // seq * E + e
  // b*E*4 is a multiple of 32 (E % 8 == 0), so whole warps leave together.
  if (ch >= a.batch * a.E) return;
  const int64_t seq = ch / a.E;
  const int64_t e = ch - seq * a.E;

  T* cache = static_cast<T*>(a.conv_cache_out);  // in-out
  const T* x = static_cast<const T*>(a.x);
  const T* z = static_cast<const T*>(a.z);
  const T c0 = cache[(seq * 3 + 0) * a.E + e];
  const T c1 = cache[(seq * 3 + 1) * a.E + e];
  const T c2 = cache[(seq * 3 + 2) * a.E + e];
  const T xt = x[seq * a.s.x_seq + e];
  const float zt = IO<T>::to_f(z[seq * a.s.z_seq + e]);

  const float conv = fmaf(a.conv_w[e * 4 + 3], IO<T>::to_f(xt),
                          fmaf(a.conv_w[e * 4 + 2], IO<T>::to_f(c2),
                               fmaf(a.conv_w[e * 4 + 1], IO<T>::to_f(c1),
                                    fmaf(a.conv_w[e * 4 + 0], IO<T>::to_f(c0), a.conv_b[e]))));
  const float u = silu(conv);
  const float dt = dt_of(fmaf(a.dt_raw[seq * a.s.dt_seq], a.w_dt[e], a.dt_bias[e]), a.dt_min, a.dt_max);
  const float zg = silu(zt);

  float4* hp = reinterpret_cast<float4*>(a.ssm_state_out + ch * 16 + 4 * q);
  float4 hv = *hp;
  const float4 Bv = *reinterpret_cast<const float4*>(a.B + seq * a.s.bc_seq + 4 * q);
  const float4 Cv = *reinterpret_cast<const float4*>(a.C + seq * a.s.bc_seq + 4 * q);
  float h[4] = {hv.x, hv.y, hv.z, hv.w};
  const float bb[4] = {Bv.x, Bv.y, Bv.z, Bv.w};
  const float cc[4] = {Cv.x, Cv.y, Cv.z, Cv.w};
  float yp = 0.0f;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const float A = -expf(a.A_log[e * 16 + 4 * q + s]);
    float dA, coef;
    if constexpr (ZOH) {
      const float xa = dt * A;
      dA = ex2_approx(xa * kLog2e);
      coef = expm1_nonpos(xa, dA) / A * u;
    } else {
      dA = ex2_approx(dt * (A * kLog2e));
      coef = dt * u;
    }
    h[s] = fmaf(dA, h[s], coef * bb[s]);
    yp = fmaf(cc[s], h[s], yp);
  }
  yp += __shfl_xor_sync(0xffffffffu, yp, 1);
  yp += __shfl_xor_sync(0xffffffffu, yp, 2);
  *hp = make_float4(h[0], h[1], h[2], h[3]);
  __syncwarp();  // every lane of the channel has read the old cache rows
  if (q == 0) static_cast<T*>(a.y)[seq * a.s.y_seq + e] = IO<T>::from_f((yp + a.D[e] * u) * zg);
  if (q == 1) cache[(seq * 3 + 0) * a.E + e] = c1;
  if (q == 2) cache[(seq * 3 + 1) * a.E + e] = c2;
  if (q == 3) cache[(seq * 3 + 2) * a.E + e] = xt;
}

template <typename T, bool ZOH>
cudaError_t launch(const KernelArgs& a, cudaStream_t st) {
  const int64_t threads = a.batch * a.E * 4;
  const int64_t blocks = (threads + kDecodeThreads - 1) / kDecodeThreads;
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
