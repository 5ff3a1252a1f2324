// pipe_rates.cu -- B200 unit rates behind the prefill roofline (standalone probe).
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o pipe_rates pipe_rates.cu && ./pipe_rates
//
// Three tables, each from clock64() deltas of blocks that are all resident at
// once (the slowest block's cycles divide the work of all of them):
//  1. lane-operations per clock per SM of the pipes the selective scan uses
//     (SFU ex2/rcp/lg2, FP32 FMA, packed f32x2 FMA), 16 warps/SM,
//     8 independent chains per thread;
//  2. SFU ex2 rate against warps per SM and independent chains per thread,
//     with and without FMA work between the exponentials (latency hiding);
//  3. warp-instructions per clock per SM of shared-memory loads and shuffles
//     by access pattern (broadcast, lane-distinct, warp-uniform addresses).
// Every shared-memory index is masked into its 4096-float array and every
// output buffer is sized for the largest grid used.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#define CK(x)                                                                         \
  do {                                                                                \
    cudaError_t e_ = (x);                                                             \
    if (e_ != cudaSuccess) {                                                          \
      std::printf("CUDA error %s at line %d\n", cudaGetErrorString(e_), __LINE__);    \
      std::exit(1);                                                                   \
    }                                                                                 \
  } while (0)

static long long max_cycles(const long long* dcyc, int n) {
  std::vector<long long> c(n);
  CK(cudaMemcpy(c.data(), dcyc, n * sizeof(long long), cudaMemcpyDeviceToHost));
  return *std::max_element(c.begin(), c.end());
}

// ------------------------------------------------------------ 1. pipes ---
enum PipeOp { kEx2, kRcp, kLg2, kFfma, kFfma2 };
constexpr int kChains = 8;

template <PipeOp OP>
__global__ void pipe_kernel(float* out, int iters, long long* cyc) {
  float x[kChains];
  uint64_t p[kChains];
  uint32_t u[kChains];
  uint64_t a2, b2;
  asm("mov.b64 %0, {%1, %1};" : "=l"(a2) : "f"(0.999f));
  asm("mov.b64 %0, {%1, %1};" : "=l"(b2) : "f"(0.001f));
#pragma unroll
  for (int c = 0; c < kChains; ++c) {
    x[c] = 0.5f + 0.01f * c + threadIdx.x * 1e-5f;
    asm("mov.b64 %0, {%1, %2};" : "=l"(p[c]) : "f"(x[c]), "f"(x[c] + 0.1f));
    u[c] = threadIdx.x + c;
  }
  __syncthreads();
  const long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
#pragma unroll
      for (int c = 0; c < kChains; ++c) {
        if (OP == kEx2) asm volatile("ex2.approx.ftz.f32 %0, %0;" : "+f"(x[c]));
        if (OP == kRcp) asm volatile("{ .reg .f32 t; add.f32 t, %0, 0f3F800000; rcp.approx.ftz.f32 %0, t; }" : "+f"(x[c]));
        if (OP == kLg2) asm volatile("{ .reg .f32 t; add.f32 t, %0, 0f40000000; lg2.approx.ftz.f32 %0, t; }" : "+f"(x[c]));
        if (OP == kFfma) asm volatile("fma.rn.f32 %0, %0, 0f3F7FBE77, 0f3A83126F;" : "+f"(x[c]));
        if (OP == kFfma2) asm volatile("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(p[c]) : "l"(a2), "l"(b2));
      }
    }
  }
  const long long t1 = clock64();
  __syncthreads();
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
  float s = 0.0f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p[c]));
    s += x[c] + lo + hi + static_cast<float>(u[c]);
  }
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

template <PipeOp OP>
static void run_pipe(const char* name, double lanes_per_op, int nsm, float* dout, long long* dcyc) {
  const int threads = 256, blocks = nsm * 2, iters = 2048;  // 16 warps per SM
  pipe_kernel<OP><<<blocks, threads>>>(dout, 16, dcyc);
  CK(cudaDeviceSynchronize());
  pipe_kernel<OP><<<blocks, threads>>>(dout, iters, dcyc);
  CK(cudaDeviceSynchronize());
  const long long mx = max_cycles(dcyc, blocks);
  const double ops = static_cast<double>(blocks) * threads * iters * 4 * kChains * lanes_per_op;
  std::printf("| %-26s | %7.2f |\n", name, ops / nsm / static_cast<double>(mx));
}

// ---------------------------------------------- 2. SFU latency hiding ---
template <int I, int F>
__global__ void ex2_ilp_kernel(float* out, int iters, long long* cyc) {
  float x[I], y[I];
#pragma unroll
  for (int c = 0; c < I; ++c) x[c] = y[c] = 0.5f + 0.01f * c + threadIdx.x * 1e-5f;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < I; ++c) {
      asm volatile("{ .reg .f32 t; mul.f32 t, %0, 0fBF000000; ex2.approx.ftz.f32 %0, t; }" : "+f"(x[c]));
#pragma unroll
      for (int f = 0; f < F; ++f) asm volatile("fma.rn.f32 %0, %0, 0f3F7FBE77, %1;" : "+f"(y[c]) : "f"(x[c]));
    }
  }
  const long long t1 = clock64();
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
  float s = 0.0f;
#pragma unroll
  for (int c = 0; c < I; ++c) s += x[c] + y[c];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

template <int I, int F>
static double run_ex2_ilp(int nsm, int warps_per_sm, float* dout, long long* dcyc) {
  const int blocks = nsm * warps_per_sm, iters = 16384 / I;  // one warp per block
  ex2_ilp_kernel<I, F><<<blocks, 32>>>(dout, 8, dcyc);
  CK(cudaDeviceSynchronize());
  ex2_ilp_kernel<I, F><<<blocks, 32>>>(dout, iters, dcyc);
  CK(cudaDeviceSynchronize());
  const long long mx = max_cycles(dcyc, blocks);
  return static_cast<double>(blocks) * 32 * iters * I / nsm / static_cast<double>(mx);
}

// -------------------------------------------- 3. shared-memory delivery ---
enum SmemPattern {
  kLds32Bcast,       // every lane the same address, changing with the loop counter
  kLds64Bcast,
  kLds128Bcast,
  kLds128Quads,      // four 16-byte addresses per warp (lane & 3)
  kLds128Distinct,   // 32 consecutive 16-byte words
  kLds64Distinct,    // 32 consecutive 8-byte words
  kShflBcast,        // shfl.idx from lane 0
  kShflQuads,        // shfl.idx from lane & 3
  kLds32WarpTid,     // per-warp address from tid >> 5
  kLds32WarpShfl,    // per-warp address from a shuffled (provably uniform) warp index
  kLds128WarpTid,
  kLds128WarpShfl,
  kLds32Cta,         // one address per CTA from blockIdx (uniform register, same in every warp)
  kLds128Cta,
  kLds32SameTid,     // the same address in every warp, but from a per-thread register (tid >> 9 == 0)
  kLds128SameTid,
};

template <SmemPattern P>
__global__ void smem_kernel(float* out, int iters, long long* cyc) {
  __shared__ __align__(16) float s[4096];
  for (int i = threadIdx.x; i < 4096; i += blockDim.x) s[i] = i * 0.5f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wtid = threadIdx.x >> 5;
  const int wshf = __shfl_sync(0xffffffffu, wtid, 0);
  float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
  const float v = lane * 1.0f;
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int base = ((it * 16 + u) * 32) & 2047;  // multiple of 32 floats, < 2048
      if (P == kLds32Bcast) a0 += s[base];
      if (P == kLds64Bcast) {
        const float2 q = *reinterpret_cast<const float2*>(s + base);
        a0 += q.x, a1 += q.y;
      }
      if (P == kLds128Bcast) {
        const float4 q = *reinterpret_cast<const float4*>(s + base);
        a0 += q.x, a1 += q.y, a2 += q.z, a3 += q.w;
      }
      if (P == kLds128Quads) {
        const float4 q = *reinterpret_cast<const float4*>(s + base + 4 * (lane & 3));
        a0 += q.x, a1 += q.y, a2 += q.z, a3 += q.w;
      }
      if (P == kLds128Distinct) {
        const float4 q = *reinterpret_cast<const float4*>(s + ((base + 4 * lane) & 4095));
        a0 += q.x, a1 += q.y, a2 += q.z, a3 += q.w;
      }
      if (P == kLds64Distinct) {
        const float2 q = *reinterpret_cast<const float2*>(s + ((base + 2 * lane) & 4095));
        a0 += q.x, a1 += q.y;
      }
      if (P == kShflBcast) a0 += __shfl_sync(0xffffffffu, v + u, 0);
      if (P == kShflQuads) a0 += __shfl_sync(0xffffffffu, v + u, lane & 3);
      if (P == kLds32WarpTid) a0 += s[(base + 64 * wtid) & 4095];
      if (P == kLds32WarpShfl) a0 += s[(base + 64 * wshf) & 4095];
      if (P == kLds128WarpTid) {
        const float4 q = *reinterpret_cast<const float4*>(s + ((base + 64 * wtid) & 4095));
        a0 += q.x, a1 += q.y, a2 += q.z, a3 += q.w;
      }
      if (P == kLds128WarpShfl) {
        const float4 q = *reinterpret_cast<const float4*>(s + ((base + 64 * wshf) & 4095));
        a0 += q.x, a1 += q.y, a2 += q.z, a3 += q.w;
      }
      if (P == kLds32Cta) a0 += s[(base + 64 * (blockIdx.x & 7)) & 4095];
      if (P == kLds128Cta) {
        const float4 q = *reinterpret_cast<const float4*>(s + ((base + 64 * (blockIdx.x & 7)) & 4095));
        a0 += q.x, a1 += q.y, a2 += q.z, a3 += q.w;
      }
      if (P == kLds32SameTid) a0 += s[(base + 64 * (threadIdx.x >> 9)) & 4095];
      if (P == kLds128SameTid) {
        const float4 q = *reinterpret_cast<const float4*>(s + ((base + 64 * (threadIdx.x >> 9)) & 4095));
        a0 += q.x, a1 += q.y, a2 += q.z, a3 += q.w;
      }
    }
  }
  const long long t1 = clock64();
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
  out[blockIdx.x * blockDim.x + threadIdx.x] = a0 + a1 + a2 + a3;
}

template <SmemPattern P>
static void run_smem(const char* name, int nsm, float* dout, long long* dcyc) {
  const int iters = 2048;  // one block of 16 warps per SM
  smem_kernel<P><<<nsm, 512>>>(dout, 8, dcyc);
  CK(cudaDeviceSynchronize());
  smem_kernel<P><<<nsm, 512>>>(dout, iters, dcyc);
  CK(cudaDeviceSynchronize());
  const long long mx = max_cycles(dcyc, nsm);
  std::printf("| %-44s | %6.3f |\n", name, 16.0 * iters * 16 / static_cast<double>(mx));
}

int main() {
  cudaDeviceProp prop;
  CK(cudaGetDeviceProperties(&prop, 0));
  const int nsm = prop.multiProcessorCount;
  std::printf("device %s, %d SMs, cc %d.%d\n\n", prop.name, nsm, prop.major, prop.minor);
  float* dout;
  long long* dcyc;
  CK(cudaMalloc(&dout, static_cast<size_t>(nsm) * 32 * 512 * sizeof(float)));
  CK(cudaMalloc(&dcyc, static_cast<size_t>(nsm) * 32 * sizeof(long long)));

  std::printf("| operation (16 warps/SM, 8 chains) | lane-ops/clk/SM |\n|---|---|\n");
  run_pipe<kEx2>("ex2.approx (SFU)", 1, nsm, dout, dcyc);
  run_pipe<kRcp>("rcp.approx + fadd", 1, nsm, dout, dcyc);
  run_pipe<kLg2>("lg2.approx + fadd", 1, nsm, dout, dcyc);
  run_pipe<kFfma>("fma.rn.f32", 1, nsm, dout, dcyc);
  run_pipe<kFfma2>("fma.rn.f32x2 (2 lanes/op)", 2, nsm, dout, dcyc);

  std::printf("\n| warps/SM | 1 chain | 2 chains | 4 chains | 8 chains | 8 chains + 4 FMA each |\n|---|---|---|---|---|---|\n");
  for (int w : {4, 8, 16, 32}) {
    std::printf("| %d | %.2f | %.2f | %.2f | %.2f | %.2f |\n", w, run_ex2_ilp<1, 0>(nsm, w, dout, dcyc),
                run_ex2_ilp<2, 0>(nsm, w, dout, dcyc), run_ex2_ilp<4, 0>(nsm, w, dout, dcyc),
                run_ex2_ilp<8, 0>(nsm, w, dout, dcyc), run_ex2_ilp<8, 4>(nsm, w, dout, dcyc));
  }

  std::printf("\n| shared-memory access (16 warps/SM) | warp-instr/clk/SM |\n|---|---|\n");
  run_smem<kLds32Bcast>("LDS.32 broadcast", nsm, dout, dcyc);
  run_smem<kLds64Bcast>("LDS.64 broadcast", nsm, dout, dcyc);
  run_smem<kLds128Bcast>("LDS.128 broadcast", nsm, dout, dcyc);
  run_smem<kLds128Quads>("LDS.128, 4 addresses (lane & 3)", nsm, dout, dcyc);
  run_smem<kLds128Distinct>("LDS.128 lane-distinct (512 B)", nsm, dout, dcyc);
  run_smem<kLds64Distinct>("LDS.64 lane-distinct (256 B)", nsm, dout, dcyc);
  run_smem<kShflBcast>("SHFL.IDX from lane 0", nsm, dout, dcyc);
  run_smem<kShflQuads>("SHFL.IDX from lane & 3", nsm, dout, dcyc);
  run_smem<kLds32WarpTid>("LDS.32 per-warp address from tid >> 5", nsm, dout, dcyc);
  run_smem<kLds32WarpShfl>("LDS.32 per-warp address, shuffled warp index", nsm, dout, dcyc);
  run_smem<kLds128WarpTid>("LDS.128 per-warp address from tid >> 5", nsm, dout, dcyc);
  run_smem<kLds128WarpShfl>("LDS.128 per-warp address, shuffled warp index", nsm, dout, dcyc);
  run_smem<kLds32Cta>("LDS.32 CTA-uniform address (blockIdx)", nsm, dout, dcyc);
  run_smem<kLds128Cta>("LDS.128 CTA-uniform address (blockIdx)", nsm, dout, dcyc);
  run_smem<kLds32SameTid>("LDS.32 same address, per-thread register", nsm, dout, dcyc);
  run_smem<kLds128SameTid>("LDS.128 same address, per-thread register", nsm, dout, dcyc);

  CK(cudaFree(dout));
  CK(cudaFree(dcyc));
  return 0;
}
