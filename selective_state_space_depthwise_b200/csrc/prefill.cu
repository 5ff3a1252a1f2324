// prefill.cu -- full-sequence selective scan for sm_100a.
//
// One fused kernel computes, for a tile of NCH channels of one sequence and
// the whole length L, the block core of "Axon-SSM: selective state space
// model" ("Algorithm" diagram): causal depthwise conv (K=4) + SiLU, dt =
// clip(softplus(dt_raw*w_dt + dt_bias)), dA = exp(dt*A) with A = -exp(A_log),
// the scan h = dA*h + dt*B*u (the _ssm_fma leaf of "JIT-compiled kernels"),
// y = C.h + D*u and the gate y*SiLU(z). dA, dB and h never reach HBM: the 16
// states of a channel stay in registers for the whole walk over L.
//
// Work split. G threads share a channel and hold 16/G states each. Tokens are
// processed in rounds of G: in a round, thread j does the per-token work (conv,
// SiLU, dt, SiLU(z)) of token j, the group exchanges dt and dt*u by shuffles,
// every thread advances its states through the G tokens in order, and the
// partial readouts are reduce-scattered so that thread j ends with the full
// C.h of token j. G > 1 gives more warps when b*E is small (b = 1 shapes)
// without splitting L.
//
// Data movement. L is walked in stages of kTok tokens through a kStages-deep
// ring in shared memory filled by cp.async: the x tile carries a 3-row halo
// (the conv history; zeros or conv_cache_in before token 0), B and C (shared by
// all channels) and dt_raw are staged once per CTA. Output tiles go through
// shared memory and leave as 16-byte stores. Tokens past L are zero-filled and
// given dt = 0, which leaves the states unchanged.
#include <cuda_bf16.h>

#include "ssm_internal.h"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kTok = 64;    // tokens per pipeline stage
constexpr int kStages = 3;  // ring depth

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes < 16 zero-fills the rest.
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_4(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Shared-memory layout of one pipeline stage (byte offsets, all 16-aligned).
template <typename T, int NCH>
struct Stage {
  static constexpr int kXRows = kTok + 3;
  static constexpr int kRow = NCH * static_cast<int>(sizeof(T));  // bytes per token row
  static_assert(kRow % 16 == 0, "a channel tile row must be a whole number of 16-byte chunks");
  static constexpr int kX = 0;
  static constexpr int kZ = kX + kXRows * kRow;
  static constexpr int kB = kZ + kTok * kRow;
  static constexpr int kC = kB + kTok * 16 * 4;
  static constexpr int kD = kC + kTok * 16 * 4;
  static constexpr int kBytes = kD + kTok * 4;
  static constexpr int kYBytes = kTok * kRow;
  static constexpr int kTotal = kStages * kBytes + kYBytes;
};

// Issue the cp.async copies of stage [t0, t0 + kTok) of sequence `seq`,
// channels [e0, e0 + NCH).
template <typename T, int NCH, int NT>
__device__ __forceinline__ void load_stage(unsigned char* st, const KernelArgs& a, int64_t seq, int64_t e0,
                                           int64_t t0, int tid) {
  using S = Stage<T, NCH>;
  constexpr int EPC = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte chunk
  constexpr int CPR = NCH / EPC;                          // chunks per token row
  const T* x = static_cast<const T*>(a.x);
  const T* z = static_cast<const T*>(a.z);
  const T* hist = static_cast<const T*>(a.conv_cache_in);
  for (int i = tid; i < S::kXRows * CPR; i += NT) {
    const int r = i / CPR, q = i % CPR;
    const int64_t t = t0 - 3 + r;
    const int64_t e = e0 + q * EPC;
    const void* src = a.x;
    int bytes = 0;
    if (e < a.E) {
      if (t >= 0 && t < a.L) {
        src = x + seq * a.s.x_seq + t * a.s.x_tok + e;
        bytes = 16;
      } else if (t < 0 && hist != nullptr) {
        src = hist + (seq * 3 + (3 + t)) * a.E + e;
        bytes = 16;
      }
    }
    cp_async_16(st + S::kX + r * S::kRow + q * 16, src, bytes);
  }
  for (int i = tid; i < kTok * CPR; i += NT) {
    const int r = i / CPR, q = i % CPR;
    const int64_t t = t0 + r;
    const int64_t e = e0 + q * EPC;
    const bool ok = t < a.L && e < a.E;
    cp_async_16(st + S::kZ + r * S::kRow + q * 16, ok ? z + seq * a.s.z_seq + t * a.s.z_tok + e : a.z, ok ? 16 : 0);
  }
  for (int i = tid; i < kTok * 4; i += NT) {
    const int r = i >> 2, q = i & 3;
    const int64_t t = t0 + r;
    const bool ok = t < a.L;
    const int64_t off = seq * a.s.bc_seq + t * a.s.bc_tok + 4 * q;
    cp_async_16(st + S::kB + (r * 16 + 4 * q) * 4, ok ? a.B + off : a.B, ok ? 16 : 0);
    cp_async_16(st + S::kC + (r * 16 + 4 * q) * 4, ok ? a.C + off : a.C, ok ? 16 : 0);
  }
  for (int i = tid; i < kTok; i += NT) {
    const int64_t t = t0 + i;
    const bool ok = t < a.L;
    cp_async_4(st + S::kD + 4 * i, ok ? a.dt_raw + seq * a.s.dt_seq + t : a.dt_raw, ok ? 4 : 0);
  }
}

// Reduce-scatter over the G lanes of a group: on entry v[i] is this lane's
// partial for token i; on exit v[0] of lane j holds the group sum for token j.
template <int G, int H>
struct ReduceScatter {
  static __device__ __forceinline__ void run(float* v, int j) {
    const bool up = (j & H) != 0;
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const float send = up ? v[i] : v[i + H];
      const float keep = up ? v[i + H] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, H);
    }
    ReduceScatter<G, H / 2>::run(v, j);
  }
};

template <int G>
struct ReduceScatter<G, 0> {
  static __device__ __forceinline__ void run(float*, int) {}
};

template <int K>
__device__ __forceinline__ void load_k(const float* p, float (&v)[K]) {
  if constexpr (K % 4 == 0) {
#pragma unroll
    for (int s = 0; s < K; s += 4) {
      const float4 q = *reinterpret_cast<const float4*>(p + s);
      v[s] = q.x;
      v[s + 1] = q.y;
      v[s + 2] = q.z;
      v[s + 3] = q.w;
    }
  } else if constexpr (K == 2) {
    const float2 q = *reinterpret_cast<const float2*>(p);
    v[0] = q.x;
    v[1] = q.y;
  } else {
    v[0] = *p;
  }
}

template <typename T, int G, int NCH, bool ZOH>
__global__ void __launch_bounds__(NCH* G) prefill_kernel(const KernelArgs a) {
  constexpr int NT = NCH * G;
  constexpr int K = 16 / G;  // states per thread
  using S = Stage<T, NCH>;
  constexpr int EPC = 16 / static_cast<int>(sizeof(T));
  constexpr int CPR = NCH / EPC;
  extern __shared__ __align__(128) unsigned char smem[];
  T* ys = reinterpret_cast<T*>(smem + kStages * S::kBytes);

  const int tid = threadIdx.x;
  const int c = tid / G;  // channel within the tile
  const int j = tid % G;  // state slice; also the token this lane owns in a round
  const int64_t tiles_per_seq = (a.E + NCH - 1) / NCH;
  const int64_t seq = blockIdx.x / tiles_per_seq;
  const int64_t e0 = (blockIdx.x % tiles_per_seq) * NCH;
  const int64_t e = e0 + c;
  const bool ch_ok = e < a.E;
  const int64_t ec = ch_ok ? e : a.E - 1;  // clamped index for parameter loads

  const float cw0 = a.conv_w[ec * 4 + 0], cw1 = a.conv_w[ec * 4 + 1];
  const float cw2 = a.conv_w[ec * 4 + 2], cw3 = a.conv_w[ec * 4 + 3];
  const float cb = a.conv_b[ec], wdt = a.w_dt[ec], dtb = a.dt_bias[ec], Dd = a.D[ec];
  const float lo = a.dt_min, hi = a.dt_max;
  float a2[K];  // A_n * log2(e), so that exp(dt*A_n) = 2^(dt*a2_n)
  float Av[K];  // A_n (ZOH only)
  float h[K];
#pragma unroll
  for (int s = 0; s < K; ++s) {
    const float A = -expf(a.A_log[ec * 16 + j * K + s]);
    Av[s] = A;
    a2[s] = A * kLog2e;
    h[s] = a.ssm_state_in ? a.ssm_state_in[(seq * a.E + ec) * 16 + j * K + s] : 0.0f;
  }
  (void)Av;

  const int64_t L = a.L;
  const int64_t n_stages = (L + kTok - 1) / kTok;
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < n_stages) load_stage<T, NCH, NT>(smem + s * S::kBytes, a, seq, e0, static_cast<int64_t>(s) * kTok, tid);
    cp_async_commit();
  }

  for (int64_t it = 0; it < n_stages; ++it) {
    cp_async_wait<kStages - 2>();
    __syncthreads();  // stage `it` landed for everyone; previous output tile drained
    {
      const int64_t nx = it + kStages - 1;
      if (nx < n_stages) load_stage<T, NCH, NT>(smem + (nx % kStages) * S::kBytes, a, seq, e0, nx * kTok, tid);
      cp_async_commit();
    }
    const unsigned char* st = smem + (it % kStages) * S::kBytes;
    const T* xs = reinterpret_cast<const T*>(st + S::kX);
    const T* zs = reinterpret_cast<const T*>(st + S::kZ);
    const float* Bs = reinterpret_cast<const float*>(st + S::kB);
    const float* Cs = reinterpret_cast<const float*>(st + S::kC);
    const float* Ds = reinterpret_cast<const float*>(st + S::kD);
    const int64_t t0 = it * kTok;

#pragma unroll 1
    for (int r = 0; r < kTok; r += G) {
      // Per-token work for the token this lane owns (row tl of the stage).
      const int tl = r + j;
      const float x0 = IO<T>::to_f(xs[(tl + 0) * NCH + c]);
      const float x1 = IO<T>::to_f(xs[(tl + 1) * NCH + c]);
      const float x2 = IO<T>::to_f(xs[(tl + 2) * NCH + c]);
      const float x3 = IO<T>::to_f(xs[(tl + 3) * NCH + c]);
      const float conv = fmaf(cw3, x3, fmaf(cw2, x2, fmaf(cw1, x1, fmaf(cw0, x0, cb))));
      const float u = silu(conv);
      float dt = dt_of(fmaf(Ds[tl], wdt, dtb), lo, hi);
      if (t0 + tl >= L) dt = 0.0f;  // past the end: keep the state
      const float inj = ZOH ? u : dt * u;
      const float zg = silu(IO<T>::to_f(zs[tl * NCH + c]));

      float dtv[G], injv[G], yp[G];
#pragma unroll
      for (int i = 0; i < G; ++i) {
        dtv[i] = __shfl_sync(0xffffffffu, dt, i, G);
        injv[i] = __shfl_sync(0xffffffffu, inj, i, G);
      }
#pragma unroll
      for (int i = 0; i < G; ++i) {
        float bv[K], cv[K];
        load_k<K>(Bs + (r + i) * 16 + j * K, bv);
        load_k<K>(Cs + (r + i) * 16 + j * K, cv);
        float acc = 0.0f;
#pragma unroll
        for (int s = 0; s < K; ++s) {
          float dA, coef;
          if constexpr (ZOH) {
            const float xa = dtv[i] * Av[s];
            dA = ex2_approx(xa * kLog2e);
            coef = expm1_nonpos(xa, dA) / Av[s] * injv[i];  // (e^{dt A} - 1)/A * u
          } else {
            dA = ex2_approx(dtv[i] * a2[s]);
            coef = injv[i];  // dt * u
          }
          h[s] = fmaf(dA, h[s], coef * bv[s]);
          acc = fmaf(cv[s], h[s], acc);
        }
        yp[i] = acc;
      }
      ReduceScatter<G, G / 2>::run(yp, j);
      ys[tl * NCH + c] = IO<T>::from_f((yp[0] + Dd * u) * zg);
    }
    __syncthreads();  // output tile complete
    for (int i = tid; i < kTok * CPR; i += NT) {
      const int rr = i / CPR, q = i % CPR;
      const int64_t t = t0 + rr;
      const int64_t eo = e0 + q * EPC;
      if (t < L && eo < a.E) {
        T* dst = static_cast<T*>(a.y) + seq * a.s.y_seq + t * a.s.y_tok + eo;
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(ys + rr * NCH + q * EPC);
      }
    }
  }
  cp_async_wait<0>();

  if (ch_ok) {
#pragma unroll
    for (int s = 0; s < K; ++s) a.ssm_state_out[(seq * a.E + e) * 16 + j * K + s] = h[s];
    if (j == 0) {
      // conv_cache_out = last 3 raw rows of [history, x]; read all before writing
      // (the output may alias conv_cache_in).
      const T* x = static_cast<const T*>(a.x);
      const T* hist = static_cast<const T*>(a.conv_cache_in);
      T keep[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int64_t t = L - 3 + k;
        if (t >= 0)
          keep[k] = x[seq * a.s.x_seq + t * a.s.x_tok + e];
        else
          keep[k] = hist ? hist[(seq * 3 + (3 + t)) * a.E + e] : IO<T>::from_f(0.0f);
      }
      T* out = static_cast<T*>(a.conv_cache_out);
#pragma unroll
      for (int k = 0; k < 3; ++k) out[(seq * 3 + k) * a.E + e] = keep[k];
    }
  }
}

template <typename T, int G, int NCH, bool ZOH>
cudaError_t launch_one(const KernelArgs& a, cudaStream_t st) {
  using S = Stage<T, NCH>;
  auto kern = prefill_kernel<T, G, NCH, ZOH>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
  if (err != cudaSuccess) return err;
  const int64_t tiles = a.batch * ((a.E + NCH - 1) / NCH);
  if (tiles > 0x7fffffff) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(tiles), NCH * G, S::kTotal, st>>>(a);
  return cudaGetLastError();
}

template <typename T, bool ZOH>
cudaError_t dispatch(const KernelArgs& a, PrefillShape sh, cudaStream_t st) {
#define SSM_CASE(G_, N_) \
  if (sh.G == G_ && sh.NCH == N_) return launch_one<T, G_, N_, ZOH>(a, st);
  SSM_CASE(1, 32)
  SSM_CASE(1, 64)
  SSM_CASE(2, 16)
  SSM_CASE(2, 32)
  SSM_CASE(2, 64)
  SSM_CASE(4, 8)
  SSM_CASE(4, 16)
  SSM_CASE(4, 32)
  SSM_CASE(8, 8)
  SSM_CASE(8, 16)
  SSM_CASE(8, 32)
  SSM_CASE(16, 8)
  SSM_CASE(16, 16)
  SSM_CASE(16, 32)
#undef SSM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

bool prefill_shape_supported(PrefillShape sh) {
  const int g = sh.G, n = sh.NCH;
  const bool g_ok = g == 1 || g == 2 || g == 4 || g == 8 || g == 16;
  const bool n_ok = n == 8 || n == 16 || n == 32 || n == 64;
  return g_ok && n_ok && g * n >= 32 && g * n <= 512;
}

// Enough warps to give every SM sub-partition about two, without splitting L:
// grow G (threads per channel) until b*E*G/32 reaches that, then pick the
// widest channel tile that still leaves every SM a tile.
PrefillShape choose_prefill_shape(int64_t batch, int64_t E, int64_t /*L*/, int num_sms) {
  const int64_t ch = batch * E;
  const int64_t want_threads = static_cast<int64_t>(num_sms) * 4 * 2 * 32;
  int g = 1;
  while (g < 16 && ch * g < want_threads) g *= 2;
  int n = 32;
  while (n > 8 && batch * ((E + n - 1) / n) < num_sms && n * g > 32) n /= 2;
  if (n * g < 32) n = 32 / g;
  if (n * g > 512) n = 512 / g;
  return PrefillShape{g, n};
}

cudaError_t launch_prefill(const KernelArgs& a, bool io_bf16, bool zoh, PrefillShape sh, cudaStream_t st) {
  if (!prefill_shape_supported(sh)) return cudaErrorInvalidValue;
  if (io_bf16) return zoh ? dispatch<__nv_bfloat16, true>(a, sh, st) : dispatch<__nv_bfloat16, false>(a, sh, st);
  return zoh ? dispatch<float, true>(a, sh, st) : dispatch<float, false>(a, sh, st);
}

}  // namespace ssm
