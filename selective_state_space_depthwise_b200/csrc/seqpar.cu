// seqpar.cu -- sequence-parallel prefill: the summary of one segment of a
// sequence and the carry of summaries into the next segment.
//
// A long sequence split into segments (one per GPU, or pieces of one context)
// is computed in the three steps of "What is the Mamba model?" (velog,
// Texnee), "chunkscan", with the segment as the chunk:
//  1. summary (intra-chunk step): every segment, independently, reduces to
//     its final state from a zero start, h_zero, and its dt sum, dtsum;
//  2. carry (inter-chunk step): the state entering segment r follows from the
//     summaries of segments 0..r-1 by h <- exp(A dtsum_j) h + h_zero_j, the
//     closed form of "Mamba/SSM basics" (molayo insights), "Technical
//     details" (h_t = A_t...A_1 h_0 + sum_j A_t...A_{j+1} B_j x_j) taken a
//     segment at a time;
//  3. combine: the ordinary prefill of segment r started from that state
//     (ssm_prefill with ssm_state_in), so outputs are rounded once.
//
// The summary is not a second sequential scan. With R_t = sum_{i>t} dt_i the
// dt mass after token t, the zero-start final state is
//     h_zero_n = sum_t exp(A_n R_t) inj_{t,n},
// inj = dt B u (Euler-B) or (exp(dt A)-1)/A B u (ZOH): a weighted sum over
// tokens with no dependence between them once R_t is known. The kernel
// computes it on 256-token blocks in parallel (R_t local to the block, so no
// large sums are differenced; each thread walks its block backwards, R being
// a running sum), and a second kernel folds the blocks in order with the
// block dt totals -- the same carry at block granularity.
//
// Cost per channel-token: 16 exp2 for the weights (32 for ZOH), one for dt and
// two for SiLU of the conv, all independent across tokens; no z, C or output
// traffic. x (io dtype), B and dt_raw are read once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssm.h"
#include "ssm_internal.h"
#include "sm100_ptx.cuh"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kN = 16;       // states
constexpr int kSegTok = 64;  // tokens per staged sub-block of the summary kernel
// Measured on B200 (8192-token segment, E = 7680): 1 sub-block at 8 CTAs per
// SM 317 us, 2 at 7 CTAs 303 us, 4 at 7 CTAs 300 us (fewer blocks to fold).
#ifndef SSM_SEG_SUB
#define SSM_SEG_SUB 4
#endif
#ifndef SSM_SEG_MINB
#define SSM_SEG_MINB 7
#endif
constexpr int kSegSub = SSM_SEG_SUB;  // sub-blocks per CTA: a block (one fold step) is kSegSub x 64 tokens
constexpr int kSegCh = 128;  // channels per CTA: 4 warps, lane = channel
constexpr int kSegThreads = 128;
// State pairs per token whose decay exp2 runs as an FMA-pipe polynomial
// (Euler-B): the SFU is the summary kernel's binding unit and the FMA pipe
// has room.
#ifndef SSM_SEG_POLY
#define SSM_SEG_POLY 1
#endif
constexpr int kSegPoly = SSM_SEG_POLY;

struct SegArgs {
  const void* x;
  const float* B;
  const float* dt_raw;
  const float* conv_w;
  const float* conv_b;
  const float* w_dt;
  const float* dt_bias;
  const float* A_log;
  const void* conv_cache_in;  // [b, 3, E] io dtype, or null (zero history)
  float* part;                // [b, nblk, N + 1, E]: per block, state contribution and dt total
  float* summary;             // [b, N + 1, E]
  int64_t batch, T, E, nblk;
  int64_t x_tok, x_seq, bc_tok, bc_seq, dt_seq;
  float dt_min, dt_max;
};

// 16-byte global -> shared copy through the async-copy path; src_bytes = 0
// writes zeros and reads nothing.
__device__ __forceinline__ void cp_async_16z(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_4z(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_all_done() {
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// One CTA per (block of kSegSub x 64 tokens, 128 channels, sequence). Each
// 64-token sub-block's raw x rows (with the 3 rows before it), B rows and
// dt_raw are staged in shared memory, last sub-block first; each thread walks
// its channel backwards through them, so R, the dt mass after the current
// token, is one running sum across the whole block.
template <typename T, bool ZOH>
__global__ void __launch_bounds__(kSegThreads, ZOH ? 4 : SSM_SEG_MINB) segment_block_kernel(const SegArgs a) {
  constexpr int kRowChunks = kSegCh * int(sizeof(T)) / 16;  // 16-byte pieces of one x row
  constexpr int kChPerChunk = 16 / int(sizeof(T));
  __shared__ __align__(16) float Bs[kSegTok][kN];
  __shared__ __align__(16) float dr[kSegTok];
  __shared__ __align__(16) T xs[kSegTok + 3][kSegCh];  // row r = token t_sub - 3 + r

  const int tid = threadIdx.x;
  const int64_t blk = blockIdx.x, s = blockIdx.z;
  const int64_t t_cta = blk * kSegTok * kSegSub;
  const int64_t e0 = int64_t(blockIdx.y) * kSegCh;
  const int c = tid;  // channel within the CTA
  const int64_t e = e0 + c;
  const int64_t ec = e < a.E ? e : a.E - 1;  // clamped for parameter loads; idle lanes store nothing

  const float4 cw = *reinterpret_cast<const float4*>(a.conv_w + ec * 4);
  const float cb = a.conv_b[ec], wdt = a.w_dt[ec], dtb = a.dt_bias[ec];
  float a2[kN];  // A_n log2(e)
  float An[ZOH ? kN : 1], rAn[ZOH ? kN : 1];  // A_n and 1 / A_n (ZOH only)
#pragma unroll
  for (int n = 0; n < kN; ++n) {
    const float A = -expf(a.A_log[ec * kN + n]);
    a2[n] = A * kLog2e;
    if constexpr (ZOH) {
      An[n] = A;
      rAn[n] = 1.0f / A;
    }
  }
  float acc[kN];
#pragma unroll
  for (int n = 0; n < kN; ++n) acc[n] = 0.0f;
  float R = 0.0f;

  const T* xseq = static_cast<const T*>(a.x) + s * a.x_seq;
  const T* hist = static_cast<const T*>(a.conv_cache_in);
  const float* Bseq = a.B + s * a.bc_seq;
#pragma unroll 1
  for (int sub = kSegSub - 1; sub >= 0; --sub) {
    const int64_t t_sub = t_cta + int64_t(sub) * kSegTok;
    if (t_sub >= a.T) continue;  // block-uniform
    const int nt = int(a.T - t_sub < kSegTok ? a.T - t_sub : kSegTok);
    __syncthreads();  // the previous sub-block's rows are no longer read
    // Stage. Rows past the segment's end and channels past E are zero-filled.
    for (int i = tid; i < (kSegTok + 3) * kRowChunks; i += kSegThreads) {
      const int r = i / kRowChunks, q = i % kRowChunks;
      const int64_t t = t_sub - 3 + r, ee = e0 + int64_t(q) * kChPerChunk;
      const void* src = a.x;
      uint32_t nb = 0;
      if (ee < a.E && t < a.T) {
        if (t >= 0) {
          src = xseq + t * a.x_tok + ee;
          nb = 16;
        } else if (hist) {
          src = hist + (s * 3 + (t + 3)) * a.E + ee;
          nb = 16;
        }
      }
      cp_async_16z(smem_addr(&xs[r][q * kChPerChunk]), src, nb);
    }
    for (int i = tid; i < kSegTok * (kN / 4); i += kSegThreads) {
      const int r = i >> 2, q = i & 3;
      const bool in = r < nt;
      cp_async_16z(smem_addr(&Bs[r][4 * q]), in ? Bseq + (t_sub + r) * a.bc_tok + 4 * q : a.B, in ? 16 : 0);
    }
    if (tid < kSegTok) {
      const bool in = tid < nt;
      cp_async_4z(smem_addr(&dr[tid]), in ? a.dt_raw + s * a.dt_seq + t_sub + tid : a.dt_raw, in ? 4 : 0);
    }
    cp_async_all_done();
    __syncthreads();

    // x window of token t: rows t .. t+3 (tokens t-3 .. t); slides down by one row.
    float x3 = IO<T>::to_f(xs[nt + 2][c]), x2 = IO<T>::to_f(xs[nt + 1][c]), x1 = IO<T>::to_f(xs[nt][c]);
#pragma unroll 2
    for (int t = nt - 1; t >= 0; --t) {
      const float x0 = IO<T>::to_f(xs[t][c]);
      const float conv = fmaf(cw.w, x3, fmaf(cw.z, x2, fmaf(cw.y, x1, fmaf(cw.x, x0, cb))));
      x3 = x2;
      x2 = x1;
      x1 = x0;
      const float u = silu(conv);
      const float dt = dt_of(fmaf(dr[t], wdt, dtb), a.dt_min, a.dt_max);
      const float4* Bt = reinterpret_cast<const float4*>(&Bs[t][0]);
      if constexpr (ZOH) {
#pragma unroll
        for (int q = 0; q < kN / 4; ++q) {
          const float4 b4 = Bt[q];
          const float bq[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int n = 4 * q + i;
            const float xa = dt * An[n];
            const float inj = u * bq[i] * zoh_scale(xa, dt, ex2_approx(xa * kLog2e), rAn[n]);
            acc[n] = fmaf(ex2_approx(a2[n] * R), inj, acc[n]);
          }
        }
      } else {
        // Euler-B, packed in state pairs: acc += e^{A R} (dt u) B.
        const uint64_t R2 = pk2(R, R), v2 = pk2(dt * u, dt * u);
#pragma unroll
        for (int p = 0; p < kN / 2; ++p) {
          const float4 b4 = Bt[p / 2];
          const uint64_t b2 = (p & 1) ? pk2(b4.z, b4.w) : pk2(b4.x, b4.y);
          float y0, y1;
          upk2(fmul2(R2, pk2(a2[2 * p], a2[2 * p + 1])), y0, y1);
          // the last kSegPoly pairs take the FMA-pipe exp2, the others the SFU
          const uint64_t decay = p >= kN / 2 - kSegPoly ? ex2_poly2(y0, y1) : pk2(ex2_approx(y0), ex2_approx(y1));
          uint64_t ap = pk2(acc[2 * p], acc[2 * p + 1]);
          ap = ffma2(decay, fmul2(v2, b2), ap);
          upk2(ap, acc[2 * p], acc[2 * p + 1]);
        }
      }
      R += dt;
    }
  }

  if (e < a.E) {
    float* out = a.part + ((s * a.nblk + blk) * (kN + 1)) * a.E + e;
#pragma unroll
    for (int n = 0; n < kN; ++n) out[n * a.E] = acc[n];
    out[kN * a.E] = R;
  }
}

// Fold the blocks of a segment in token order: h <- exp(A_n tot_k) h + part_k.
// One thread per (sequence, row n of N + 1, channel); row N sums the totals.
__global__ void segment_fold_kernel(const SegArgs a) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int n = blockIdx.y;
  const int64_t s = blockIdx.z;
  if (e >= a.E) return;
  const float* p = a.part + (s * a.nblk * (kN + 1)) * a.E + e;
  const int64_t blk_stride = (kN + 1) * a.E;
  float h = 0.0f;
  if (n == kN) {
    for (int64_t k = 0; k < a.nblk; ++k) h += p[k * blk_stride + kN * a.E];
  } else {
    const float a2 = -expf(a.A_log[e * kN + n]) * kLog2e;
#pragma unroll 8
    for (int64_t k = 0; k < a.nblk; ++k)
      h = fmaf(ex2_approx(a2 * p[k * blk_stride + kN * a.E]), h, p[k * blk_stride + n * a.E]);
  }
  a.summary[(s * (kN + 1) + n) * a.E + e] = h;
}

struct CarryArgs {
  const float* summaries;  // [count, b, N + 1, E]
  const float* A_log;
  const float* h_init;     // [b, E, N] or null
  float* h_out;            // [b, E, N]
  int64_t count, batch, E;
};

// The state entering the segment after `count` summarised ones, one thread
// per (sequence, channel, state): h <- exp(A_n dtsum_j) h + h_zero_j, j in order.
__global__ void segment_carry_kernel(const CarryArgs a) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= a.batch * a.E * kN) return;
  const int n = int(i % kN);
  const int64_t e = (i / kN) % a.E, s = i / (kN * a.E);
  const float a2 = -expf(a.A_log[e * kN + n]) * kLog2e;
  float h = a.h_init ? a.h_init[i] : 0.0f;
  const int64_t seg_stride = a.batch * (kN + 1) * a.E;
  const float* p = a.summaries + s * (kN + 1) * a.E + e;
#pragma unroll 4
  for (int64_t j = 0; j < a.count; ++j) h = fmaf(ex2_approx(a2 * p[j * seg_stride + kN * a.E]), h, p[j * seg_stride + n * a.E]);
  a.h_out[i] = h;
}

int64_t seg_blocks(int64_t T) { return (T + kSegTok * kSegSub - 1) / (kSegTok * kSegSub); }

}  // namespace
}  // namespace ssm

extern "C" {

size_t ssm_segment_summary_workspace_bytes(const ssm_dims* dims) {
  ssm::Strides s;
  if (ssm::check_dims(dims, true, &s) != SSM_OK) return 0;
  return size_t(dims->batch) * size_t(ssm::seg_blocks(dims->seqlen)) * (ssm::kN + 1) * size_t(dims->d_inner) *
         sizeof(float);
}

ssm_status ssm_segment_summary(const ssm_dims* dims, const ssm_weights* w, const void* x, const float* B,
                               const float* dt_raw, const void* conv_cache_in, float* summary, void* workspace,
                               size_t workspace_bytes, void* stream) {
  using ssm::fail;
  ssm::Strides s;
  ssm_status st = ssm::check_dims(dims, true, &s);
  if (st != SSM_OK) return st;
  if ((st = ssm::check_weights(w)) != SSM_OK) return st;
  if (!summary || !ssm::aligned(summary, 16)) return fail(SSM_ERR_INVALID_ARG, "summary is NULL or not 16-byte aligned");
  const int64_t T = dims->seqlen, E = dims->d_inner, b = dims->batch;
  if (T > 0) {
    if (!x || !ssm::aligned(x, 16)) return fail(SSM_ERR_INVALID_ARG, "x is NULL or not 16-byte aligned");
    if (!B || !ssm::aligned(B, 16)) return fail(SSM_ERR_INVALID_ARG, "B is NULL or not 16-byte aligned");
    if (!dt_raw || !ssm::aligned(dt_raw, 4)) return fail(SSM_ERR_INVALID_ARG, "dt_raw is NULL or not 4-byte aligned");
  }
  if (conv_cache_in && !ssm::aligned(conv_cache_in, 16))
    return fail(SSM_ERR_INVALID_ARG, "conv_cache_in not 16-byte aligned");
  const size_t need = ssm_segment_summary_workspace_bytes(dims);
  if (need && (!workspace || workspace_bytes < need || !ssm::aligned(workspace, 16)))
    return fail(SSM_ERR_INVALID_ARG, "workspace: need %zu bytes, 16-byte aligned", need);
  const int64_t nblk = ssm::seg_blocks(T);
  if (nblk > 0x7fffffffLL || b > 65535)
    return fail(SSM_ERR_INVALID_ARG, "segment of %lld tokens x %lld sequences is too large for one launch",
                (long long)T, (long long)b);

  ssm::SegArgs a{};
  a.x = x;
  a.B = B;
  a.dt_raw = dt_raw;
  a.conv_w = w->conv_w;
  a.conv_b = w->conv_b;
  a.w_dt = w->w_dt;
  a.dt_bias = w->dt_bias;
  a.A_log = w->A_log;
  a.conv_cache_in = conv_cache_in;
  a.part = static_cast<float*>(workspace);
  a.summary = summary;
  a.batch = b;
  a.T = T;
  a.E = E;
  a.nblk = nblk;
  a.x_tok = s.x_tok;
  a.x_seq = s.x_seq;
  a.bc_tok = s.bc_tok;
  a.bc_seq = s.bc_seq;
  a.dt_seq = s.dt_seq;
  a.dt_min = dims->dt_min;
  a.dt_max = dims->dt_max;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const bool bf16 = dims->io_dtype == SSM_BF16, zoh = dims->discretization == SSM_DISC_ZOH;
  if (nblk > 0) {
    const dim3 grid(unsigned(nblk), unsigned((E + ssm::kSegCh - 1) / ssm::kSegCh), unsigned(b));
    const dim3 block(ssm::kSegThreads);
    if (bf16 && zoh)
      ssm::segment_block_kernel<__nv_bfloat16, true><<<grid, block, 0, cs>>>(a);
    else if (bf16)
      ssm::segment_block_kernel<__nv_bfloat16, false><<<grid, block, 0, cs>>>(a);
    else if (zoh)
      ssm::segment_block_kernel<float, true><<<grid, block, 0, cs>>>(a);
    else
      ssm::segment_block_kernel<float, false><<<grid, block, 0, cs>>>(a);
  }
  ssm::segment_fold_kernel<<<dim3(unsigned((E + 127) / 128), ssm::kN + 1, unsigned(b)), 128, 0, cs>>>(a);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "segment summary launch: %s", cudaGetErrorString(err));
  return fail(SSM_OK, "");
}

ssm_status ssm_segment_carry(const ssm_dims* dims, const ssm_weights* w, const float* summaries, int64_t count,
                             const float* ssm_state_in, float* ssm_state_out, void* stream) {
  using ssm::fail;
  ssm::Strides s;
  ssm_status st = ssm::check_dims(dims, true, &s);
  if (st != SSM_OK) return st;
  if ((st = ssm::check_weights(w)) != SSM_OK) return st;
  if (count < 0) return fail(SSM_ERR_INVALID_ARG, "count=%lld must be >= 0", (long long)count);
  if (count > 0 && (!summaries || !ssm::aligned(summaries, 4)))
    return fail(SSM_ERR_INVALID_ARG, "summaries is NULL or not 4-byte aligned");
  if (!ssm_state_out || !ssm::aligned(ssm_state_out, 4))
    return fail(SSM_ERR_INVALID_ARG, "ssm_state_out is NULL or not 4-byte aligned");
  if (ssm_state_in && !ssm::aligned(ssm_state_in, 4)) return fail(SSM_ERR_INVALID_ARG, "ssm_state_in not 4-byte aligned");
  ssm::CarryArgs a{summaries, w->A_log, ssm_state_in, ssm_state_out, count, dims->batch, dims->d_inner};
  const int64_t n = dims->batch * dims->d_inner * ssm::kN;
  const int64_t blocks = (n + 255) / 256;
  if (blocks > 0x7fffffffLL) return fail(SSM_ERR_INVALID_ARG, "state too large for one launch");
  ssm::segment_carry_kernel<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "segment carry launch: %s", cudaGetErrorString(err));
  return fail(SSM_OK, "");
}

}  // extern "C"
