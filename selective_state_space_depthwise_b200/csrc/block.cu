// block.cu -- the AxonSSMBlock forward around the prefill core ("Axon-SSM:
// selective state space model", "Algorithm" diagram): in_proj and out_proj as
// this library's tcgen05 GEMM (gemm.cu), x_proj as one fused tcgen05 kernel,
// the core as prefill.cu's kernel reading x and z in place from the in_proj
// output, and out_proj reading the core's gated output y as its A operand.
//
// x_proj kernel. A CTA owns 128 tokens of one sequence (the MMA's M) and a
// contiguous range of the E channels, walked in chunks of 64 (K). Per chunk:
//  1. TMA brings the x tile (131 rows: 3 halo rows for the conv) and the W_x
//     tile (48 rows = the 33 outputs padded to a multiple of 16, zero-filled by
//     TMA past row 33; 128-byte swizzled, the MMA's B operand) into a 3-slot
//     ring, issued two chunks ahead;
//  2. the eight warps compute u = SiLU(conv1d(x)) for their 16 tokens (lane =
//     channel pair, a 3-row sliding window in registers, the conv weights of
//     the next chunk loaded one chunk ahead) and write it as bf16 straight
//     into the MMA's A tile (2 slots), in the 128-byte swizzled K-major layout;
//  3. one thread issues four tcgen05 MMAs (K = 16 each, bf16 x bf16 -> fp32)
//     into a 48-column TMEM accumulator and commits them to the A slot's
//     mbarrier; slots are refilled only after the MMAs that read them completed.
// Split K: when 128-token tiles alone would not fill the GPU, a thread-block
// cluster of S CTAs (S <= 8, along grid z) shares one tile, each CTA summing a
// contiguous channel range in its own TMEM. The partial 128 x 48 tiles go to
// shared memory and CTA r of the cluster adds, in the fixed order 0..S-1 over
// distributed shared memory, the rows of tokens [r 128/S, (r+1) 128/S) and
// writes B, C ([b, L, 32] fp32) and dt_raw ([b, L] fp32). u never reaches
// memory. Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "ssm.h"
#include "tma_map.cuh"
#include "ssm_internal.h"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kXpTok = 128;      // tokens per CTA (MMA M)
constexpr int kXpK = 64;         // channels per chunk: 128 bytes of bf16, one swizzle row
constexpr int kXpN = 48;         // MMA N: the 2N + 1 = 33 outputs padded to a multiple of 16
constexpr int kXpOut = 33;
// Eight warps: warp w forms token rows 16w .. 16w + 15 of each A tile; in the
// epilogue warps w and w + 4 read TMEM lanes (tokens) 32 (w mod 4) ..,
// columns 0-31 and 32-47. Four warps of 32 rows left one warp per SM
// sub-partition at the layer shape (one CTA per SM): x_proj alone took 49.0
// against 40.9 us at 2048 tokens, 185 against 153 us at 16384.
constexpr int kXpThreads = 256;
constexpr int kXpRows = kXpTok / (kXpThreads / 32);  // A-tile rows per warp
constexpr uint32_t kXpTmemCols = 64;
constexpr int kXpStages = 3;     // x / W_x TMA ring
constexpr int kXpMaxSplit = 8;   // portable cluster size

struct XpSmem {
  static constexpr int kABytes = kXpTok * 128;          // [128 rows][128 B], swizzled
  static constexpr int kWBytes = kXpN * 128;            // [48 rows][128 B], swizzled by TMA
  static constexpr int kXBytes = (kXpTok + 3) * 128;    // [131 rows][64 channels] bf16
  static constexpr int kA = 0;                          // 2 slots, 1024-aligned
  static constexpr int kW = 2 * kABytes;                // kXpStages slots, 1024-aligned
  static constexpr int kX = kW + kXpStages * kWBytes;   // kXpStages slots
  static constexpr int kP = kX;                         // partial sums [128][48] fp32, after the loop
  static constexpr int kBar = kX + kXpStages * kXBytes; // full[kXpStages], done[2]
  static constexpr int kTmemSlot = kBar + (kXpStages + 2) * 8;
  static constexpr int kAbort = kTmemSlot + 4;          // set when a bounded wait gave up
  static constexpr int kLast = kTmemSlot + 8;           // the last chunk whose MMAs were committed
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr uint32_t kTx = static_cast<uint32_t>(kWBytes + kXBytes);
  static_assert(kW % 1024 == 0 && kWBytes % 1024 == 0 && kABytes % 1024 == 0, "swizzled tiles need 1 KB");
  static_assert(kXpTok * kXpN * 4 <= kXpStages * kXBytes, "the partial tile reuses the x ring");
};

// Instruction descriptor: bf16 A and B (K-major), fp32 D, M = 128, N = 48.
constexpr uint32_t kXpIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kXpN >> 3) << 17) |
                              (static_cast<uint32_t>(kXpTok >> 4) << 24);

struct XprojArgs {
  const float* conv_w;                  // [E][4]
  const float* conv_b;                  // [E]
  const __nv_bfloat16* conv_cache_in;   // [b][3][E] or null (zeros)
  float* bc;                            // [b][L][32]: B then C
  float* dt_raw;                        // [b][L]
  int64_t L, E;
  int* err;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
  __nv_bfloat162 v;
  *reinterpret_cast<uint32_t*>(&v) = w;
  return __bfloat1622float2(v);
}

struct ConvPair {  // conv weights and biases of one lane's channel pair in one chunk
  float4 w0, w1;
  float b0, b1;
};

__device__ __forceinline__ ConvPair load_conv_pair(const XprojArgs& a, int64_t e0) {
  ConvPair p;
  const bool v0 = e0 < a.E, v1 = e0 + 1 < a.E;
  p.w0 = v0 ? reinterpret_cast<const float4*>(a.conv_w)[e0] : make_float4(0.f, 0.f, 0.f, 0.f);
  p.w1 = v1 ? reinterpret_cast<const float4*>(a.conv_w)[e0 + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
  p.b0 = v0 ? a.conv_b[e0] : 0.0f;
  p.b1 = v1 ? a.conv_b[e0 + 1] : 0.0f;
  return p;
}

__global__ void __launch_bounds__(kXpThreads) xproj_kernel(const __grid_constant__ CUtensorMap map_x,
                                                          const __grid_constant__ CUtensorMap map_w,
                                                          const XprojArgs a) {
  using S = XpSmem;
  // Launched overlapped with in_proj (programmatic dependent launch): nothing
  // in global memory is touched before it has finished.
  griddep_wait();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0), lane = tid & 31;
  const int seq = blockIdx.y;
  const int t0 = blockIdx.x * kXpTok;
  const int split = gridDim.z, rank = blockIdx.z;  // the cluster spans grid z
  const int nk = static_cast<int>((a.E + kXpK - 1) / kXpK);
  const int c_begin = rank * nk / split, nloc = (rank + 1) * nk / split - c_begin;
  auto full = [&](int j) { return sb + S::kBar + 8 * (j % kXpStages); };
  auto done = [&](int j) { return sb + S::kBar + 8 * kXpStages + 8 * (j & 1); };
  auto issue = [&](int j) {  // thread 0: the tiles of local chunk j
    const int slot = j % kXpStages, c = c_begin + j;
    mbar_arrive_expect_tx(full(j), S::kTx);
    tma_load_3d(sb + S::kX + slot * S::kXBytes, &map_x, c * kXpK, t0 - 3, seq, full(j));
    tma_load_3d(sb + S::kW + slot * S::kWBytes, &map_w, c * kXpK, 0, 0, full(j));
  };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kAbort);
  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < kXpStages + 2; ++i) mbar_init(sb + S::kBar + 8 * i, 1);
    mbar_fence_init();
    prefetch_tensormap(&map_x);
    prefetch_tensormap(&map_w);
    for (int j = 0; j < kXpStages && j < nloc; ++j) issue(j);
  }
  if (warp == 0) {
    tmem_alloc(sb + S::kTmemSlot, kXpTmemCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + S::kTmemSlot);

  int issued = -1;  // the last local chunk whose MMAs thread 0 committed
  ConvPair cw = load_conv_pair(a, static_cast<int64_t>(c_begin) * kXpK + 2 * lane);
  for (int j = 0; j < nloc; ++j) {
    const int c = c_begin + j;
    // the next chunk's conv weights, one chunk ahead
    const ConvPair cw_next =
        j + 1 < nloc ? load_conv_pair(a, static_cast<int64_t>(c + 1) * kXpK + 2 * lane) : cw;
    if (!mbar_wait_bounded(full(j), static_cast<uint32_t>((j / kXpStages) & 1), a.err, 3)) *abort_flag = 1;
    if (j >= 2 && !mbar_wait_bounded(done(j), static_cast<uint32_t>(((j - 2) >> 1) & 1), a.err, 4))
      *abort_flag = 1;  // the MMAs of chunk j - 2 have finished reading this A slot
    const int64_t e0 = static_cast<int64_t>(c) * kXpK + 2 * lane;
    const bool v0 = e0 < a.E, v1 = e0 + 1 < a.E;
    const uint32_t* xt = reinterpret_cast<const uint32_t*>(smem + S::kX + (j % kXpStages) * S::kXBytes);
    unsigned char* At = smem + S::kA + (j & 1) * S::kABytes;
    // window = tile rows r, r+1, r+2 (tokens t0 + r - 3 ..); rows before token 0 are
    // zero-filled by TMA and replaced by the incoming conv cache when there is one
    const int r0 = kXpRows * warp;
    float2 x0 = unpack_bf16x2(xt[(r0 + 0) * 32 + lane]);
    float2 x1 = unpack_bf16x2(xt[(r0 + 1) * 32 + lane]);
    float2 x2 = unpack_bf16x2(xt[(r0 + 2) * 32 + lane]);
    if (t0 == 0 && warp == 0 && a.conv_cache_in) {
      const __nv_bfloat16* h = a.conv_cache_in + static_cast<int64_t>(seq) * 3 * a.E;
      float2 hv[3];
#pragma unroll
      for (int k = 0; k < 3; ++k)
        hv[k] = make_float2(v0 ? __bfloat162float(h[k * a.E + e0]) : 0.0f,
                            v1 ? __bfloat162float(h[k * a.E + e0 + 1]) : 0.0f);
      x0 = hv[0], x1 = hv[1], x2 = hv[2];
    }
    // Fully unrolled, so the compiler can hide the window loads and the SFU
    // latency across the whole run (four warps with 8 of their 32 rows
    // unrolled: 53 us at 2048 tokens).
#pragma unroll
    for (int i = 0; i < kXpRows; ++i) {
      const int r = r0 + i;
      const float2 x3 = unpack_bf16x2(xt[(r + 3) * 32 + lane]);
      const float c0 =
          fmaf(cw.w0.w, x3.x, fmaf(cw.w0.z, x2.x, fmaf(cw.w0.y, x1.x, fmaf(cw.w0.x, x0.x, cw.b0))));
      const float c1 =
          fmaf(cw.w1.w, x3.y, fmaf(cw.w1.z, x2.y, fmaf(cw.w1.y, x1.y, fmaf(cw.w1.x, x0.y, cw.b1))));
      const uint32_t u = pack_bf16x2(v0 ? silu(c0) : 0.0f, v1 ? silu(c1) : 0.0f);
      // element (row r, k = 2 lane) of the 128-byte swizzled K-major tile
      *reinterpret_cast<uint32_t*>(At + r * 128 + ((((lane >> 2) ^ (r & 7))) << 4) + ((lane & 3) << 2)) = u;
      x0 = x1, x1 = x2, x2 = x3;
    }
    fence_proxy_async_smem();  // the tile's generic-proxy writes become visible to the tensor core
    __syncthreads();
    if (*abort_flag) break;  // a wait gave up: stop queueing work (every thread sees the flag here)
    if (tid == 0) {
      tcgen05_fence_after();
      const uint32_t a_base = sb + S::kA + (j & 1) * S::kABytes;
      const uint32_t w_base = sb + S::kW + (j % kXpStages) * S::kWBytes;
#pragma unroll
      for (int kk = 0; kk < kXpK / 16; ++kk)
        umma_f16_ss(tmem, umma_desc_k_sw128(a_base + 32 * kk), umma_desc_k_sw128(w_base + 32 * kk), kXpIdesc,
                    j > 0 || kk > 0);
      umma_commit(done(j));
      issued = j;
      // chunk j + 2 refills the ring slot chunk j - 1 used: wait for those MMAs first
      if (j >= 1 && j + 2 < nloc) {
        if (mbar_wait_bounded(done(j - 1), static_cast<uint32_t>(((j - 1) >> 1) & 1), a.err, 5))
          issue(j + 2);
        else
          *abort_flag = 1;
      }
    }
    cw = cw_next;
  }
  // Every thread waits (bounded) for the last MMAs thread 0 committed.
  volatile int* last_slot = reinterpret_cast<volatile int*>(smem + S::kLast);
  if (tid == 0) *last_slot = issued;
  __syncthreads();
  const int last = *last_slot;
  if (last >= 0) mbar_wait_bounded(done(last), static_cast<uint32_t>((last >> 1) & 1), a.err, 6);
  tcgen05_fence_after();

  // This CTA's partial [128 tokens][48] tile into shared memory (the x ring is free).
  float* P = reinterpret_cast<float*>(smem + S::kP);
  {
    const int q = warp & 3, row = 32 * q + lane;
    // 16-column groups of the accumulator: warps 0-3 read groups 0 and 1, warps 4-7 group 2
    const int jj0 = warp < 4 ? 0 : 2, jj1 = warp < 4 ? 2 : kXpN / 16;
    for (int jj = jj0; jj < jj1; ++jj) {
      uint32_t r[16];
      if (last >= 0) {
        tmem_ld_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) + 16 * jj, r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) r[q] = 0u;  // no channel range here: contributes zeros
      }
      float4* dst = reinterpret_cast<float4*>(P + row * kXpN + 16 * jj);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                             __uint_as_float(r[4 * q + 3]));
    }
  }
  cluster_sync();
  // CTA `rank` sums the cluster's partials, in rank order, for its share of the tokens.
  const int per = kXpTok / split;
  for (int idx = tid; idx < per * kXpOut; idx += kXpThreads) {
    const int tl = rank * per + idx / kXpOut, o = idx % kXpOut;
    const uint32_t addr = sb + S::kP + static_cast<uint32_t>((tl * kXpN + o) * 4);
    float sum = 0.0f;
    for (int q = 0; q < split; ++q) sum += ld_shared_cluster_f32(addr, static_cast<uint32_t>(q));
    const int64_t t = t0 + tl;
    if (t < a.L) {
      const int64_t row = static_cast<int64_t>(seq) * a.L + t;
      if (o < 32)
        a.bc[row * 32 + o] = sum;
      else
        a.dt_raw[row] = sum;
    }
  }
  cluster_sync();  // the partials stay alive until every CTA of the cluster has read them
  tcgen05_fence_before();
  // The next kernel may now be launched (it waits for this one to finish
  // before it reads anything); signalling this late, not at the start, keeps
  // its waiting CTAs off the SMs while this kernel still runs.
  griddep_launch_dependents();
  __syncthreads();
  if (warp == 0) {
    tcgen05_fence_after();
    tmem_dealloc(tmem, kXpTmemCols);
  }
}

bool bf16_map3(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
               uint64_t s2_bytes, uint32_t b0, uint32_t b1, CUtensorMapSwizzle swz) {
  const uint64_t dims[3] = {d0, d1, d2}, strides[2] = {s1_bytes, s2_bytes};
  const uint32_t box[3] = {b0, b1, 1};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, swz);
}

// x = the first E columns of xz [b][L][2E] (bf16); W_x [33][E] (bf16).
cudaError_t launch_xproj(const XprojArgs& a, const void* xz, const void* w_x, int64_t batch, int num_sms,
                         cudaStream_t st, bool pdl) {
  CUtensorMap mx, mw;
  const uint64_t E = static_cast<uint64_t>(a.E), L = static_cast<uint64_t>(a.L);
  if (!bf16_map3(&mx, xz, E, L, static_cast<uint64_t>(batch), 2 * E * 2, L * 2 * E * 2, kXpK, kXpTok + 3,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !bf16_map3(&mw, w_x, E, kXpOut, 1, E * 2, kXpOut * E * 2, kXpK, kXpN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int smem = XpSmem::kTotal + 1024;
  cudaError_t err = cudaFuncSetAttribute(xproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int64_t gx = (a.L + kXpTok - 1) / kXpTok;
  if (gx > 0x7fffffff || batch > 65535) return cudaErrorInvalidConfiguration;
  // Split the channels over a cluster until the grid covers two CTAs per SM.
  const int64_t tiles = gx * batch, nk = (a.E + kXpK - 1) / kXpK;
  int split = 1;
  while (split < kXpMaxSplit && 2 * split <= nk && tiles * split < 2 * static_cast<int64_t>(num_sms)) split *= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(batch), static_cast<unsigned>(split));
  cfg.blockDim = dim3(kXpThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned>(split);
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  err = cudaLaunchKernelEx(&cfg, xproj_kernel, mx, mw, a);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct BlockLayout {
  size_t xz, bc, dt, y, gemm, gemm_bytes, bytes;
};

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();  // no device: the default SM count
  return sms > 0 ? sms : 148;
}

BlockLayout block_layout(const ssm_block_dims* d) {
  const size_t M = static_cast<size_t>(d->batch * d->seqlen), E = static_cast<size_t>(d->d_inner);
  BlockLayout l{};
  size_t off = 0;
  l.xz = off, off = align_up(off + M * 2 * E * 2);
  l.bc = off, off = align_up(off + M * 32 * 4);
  l.dt = off, off = align_up(off + M * 4);
  l.y = off, off = align_up(off + M * E * 2);
  // cut-tile scratch of whichever projection needs more (in_proj and out_proj run one after the other)
  const int sms = sm_count();
  const int64_t Mi = static_cast<int64_t>(M), Ei = static_cast<int64_t>(E), Dm = d->d_model;
  const size_t g_in = gemm_workspace_bytes(Mi, 2 * Ei, Dm, sms), g_out = gemm_workspace_bytes(Mi, Dm, Ei, sms);
  l.gemm_bytes = g_in > g_out ? g_in : g_out;
  l.gemm = off, off = align_up(off + l.gemm_bytes);
  l.bytes = off;
  return l;
}

ssm_status check_block_dims(const ssm_block_dims* d) {
  if (!d) return fail(SSM_ERR_INVALID_ARG, "dims is NULL");
  if (d->d_state != 16) return fail(SSM_ERR_UNSUPPORTED, "d_state=%d: only 16 is built", d->d_state);
  if (d->d_conv != 4) return fail(SSM_ERR_UNSUPPORTED, "d_conv=%d: only 4 is built", d->d_conv);
  if (d->io_dtype != SSM_BF16) return fail(SSM_ERR_UNSUPPORTED, "the block forward is built for bf16 only");
  if (d->batch <= 0 || d->batch > 65535)
    return fail(SSM_ERR_INVALID_ARG, "batch=%lld must be in 1..65535", (long long)d->batch);
  if (d->seqlen < 0) return fail(SSM_ERR_INVALID_ARG, "seqlen=%lld must be >= 0", (long long)d->seqlen);
  if (d->d_model <= 0 || d->d_model % 8 != 0)
    return fail(SSM_ERR_INVALID_ARG, "d_model=%lld must be a positive multiple of 8", (long long)d->d_model);
  if (d->d_inner <= 0 || d->d_inner % 8 != 0)
    return fail(SSM_ERR_INVALID_ARG, "d_inner=%lld must be a positive multiple of 8", (long long)d->d_inner);
  if (!(d->dt_min > 0.0f) || !(d->dt_max >= d->dt_min))
    return fail(SSM_ERR_INVALID_ARG, "need 0 < dt_min <= dt_max (got %g, %g)", d->dt_min, d->dt_max);
  if (d->discretization != SSM_DISC_EULER_B && d->discretization != SSM_DISC_ZOH)
    return fail(SSM_ERR_INVALID_ARG, "discretization=%d unknown", d->discretization);
  return SSM_OK;
}

ssm_dims core_dims(const ssm_block_dims* d) {
  ssm_dims c{};
  c.batch = d->batch, c.seqlen = d->seqlen, c.d_inner = d->d_inner, c.d_state = 16, c.d_conv = 4;
  c.dt_min = d->dt_min, c.dt_max = d->dt_max, c.io_dtype = SSM_BF16, c.discretization = d->discretization;
  return c;
}

}  // namespace
}  // namespace ssm

extern "C" {

size_t ssm_block_workspace_bytes(const ssm_block_dims* dims) {
  if (ssm::check_block_dims(dims) != SSM_OK) return 0;
  return ssm::block_layout(dims).bytes;
}

ssm_status ssm_block_forward(const ssm_block_dims* dims, const ssm_weights* w, const ssm_block_weights* proj,
                             const void* hidden, const void* conv_cache_in, const float* ssm_state_in, void* out,
                             void* conv_cache_out, float* ssm_state_out, void* workspace, size_t workspace_bytes,
                             void* stream) {
  using ssm::fail;
  ssm_status st = ssm::check_block_dims(dims);
  if (st != SSM_OK) return st;
  if ((st = ssm::check_weights(w)) != SSM_OK) return st;
  if ((st = ssm::check_prefill_caches(conv_cache_in, ssm_state_in, conv_cache_out, ssm_state_out)) != SSM_OK)
    return st;
  ssm_dims cd = ssm::core_dims(dims);
  if (dims->seqlen == 0)  // caches only
    return ssm_prefill(&cd, w, nullptr, nullptr, nullptr, nullptr, nullptr, conv_cache_in, ssm_state_in, nullptr,
                       conv_cache_out, ssm_state_out, nullptr, 0, stream);
  if (!proj) return fail(SSM_ERR_INVALID_ARG, "proj is NULL");
  const void* pw[3] = {proj->w_in, proj->w_x, proj->w_out};
  const char* pn[3] = {"w_in", "w_x", "w_out"};
  for (int i = 0; i < 3; ++i)
    if (!pw[i] || !ssm::aligned(pw[i], 16)) return fail(SSM_ERR_INVALID_ARG, "proj.%s is NULL or misaligned", pn[i]);
  if (!hidden || !ssm::aligned(hidden, 16)) return fail(SSM_ERR_INVALID_ARG, "hidden is NULL or misaligned");
  if (!out || !ssm::aligned(out, 16)) return fail(SSM_ERR_INVALID_ARG, "out is NULL or misaligned");
  if (out == hidden) return fail(SSM_ERR_INVALID_ARG, "out must not alias hidden");
  const ssm::BlockLayout lay = ssm::block_layout(dims);
  if (!workspace || !ssm::aligned(workspace, ssm::kAlign))
    return fail(SSM_ERR_INVALID_ARG, "workspace is NULL or not %zu-byte aligned", ssm::kAlign);
  if (workspace_bytes < lay.bytes)
    return fail(SSM_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", workspace_bytes, lay.bytes);

  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const int64_t b = dims->batch, L = dims->seqlen, E = dims->d_inner, Dm = dims->d_model, M = b * L;
  void* xz = ws + lay.xz;
  float* bc = reinterpret_cast<float*>(ws + lay.bc);
  float* dt = reinterpret_cast<float*>(ws + lay.dt);
  void* y = ws + lay.y;

  int* err_word = ssm::device_error_ptr();
  if (!err_word) return fail(SSM_ERR_CUDA, "device error word: %s", cudaGetErrorString(cudaGetLastError()));
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // The four kernels run back to back; each after the first is launched
  // overlapped with the one before it (programmatic dependent launch), so its
  // launch and setup hide under that kernel's tail. The GEMMs' cut-tile
  // counters lead their shared scratch: zeroed once here (a memset between
  // two kernels would break the overlap), they are zero again after each GEMM.
  const size_t cnt_in = ssm::gemm_counter_bytes(M, 2 * E, Dm, sms), cnt_out = ssm::gemm_counter_bytes(M, Dm, E, sms);
  const size_t cnt = cnt_in > cnt_out ? cnt_in : cnt_out;
  cudaError_t err = cnt ? cudaMemsetAsync(ws + lay.gemm, 0, cnt, cs) : cudaSuccess;
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "projection scratch: %s", cudaGetErrorString(err));
  // in_proj: xz[M][2E] = hidden[M][D] . W_in[2E][D]^T
  err = ssm::gemm_bf16_tn(hidden, proj->w_in, xz, M, 2 * E, Dm, ws + lay.gemm, lay.gemm_bytes, sms, err_word, cs,
                          false, true);
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "in_proj launch: %s", cudaGetErrorString(err));
  // x_proj (fused with conv + SiLU): B, C, dt_raw
  ssm::XprojArgs xa{};
  xa.conv_w = w->conv_w;
  xa.conv_b = w->conv_b;
  xa.conv_cache_in = static_cast<const __nv_bfloat16*>(conv_cache_in);
  xa.bc = bc;
  xa.dt_raw = dt;
  xa.L = L;
  xa.E = E;
  xa.err = err_word;
  err = ssm::launch_xproj(xa, xz, proj->w_x, b, sms, cs, true);
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "x_proj launch: %s", cudaGetErrorString(err));
  // the core, on x and z in place in xz
  cd.x_tok_stride = cd.z_tok_stride = 2 * E;
  cd.x_seq_stride = cd.z_seq_stride = L * 2 * E;
  cd.y_tok_stride = E;
  cd.y_seq_stride = L * E;
  cd.bc_tok_stride = 32;
  cd.bc_seq_stride = L * 32;
  cd.dt_seq_stride = L;
  const __nv_bfloat16* xzb = static_cast<const __nv_bfloat16*>(xz);
  if ((st = ssm::prefill_entry(&cd, w, xzb, xzb + E, bc, bc + 16, dt, conv_cache_in, ssm_state_in, y,
                               conv_cache_out, ssm_state_out, nullptr, true, stream)) != SSM_OK)
    return st;
  // out_proj: out[M][D] = y[M][E] . W_out[D][E]^T
  err = ssm::gemm_bf16_tn(y, proj->w_out, out, M, Dm, E, ws + lay.gemm, lay.gemm_bytes, sms, err_word, cs, true,
                          true);
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "out_proj launch: %s", cudaGetErrorString(err));
  return ssm::fail(SSM_OK, "");
}

}  // extern "C"
