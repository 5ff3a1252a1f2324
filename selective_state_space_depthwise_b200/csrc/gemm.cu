// gemm.cu -- the block's dense projections on the tensor cores (sm_100a):
// in_proj (D -> 2E) and out_proj (E -> D) of "Axon-SSM: selective state space
// model", "Algorithm" diagram, as C[M][N] = A[M][K] . B[N][K]^T with A and B
// bf16 row-major (both K-major), fp32 accumulation and a bf16 C.
//
// One persistent CTA per SM walks output tiles of 128 x BN (BN = 256 or 160)
// in a static round-robin order over a grouped raster: tiles run in groups of
// up to 16 row blocks x every column block, row block fastest inside a group,
// so the CTAs running at the same time share both their A row blocks and their
// B column blocks in L2 (with a plain row-fastest order a wave of 148 tiles
// spans 148 row blocks of one column block, and at M = 65536 every A block
// would be read from HBM once per column block). Six warps with fixed roles:
//   warp 0     TMA producer: the A tile [128][64] and the B tile [BN][64] of
//              each 64-wide K chunk, 128-byte swizzled, into a STAGES-deep ring
//              (full / empty mbarriers per slot);
//   warp 1     MMA issuer: one thread issues four tcgen05.mma (M = 128, N = BN,
//              K = 16, kind::f16) per chunk into a TMEM accumulator, commits
//              each chunk to its slot's empty barrier and each finished tile to
//              the accumulator's full barrier; the two accumulators (2 x BN of
//              the 512 TMEM columns) alternate, so the next tile's MMAs run
//              while the epilogue drains the previous one;
//   warps 2-5  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its
//              quarter of the tile's rows) 32 columns at a time, rounds to
//              bf16, writes a [32][32] staging tile (two per warp, alternating)
//              and stores it with a TMA tile store, then frees the accumulator.
// Tails: TMA loads past M, N or K read zeros; stores are clipped at M and N.
// Every mbarrier wait is bounded; a wait that gives up sets the device error
// word and a CTA abort flag, every role leaves its loop, the producer waits
// (bounded) for its loads still in flight, the MMA thread for its last
// commit, the epilogue for its stores, and TMEM is freed before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "ssm.h"
#include "ssm_internal.h"
#include "tma_map.cuh"

namespace ssm {
namespace {

constexpr int kGBM = 128;  // tile rows: the MMA's M, one TMEM lane per row
constexpr int kGBK = 64;   // K chunk: 128 bytes of bf16, one swizzle row
constexpr int kGThreads = 192;
constexpr uint64_t kDrainNs = 200000000ull;  // 0.2 s: drain waits after an abort
// Build-time override of the output tile width (0 = chosen per shape), for
// side-by-side variant builds in measurements.
#ifndef SSM_GEMM_FORCE_BN
#define SSM_GEMM_FORCE_BN 0
#endif

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int kABytes = kGBM * 128;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kOut = STAGES * kStage;  // epilogue staging: 4 warps x 2 tiles of [32][32] bf16
  static constexpr int kOutBytes = 32 * 64;
  static constexpr int kBar = kOut + 8 * kOutBytes;  // full[S], empty[S], tfull[2], tempty[2]
  static constexpr int kTmemSlot = kBar + (2 * STAGES + 4) * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kIssued = kTmemSlot + 8;  // int64: K chunks the producer issued
  static constexpr int kTotal = kIssued + 8;
  // TMEM columns: two accumulators of BN, allocated as a power of two.
  static constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256u : 512u;
  static_assert(kStage % 1024 == 0, "swizzled operand tiles need 1 KB alignment");
};

struct GemmArgs {
  int tiles_m, tiles_n, k_chunks;
  int group_m;  // row blocks per raster group
  int* err;
};

// Tile index -> (row block, column block) of the grouped raster.
__device__ __forceinline__ void tile_coords(const GemmArgs& g, int tile, int& mb, int& nb) {
  const int per_group = g.group_m * g.tiles_n;
  const int grp = tile / per_group, r = tile - grp * per_group;
  const int m_base = grp * g.group_m;
  const int gm = min(g.group_m, g.tiles_m - m_base);  // the last group may be shorter
  mb = m_base + r % gm;
  nb = r / gm;
}

// bf16 x bf16 -> fp32, M = 128, N = BN, A and B K-major.
template <int BN>
__host__ __device__ constexpr uint32_t gemm_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
         (static_cast<uint32_t>(kGBM >> 4) << 24);
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGThreads, 1)
    gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        const __grid_constant__ CUtensorMap map_c, const GemmArgs g) {
  using S = GemmSmem<BN, STAGES>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0), lane = tid & 31;
  auto full = [&](int s) { return sb + S::kBar + 8 * s; };
  auto empty = [&](int s) { return sb + S::kBar + 8 * (STAGES + s); };
  auto tfull = [&](int b) { return sb + S::kBar + 8 * (2 * STAGES + b); };
  auto tempty = [&](int b) { return sb + S::kBar + 8 * (2 * STAGES + 2 + b); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kAbort);
  volatile int64_t* issued_slot = reinterpret_cast<volatile int64_t*>(smem + S::kIssued);
  const int ntiles = g.tiles_m * g.tiles_n;

  if (tid == 0) {
    *abort_flag = 0;
    *issued_slot = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull(b), 1);
      mbar_init(tempty(b), 4);  // one arrival per epilogue warp
    }
    mbar_fence_init();
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    prefetch_tensormap(&map_c);
  }
  if (warp == 1) {
    tmem_alloc(sb + S::kTmemSlot, S::kTmemCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + S::kTmemSlot);

  if (warp == 0) {
    // ---------------------------------------------------------- producer ---
    if (lane == 0) {
      int64_t it = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        int mb, nb;
        tile_coords(g, tile, mb, nb);
        const int m0 = mb * kGBM, n0 = nb * BN;
        for (int kc = 0; kc < g.k_chunks; ++kc, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const uint32_t round = static_cast<uint32_t>(it / STAGES);
          if (!mbar_wait_bounded(empty(s), (round & 1u) ^ 1u, g.err, 21) || *abort_flag) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(S::kStage));
          tma_load_2d(sb + s * S::kStage, &map_a, kc * kGBK, m0, full(s));
          tma_load_2d(sb + s * S::kStage + S::kABytes, &map_b, kc * kGBK, n0, full(s));
        }
      }
      *issued_slot = it;
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA ---
    if (lane == 0) {
      int64_t it = 0;
      int last_slot = -1;
      uint32_t last_round = 0;
      int i = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x, ++i) {
        const int buf = i & 1;
        if (!mbar_wait_bounded(tempty(buf), (static_cast<uint32_t>(i >> 1) & 1u) ^ 1u, g.err, 22)) {
          *abort_flag = 1;
          break;
        }
        tcgen05_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
        bool ok = true;
        for (int kc = 0; kc < g.k_chunks; ++kc, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const uint32_t round = static_cast<uint32_t>(it / STAGES);
          if (!mbar_wait_bounded(full(s), round & 1u, g.err, 23) || *abort_flag) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tcgen05_fence_after();
          const uint32_t a = sb + s * S::kStage, b = a + S::kABytes;
#pragma unroll
          for (int kk = 0; kk < kGBK / 16; ++kk)
            umma_f16_ss(d, umma_desc_k_sw128(a + 32 * kk), umma_desc_k_sw128(b + 32 * kk), gemm_idesc<BN>(),
                        kc > 0 || kk > 0);
          umma_commit(empty(s));  // the slot is free once these MMAs have read it
          last_slot = s;
          last_round = round;
        }
        if (!ok) break;
        umma_commit(tfull(buf));
      }
      // Leave no MMA running: the last commit completes after every earlier MMA.
      if (last_slot >= 0)
        mbar_wait_bounded_ns(empty(last_slot), last_round & 1u, g.err, 25, kDrainNs);
    }
  } else {
    // ---------------------------------------------------------- epilogue ---
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int ew = warp - 2;
    const uint32_t stage0 = sb + S::kOut + static_cast<uint32_t>(ew * 2) * S::kOutBytes;
    unsigned char* stage0_ptr = smem + S::kOut + ew * 2 * S::kOutBytes;
    int ob = 0, i = 0;
    // Every decision below is warp-uniform: tcgen05.ld is a .sync.aligned
    // instruction that all 32 lanes must reach together.
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
      int mb, nb;
      tile_coords(g, tile, mb, nb);
      const int m0 = mb * kGBM, n0 = nb * BN;
      const int buf = i & 1;
      const bool ok = mbar_wait_bounded(tfull(buf), static_cast<uint32_t>(i >> 1) & 1u, g.err, 24);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tcgen05_fence_after();
      const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_x32(t_row + 32 * c, r);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
          w[j] = *reinterpret_cast<const uint32_t*>(&v);
        }
        if (lane == 0) bulk_wait_read<1>();  // the store that last read staging tile `ob` is done with it
        __syncwarp();
        unsigned char* st = stage0_ptr + ob * S::kOutBytes;
#pragma unroll
        for (int j = 0; j < 4; ++j)  // row `lane`: 64 bytes
          *reinterpret_cast<uint4*>(st + lane * 64 + 16 * j) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&map_c, stage0 + static_cast<uint32_t>(ob * S::kOutBytes), n0 + 32 * c, m0 + 32 * q);
          bulk_commit();
        }
        ob ^= 1;
      }
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(buf));
    }
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();  // the single-thread roles rejoin their warps before the CTA barrier
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    // Loads the MMA thread never consumed may still be landing: wait (bounded)
    // for the last STAGES the producer issued.
    const int64_t issued = *issued_slot;
    for (int64_t it = issued > STAGES ? issued - STAGES : 0; it < issued; ++it)
      mbar_wait_bounded_ns(full(static_cast<int>(it % STAGES)), static_cast<uint32_t>(it / STAGES) & 1u, g.err, 26,
                           kDrainNs);
  }
  tcgen05_fence_before();
  __syncthreads();
  if (warp == 1) {
    tcgen05_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

bool bf16_map2(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
               uint32_t box_outer, CUtensorMapSwizzle swz) {
  const uint64_t dims[2] = {inner, outer}, strides[1] = {inner * 2};
  const uint32_t box[2] = {box_inner, box_outer};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, swz);
}

template <int BN, int STAGES>
cudaError_t launch_gemm(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, int num_sms,
                        int* err, cudaStream_t st) {
  using S = GemmSmem<BN, STAGES>;
  CUtensorMap ma, mb, mc;
  if (!bf16_map2(&ma, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kGBK, kGBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mb, B, static_cast<uint64_t>(K), static_cast<uint64_t>(N), kGBK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mc, C, static_cast<uint64_t>(N), static_cast<uint64_t>(M), 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  GemmArgs g;
  const int64_t tm = (M + kGBM - 1) / kGBM, tn = (N + BN - 1) / BN, kc = (K + kGBK - 1) / kGBK;
  if (tm * tn > 0x7fffffff) return cudaErrorInvalidConfiguration;
  g.tiles_m = static_cast<int>(tm);
  g.tiles_n = static_cast<int>(tn);
  g.k_chunks = static_cast<int>(kc);
  g.group_m = static_cast<int>(tm < 16 ? tm : 16);
  g.err = err;
  const int smem = S::kTotal + 1024;
  auto kern = gemm_bf16_tn_kernel<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = tm * tn;
  const unsigned grid = static_cast<unsigned>(tiles < num_sms ? tiles : num_sms);
  kern<<<grid, kGThreads, smem, st>>>(ma, mb, mc, g);
  return cudaGetLastError();
}

}  // namespace

int gemm_choose_bn(int64_t M, int64_t N, int num_sms) {
  // Waves of tiles per SM x tile width, the 160-wide tile charged 10% more per
  // column for its lower FLOP-per-byte (measured on B200: 128-wide tiles ran
  // at half the rate of 256-wide ones, so they are not offered). 160 wins
  // where 256-wide tiles leave most of a last wave idle (out_proj at 2048
  // tokens: 160 tiles on 148 SMs).
  const int64_t tm = (M + kGBM - 1) / kGBM;
  const int64_t w256 = (tm * ((N + 255) / 256) + num_sms - 1) / num_sms;
  const int64_t w160 = (tm * ((N + 159) / 160) + num_sms - 1) / num_sms;
  return 11 * w160 * 160 < 10 * w256 * 256 ? 160 : 256;
}

cudaError_t gemm_bf16_tn(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, int bn,
                         int num_sms, int* err, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0 || N % 8 != 0) return cudaErrorInvalidValue;
  if (num_sms <= 0) num_sms = 148;
  if (bn == 0) bn = SSM_GEMM_FORCE_BN ? SSM_GEMM_FORCE_BN : gemm_choose_bn(M, N, num_sms);
  if (bn == 256) return launch_gemm<256, 4>(A, B, C, M, N, K, num_sms, err, st);
  if (bn == 160) return launch_gemm<160, 5>(A, B, C, M, N, K, num_sms, err, st);
  return cudaErrorInvalidValue;
}

}  // namespace ssm

extern "C" ssm_status ssm_proj_gemm(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K,
                                    void* stream) {
  using ssm::fail;
  if (M <= 0 || N <= 0 || K <= 0) return fail(SSM_ERR_INVALID_ARG, "M, N, K must be positive");
  if (K % 8 != 0 || N % 8 != 0) return fail(SSM_ERR_INVALID_ARG, "K and N must be multiples of 8");
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31))
    return fail(SSM_ERR_INVALID_ARG, "M, N, K must be at most 2^31");
  const void* p[3] = {A, W, C};
  const char* names[3] = {"A", "W", "C"};
  for (int i = 0; i < 3; ++i)
    if (!p[i] || !ssm::aligned(p[i], 16)) return fail(SSM_ERR_INVALID_ARG, "%s is NULL or not 16-byte aligned", names[i]);
  if (C == A || C == W) return fail(SSM_ERR_INVALID_ARG, "C must not alias A or W");
  int* err = ssm::device_error_ptr();
  if (!err) return fail(SSM_ERR_CUDA, "device error word: %s", cudaGetErrorString(cudaGetLastError()));
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const cudaError_t e = ssm::gemm_bf16_tn(A, W, C, M, N, K, 0, sms, err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "projection GEMM launch: %s", cudaGetErrorString(e));
  return fail(SSM_OK, "");
}
