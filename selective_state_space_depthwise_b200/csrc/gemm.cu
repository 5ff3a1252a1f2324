// gemm.cu -- the block's dense projections on the tensor cores (sm_100a):
// in_proj (D -> 2E) and out_proj (E -> D) of "Axon-SSM: selective state space
// model", "Algorithm" diagram, as C[M][N] = A[M][K] . B[N][K]^T with A and B
// bf16 row-major (both K-major), fp32 accumulation and a bf16 C.
//
// One persistent CTA per SM walks output tiles of 128 x BN (BN = 256)
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
  static constexpr int kSplitFlag = kIssued + 8;  // int: this unit finished its tile (split K)
  static constexpr int kPartBar = kSplitFlag + 8;  // split K: the 4 epilogue warps published their rows
  static constexpr int kDecBar = kPartBar + 8;     // split K: the unit's tile counter was read
  static constexpr int kTotal = kDecBar + 8;
  // TMEM columns: two accumulators of BN, allocated as a power of two.
  static constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256u : 512u;
  static_assert(kStage % 1024 == 0, "swizzled operand tiles need 1 KB alignment");
};

struct GemmArgs {
  int tiles_m, tiles_n, k_chunks;
  int group_m;      // row blocks per raster group
  int nsplit;       // K slices per tile (work units = tiles x nsplit)
  float* partial;   // nsplit > 1: [tiles][nsplit] fp32 partial tiles of 128 x BN, each stored
                    // [warp quarter][32-column chunk][float4 slot][lane] so every warp
                    // instruction moves 512 contiguous bytes
  int* counters;    // nsplit > 1: [tiles], zero on entry: slices of each tile finished
  int* err;
};

// Float4 index of (tile, slice, warp quarter q, 32-column chunk c, slot j,
// lane) in the split-K partials: a warp's 32 lanes are adjacent.
__device__ __forceinline__ int64_t partial_index(const GemmArgs& g, int tile, int split, int q, int c, int j,
                                                int lane) {
  constexpr int kChunks = 256 / 32;  // BN / 32 at the only built width
  return ((((static_cast<int64_t>(tile) * g.nsplit + split) * 4 + q) * kChunks + c) * 8 + j) * 32 + lane;
}

// Work unit -> its tile and K-chunk range: the nsplit slices of a tile are
// consecutive units, so consecutive CTAs run them at the same time.
__device__ __forceinline__ void unit_range(const GemmArgs& g, int unit, int& tile, int& split, int& k0, int& k1) {
  tile = unit / g.nsplit;
  split = unit - tile * g.nsplit;
  k0 = static_cast<int>(static_cast<int64_t>(split) * g.k_chunks / g.nsplit);
  k1 = static_cast<int>(static_cast<int64_t>(split + 1) * g.k_chunks / g.nsplit);
}

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
  static_assert(BN == 256, "the split-K partial layout (partial_index) is built for 256-wide tiles");
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
  volatile int* split_flag = reinterpret_cast<volatile int*>(smem + S::kSplitFlag);
  const uint32_t part_bar = sb + S::kPartBar, dec_bar = sb + S::kDecBar;
  const int nunits = g.tiles_m * g.tiles_n * g.nsplit;

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
    mbar_init(part_bar, 4);
    mbar_init(dec_bar, 1);
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
      for (int unit = blockIdx.x; unit < nunits && !*abort_flag; unit += gridDim.x) {
        int tile, split, k0, k1, mb, nb;
        unit_range(g, unit, tile, split, k0, k1);
        tile_coords(g, tile, mb, nb);
        const int m0 = mb * kGBM, n0 = nb * BN;
        for (int kc = k0; kc < k1; ++kc, ++it) {
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
      for (int unit = blockIdx.x; unit < nunits && !*abort_flag; unit += gridDim.x, ++i) {
        int tile, split, k0, k1;
        unit_range(g, unit, tile, split, k0, k1);
        const int buf = i & 1;
        if (!mbar_wait_bounded(tempty(buf), (static_cast<uint32_t>(i >> 1) & 1u) ^ 1u, g.err, 22)) {
          *abort_flag = 1;
          break;
        }
        tcgen05_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
        bool ok = true;
        for (int kc = k0; kc < k1; ++kc, ++it) {
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
                        kc > k0 || kk > 0);
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
    for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x, ++i) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
      int tile, split, k0, k1, mb, nb;
      unit_range(g, unit, tile, split, k0, k1);
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
      bool store = true;  // this unit writes the bf16 tile
      if (g.nsplit > 1) {
        // Every slice publishes its fp32 partial; the slice that finishes the
        // tile last adds the others to its own and writes the output.
        float4* mine = reinterpret_cast<float4*>(g.partial) + partial_index(g, tile, split, q, 0, 0, lane);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_x32(t_row + 32 * c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mine[(c * 8 + j) * 32] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
        }
        // Handshake of the four epilogue warps on two mbarriers (bounded
        // waits, so a warp that left on an abort cannot strand the others):
        // all four publish their rows, then one thread counts the slice in.
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(part_bar);
        if (warp == 2 && lane == 0) {
          const bool okp = mbar_wait_bounded(part_bar, static_cast<uint32_t>(i) & 1u, g.err, 27);
          if (!okp) *abort_flag = 1;
          *split_flag = okp && atomicAdd(g.counters + tile, 1) == g.nsplit - 1;
          mbar_arrive(dec_bar);  // also after a timeout, so the others do not wait in vain
        }
        const bool okd = mbar_wait_bounded(dec_bar, static_cast<uint32_t>(i) & 1u, g.err, 28);
        if (!__all_sync(0xffffffffu, okd)) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        store = *split_flag != 0;
        if (store) __threadfence();  // the other slices' partials, published before their increments
      }
      if (store) {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_x32(t_row + 32 * c, r);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          for (int o = 0; o < g.nsplit; ++o) {
            if (o == split) continue;
            const float4* other = reinterpret_cast<const float4*>(g.partial) + partial_index(g, tile, o, q, c, 0, lane);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 p = __ldcg(other + j * 32);
              v[4 * j] += p.x, v[4 * j + 1] += p.y, v[4 * j + 2] += p.z, v[4 * j + 3] += p.w;
            }
          }
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const __nv_bfloat162 bv = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            w[j] = *reinterpret_cast<const uint32_t*>(&bv);
          }
          if (lane == 0) bulk_wait_read<1>();  // the store that last read staging tile `ob` is done with it
          __syncwarp();
          unsigned char* st = stage0_ptr + ob * S::kOutBytes;
#pragma unroll
          for (int j = 0; j < 4; ++j)  // row `lane`: 64 bytes
            *reinterpret_cast<uint4*>(st + lane * 64 + 16 * j) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&map_c, stage0 + static_cast<uint32_t>(ob * S::kOutBytes), n0 + 32 * c, m0 + 32 * q);
            bulk_commit();
          }
          ob ^= 1;
        }
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
cudaError_t launch_gemm(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, int nsplit,
                        void* ws, int num_sms, int* err, cudaStream_t st) {
  using S = GemmSmem<BN, STAGES>;
  CUtensorMap ma, mb, mc;
  if (!bf16_map2(&ma, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kGBK, kGBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mb, B, static_cast<uint64_t>(K), static_cast<uint64_t>(N), kGBK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mc, C, static_cast<uint64_t>(N), static_cast<uint64_t>(M), 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  GemmArgs g;
  const int64_t tm = (M + kGBM - 1) / kGBM, tn = (N + BN - 1) / BN, kc = (K + kGBK - 1) / kGBK;
  const int64_t units = tm * tn * nsplit;
  if (units > 0x7fffffff) return cudaErrorInvalidConfiguration;
  g.tiles_m = static_cast<int>(tm);
  g.tiles_n = static_cast<int>(tn);
  g.k_chunks = static_cast<int>(kc);
  g.group_m = static_cast<int>(tm < 16 ? tm : 16);
  g.nsplit = nsplit;
  g.partial = nullptr;
  g.counters = nullptr;
  g.err = err;
  if (nsplit > 1) {
    if (!ws) return cudaErrorInvalidValue;
    g.partial = static_cast<float*>(ws);
    g.counters = reinterpret_cast<int*>(static_cast<char*>(ws) + static_cast<size_t>(tm * tn * nsplit) * kGBM * BN * 4);
    cudaError_t e = cudaMemsetAsync(g.counters, 0, static_cast<size_t>(tm * tn) * sizeof(int), st);
    if (e != cudaSuccess) return e;
  }
  const int smem = S::kTotal + 1024;
  auto kern = gemm_bf16_tn_kernel<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(units < num_sms ? units : num_sms);
  kern<<<grid, kGThreads, smem, st>>>(ma, mb, mc, g);
  return cudaGetLastError();
}

}  // namespace

int gemm_choose_bn(int64_t /*M*/, int64_t /*N*/, int /*num_sms*/) {
  // 256 columns: measured on B200, narrower tiles (160, 128) ran at 0.5 - 0.9
  // of its rate on every projection shape, even where they left fewer SMs idle
  // in the last wave (they read more operand bytes per FLOP).
  return 256;
}

int gemm_choose_split(int64_t M, int64_t N, int64_t K, int num_sms) {
  // K slices per tile when whole tiles would leave most of a last wave idle:
  // minimise waves / slices, each extra slice charged 4% for its fp32 partial
  // (written once, read once by the slice that finishes the tile); at least 8
  // K chunks per slice. out_proj at 2048 tokens: 160 tiles on 148 SMs -> 4
  // slices (5 waves of quarter tiles instead of 2 of whole ones).
  if (num_sms <= 0) num_sms = 148;
  const int64_t tiles = ((M + kGBM - 1) / kGBM) * ((N + 255) / 256), kc = (K + kGBK - 1) / kGBK;
  int best = 1;
  double best_cost = static_cast<double>((tiles + num_sms - 1) / num_sms);
  for (int ns = 2; ns <= 4 && kc / ns >= 8; ++ns) {
    const double cost = static_cast<double>((tiles * ns + num_sms - 1) / num_sms) / ns * (1.0 + 0.04 * ns);
    if (cost < best_cost) best = ns, best_cost = cost;
  }
  return best;
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  const int ns = gemm_choose_split(M, N, K, num_sms);
  if (ns == 1) return 0;
  const int64_t tiles = ((M + kGBM - 1) / kGBM) * ((N + 255) / 256);
  return static_cast<size_t>(tiles * ns) * kGBM * 256 * 4 + static_cast<size_t>(tiles) * sizeof(int);
}

cudaError_t gemm_bf16_tn(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* ws,
                         size_t ws_bytes, int num_sms, int* err, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0 || N % 8 != 0) return cudaErrorInvalidValue;
  if (num_sms <= 0) num_sms = 148;
  const int bn = SSM_GEMM_FORCE_BN ? SSM_GEMM_FORCE_BN : gemm_choose_bn(M, N, num_sms);
  int ns = gemm_choose_split(M, N, K, num_sms);
  if (ns > 1 && (!ws || ws_bytes < gemm_workspace_bytes(M, N, K, num_sms))) return cudaErrorInvalidValue;
  if (bn == 256) return launch_gemm<256, 4>(A, B, C, M, N, K, ns, ws, num_sms, err, st);
  return cudaErrorInvalidValue;
}

}  // namespace ssm

extern "C" size_t ssm_proj_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();  // no device: the default SM count
  return ssm::gemm_workspace_bytes(M, N, K, sms);
}

extern "C" ssm_status ssm_proj_gemm(const void* A, const void* W, void* C, int64_t M, int64_t N, int64_t K,
                                    void* workspace, size_t workspace_bytes, void* stream) {
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
  const size_t need = ssm_proj_gemm_workspace_bytes(M, N, K);
  if (need && (!workspace || !ssm::aligned(workspace, 256) || workspace_bytes < need))
    return fail(SSM_ERR_INVALID_ARG, "workspace: need %zu bytes, 256-byte aligned (got %zu)", need, workspace_bytes);
  int* err = ssm::device_error_ptr();
  if (!err) return fail(SSM_ERR_CUDA, "device error word: %s", cudaGetErrorString(cudaGetLastError()));
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const cudaError_t e =
      ssm::gemm_bf16_tn(A, W, C, M, N, K, workspace, workspace_bytes, sms, err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "projection GEMM launch: %s", cudaGetErrorString(e));
  return fail(SSM_OK, "");
}
