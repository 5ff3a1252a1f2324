// gemm.cu -- the block's dense projections on the tensor cores (sm_100a):
// in_proj (D -> 2E) and out_proj (E -> D) of "Axon-SSM: selective state space
// model", "Algorithm" diagram, as C[M][N] = A[M][K] . B[N][K]^T with A and B
// bf16 row-major (both K-major), fp32 accumulation and a bf16 C.
//
// One persistent CTA per SM computes 128 x 256 output tiles. Six warps with
// fixed roles:
//   warp 0     TMA producer: the A tile [128][64] and the B tile [256][64] of
//              each 64-wide K chunk, 128-byte swizzled, into a 4-deep ring
//              (full / empty mbarriers per slot);
//   warp 1     MMA issuer: one thread issues four tcgen05.mma (M = 128,
//              N = 256, K = 16, kind::f16) per chunk into a TMEM accumulator,
//              commits each chunk to its slot's empty barrier and each
//              finished tile to the accumulator's full barrier; the two
//              accumulators (2 x 256 of the 512 TMEM columns) alternate, so
//              the next tile's MMAs run while the epilogue drains the last one;
//   warps 2-5  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its
//              quarter of the tile's rows) 32 columns at a time, rounds to
//              bf16, writes a [32][32] staging tile (two per warp, alternating)
//              and stores it with a TMA tile store, then frees the accumulator.
// Schedule. Whole tiles run round-robin over the CTAs, in a grouped raster
// (groups of 16 row blocks x every column block, row block fastest), so the
// CTAs running together share A row blocks and B column blocks in L2. What
// would be a partial last wave (between one and two tiles a CTA) is instead
// cut along K into equal runs of K chunks, one per CTA (stream-K): a tile cut
// between CTAs has every contributor write its fp32 partial and count itself
// in; the one that completes the count sums all partials in CTA order (so
// the result does not depend on who came last) and stores the tile. No CTA
// waits on another.
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
constexpr int kGBN = 256;  // tile columns: the MMA's N
constexpr int kGBK = 64;   // K chunk: 128 bytes of bf16, one swizzle row
constexpr int kStages = 4;
constexpr int kGThreads = 192;
constexpr int kMinChunksPerCta = 4;          // fewer CTAs for tiny problems
constexpr uint64_t kDrainNs = 200000000ull;  // 0.2 s: drain waits after an abort

struct GemmSmem {
  static constexpr int kABytes = kGBM * 128;
  static constexpr int kBBytes = kGBN * 128;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kOut = kStages * kStage;  // epilogue staging: 4 warps x 2 tiles of [32][32] bf16
  static constexpr int kOutBytes = 32 * 64;
  static constexpr int kBar = kOut + 8 * kOutBytes;  // full[S], empty[S], tfull[2], tempty[2], part, dec
  static constexpr int kTmemSlot = kBar + (2 * kStages + 6) * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kIssued = kTmemSlot + 8;     // int64: K chunks the producer issued
  static constexpr int kSplitFlag = kIssued + 8;    // int: this CTA completed its cut tile's count
  static constexpr int kTotal = kSplitFlag + 8;
  static constexpr uint32_t kTmemCols = 2 * kGBN;  // two accumulators
  static_assert(kStage % 1024 == 0, "swizzled operand tiles need 1 KB alignment");
};

struct GemmArgs {
  int tiles_m, tiles_n, k_chunks;
  int group_m;        // row blocks per raster group
  int ctas;           // persistent CTAs launched
  int dp_tiles;       // tiles computed whole, round-robin over the CTAs (a prefix of the raster)
  int64_t sk_chunks;  // K chunks of the stream-K part: (tiles - dp_tiles) * k_chunks
  float* partial;     // [ctas][2 slots] fp32 tiles of 128 x 256, each stored [warp quarter]
                      // [32-column chunk][float4 slot][lane]: every warp instruction
                      // moves 512 contiguous bytes
  int* counters;      // [tiles]: contributions counted so far, zero on entry
  int* err;
};

// First stream-K chunk of CTA u (u = ctas gives the end; all 0 without a
// stream-K part).
__device__ __forceinline__ int64_t sk_bound(const GemmArgs& g, int u) {
  return static_cast<int64_t>(u) * g.sk_chunks / g.ctas;
}

// The CTA whose stream-K run holds chunk `pos`.
__device__ __forceinline__ int sk_cta_of(const GemmArgs& g, int64_t pos) {
  int u = static_cast<int>(pos * g.ctas / g.sk_chunks);
  while (u + 1 < g.ctas && sk_bound(g, u + 1) <= pos) ++u;
  while (u > 0 && sk_bound(g, u) > pos) --u;
  return u;
}

// Partial slot of stream-K tile `tl` in CTA u's run: 0 if it is the run's
// first tile, else 1 (only a run's first and last tiles can be cut).
__device__ __forceinline__ int sk_slot(const GemmArgs& g, int u, int64_t tl) {
  return tl == sk_bound(g, u) / g.k_chunks ? 0 : 1;
}

// Float4 index of (CTA, slot, warp quarter q, 32-column chunk c, slot j,
// lane) in the partials.
__device__ __forceinline__ int64_t partial_index(int u, int slot, int q, int c, int j, int lane) {
  return (((((static_cast<int64_t>(u) * 2 + slot) * 4 + q) * 8 + c) * 8 + j) * 32) + lane;
}

// One tile's K range [k0, k1) in a CTA's walk.
struct Seg {
  int tile, k0, k1;
};

// The sequence of segments CTA u computes: its whole tiles, then its
// stream-K run. Every role walks the same sequence.
struct Walk {
  int u, w;
  int64_t pos, end;
  __device__ Walk(const GemmArgs& g, int u_) : u(u_), w(0), pos(sk_bound(g, u_)), end(sk_bound(g, u_ + 1)) {}
  __device__ bool next(const GemmArgs& g, Seg& s) {
    const int64_t t = u + static_cast<int64_t>(w) * g.ctas;
    if (t < g.dp_tiles) {
      s.tile = static_cast<int>(t);
      s.k0 = 0;
      s.k1 = g.k_chunks;
      ++w;
      return true;
    }
    if (pos >= end) return false;
    const int64_t kc = g.k_chunks, tl = pos / kc, rest = end - tl * kc;
    s.tile = static_cast<int>(g.dp_tiles + tl);
    s.k0 = static_cast<int>(pos - tl * kc);
    s.k1 = static_cast<int>(rest < kc ? rest : kc);
    pos = tl * kc + s.k1;
    return true;
  }
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

// bf16 x bf16 -> fp32, M = 128, N = 256, A and B K-major.
__host__ __device__ constexpr uint32_t gemm_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kGBN >> 3) << 17) |
         (static_cast<uint32_t>(kGBM >> 4) << 24);
}

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        const __grid_constant__ CUtensorMap map_c, const GemmArgs g) {
  using S = GemmSmem;
  constexpr int St = kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0), lane = tid & 31;
  const int cta = static_cast<int>(blockIdx.x);
  auto full = [&](int s) { return sb + S::kBar + 8 * s; };
  auto empty = [&](int s) { return sb + S::kBar + 8 * (St + s); };
  auto tfull = [&](int b) { return sb + S::kBar + 8 * (2 * St + b); };
  auto tempty = [&](int b) { return sb + S::kBar + 8 * (2 * St + 2 + b); };
  const uint32_t part_bar = sb + S::kBar + 8 * (2 * St + 4), dec_bar = sb + S::kBar + 8 * (2 * St + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kAbort);
  volatile int64_t* issued_slot = reinterpret_cast<volatile int64_t*>(smem + S::kIssued);
  volatile int* split_flag = reinterpret_cast<volatile int*>(smem + S::kSplitFlag);

  if (tid == 0) {
    *abort_flag = 0;
    *issued_slot = 0;
    for (int s = 0; s < St; ++s) {
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
      Walk wk(g, cta);
      Seg sg;
      while (!*abort_flag && wk.next(g, sg)) {
        int mb, nb;
        tile_coords(g, sg.tile, mb, nb);
        const int m0 = mb * kGBM, n0 = nb * kGBN;
        for (int kc = sg.k0; kc < sg.k1; ++kc, ++it) {
          const int s = static_cast<int>(it % St);
          const uint32_t round = static_cast<uint32_t>(it / St);
          if (!mbar_try_wait(empty(s), (round & 1u) ^ 1u) &&
              (*abort_flag || !mbar_wait_bounded_ns(empty(s), (round & 1u) ^ 1u, g.err, 21, 2000000000ull))) {
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
      Walk wk(g, cta);
      Seg sg;
      while (!*abort_flag && wk.next(g, sg)) {
        const int buf = i & 1;
        if (!mbar_wait_bounded(tempty(buf), (static_cast<uint32_t>(i >> 1) & 1u) ^ 1u, g.err, 22)) {
          *abort_flag = 1;
          break;
        }
        tcgen05_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * kGBN);
        bool ok = true;
        for (int kc = sg.k0; kc < sg.k1; ++kc, ++it) {
          const int s = static_cast<int>(it % St);
          const uint32_t round = static_cast<uint32_t>(it / St);
          // Fast path: the operands are usually in already; the abort flag
          // is read only when they are not.
          if (!mbar_try_wait(full(s), round & 1u) &&
              (*abort_flag || !mbar_wait_bounded_ns(full(s), round & 1u, g.err, 23, 2000000000ull))) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tcgen05_fence_after();
          // Descriptors of the slot's tiles; a 16-wide K step is 32 bytes
          // further along the swizzled rows (+2 in the address field).
          const uint64_t ad = umma_desc_k_sw128(sb + s * S::kStage);
          const uint64_t bd = umma_desc_k_sw128(sb + s * S::kStage + S::kABytes);
#pragma unroll
          for (int kk = 0; kk < kGBK / 16; ++kk)
            umma_f16_ss(d, ad + 2 * kk, bd + 2 * kk, gemm_idesc(), kc > sg.k0 || kk > 0);
          umma_commit(empty(s));  // the slot is free once these MMAs have read it
          last_slot = s;
          last_round = round;
        }
        if (!ok) break;
        umma_commit(tfull(buf));
        ++i;
      }
      // Leave no MMA running: the last commit completes after every earlier MMA.
      if (last_slot >= 0) mbar_wait_bounded_ns(empty(last_slot), last_round & 1u, g.err, 25, kDrainNs);
    }
  } else {
    // ---------------------------------------------------------- epilogue ---
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int ew = warp - 2;
    const uint32_t stage0 = sb + S::kOut + static_cast<uint32_t>(ew * 2) * S::kOutBytes;
    unsigned char* stage0_ptr = smem + S::kOut + ew * 2 * S::kOutBytes;
    int ob = 0, i = 0, np = 0;
    Walk wk(g, cta);
    Seg sg;
    // Every decision below is warp-uniform: tcgen05.ld is a .sync.aligned
    // instruction that all 32 lanes must reach together.
    while (wk.next(g, sg)) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
      int mb, nb;
      tile_coords(g, sg.tile, mb, nb);
      const int m0 = mb * kGBM, n0 = nb * kGBN;
      const int buf = i & 1;
      const bool ok = mbar_wait_bounded(tfull(buf), static_cast<uint32_t>(i >> 1) & 1u, g.err, 24);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tcgen05_fence_after();
      const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * kGBN);
      const bool whole = sg.k0 == 0 && sg.k1 == g.k_chunks;
      bool store = true;
      int u_lo = cta, u_hi = cta;
      int64_t tl = 0;
      if (!whole) {
        // A tile cut between CTAs: publish this CTA's partial; the contributor
        // that completes the count sums them all.
        tl = sg.tile - static_cast<int64_t>(g.dp_tiles);
        u_lo = sk_cta_of(g, tl * g.k_chunks);
        u_hi = sk_cta_of(g, tl * g.k_chunks + g.k_chunks - 1);
        float4* mine = reinterpret_cast<float4*>(g.partial) + partial_index(cta, sk_slot(g, cta, tl), q, 0, 0, lane);
#pragma unroll 1
        for (int c = 0; c < kGBN / 32; ++c) {
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
        // all four publish their rows, then one thread counts the tile in.
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(part_bar);
        if (warp == 2 && lane == 0) {
          const bool okp = mbar_wait_bounded(part_bar, static_cast<uint32_t>(np) & 1u, g.err, 27);
          if (!okp) *abort_flag = 1;
          *split_flag = okp && atomicAdd(g.counters + sg.tile, 1) == u_hi - u_lo;
          mbar_arrive(dec_bar);  // also after a timeout, so the others do not wait in vain
        }
        const bool okd = mbar_wait_bounded(dec_bar, static_cast<uint32_t>(np) & 1u, g.err, 28);
        ++np;
        if (!__all_sync(0xffffffffu, okd)) {
          if (lane == 0) *abort_flag = 1;
          break;
        }
        store = *split_flag != 0;
        if (store) __threadfence();  // the other contributors' partials, published before their increments
      }
      if (store) {
#pragma unroll 1
        for (int c = 0; c < kGBN / 32; ++c) {
          float v[32];
          if (whole) {
            uint32_t r[32];
            tmem_ld_x32(t_row + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          } else {
            // Contributors in CTA order; the next one's loads are in flight
            // while the current one is added.
            auto fetch = [&](int u, float4 (&dst)[8]) {
              const float4* src =
                  reinterpret_cast<const float4*>(g.partial) + partial_index(u, sk_slot(g, u, tl), q, c, 0, lane);
#pragma unroll
              for (int j = 0; j < 8; ++j) dst[j] = __ldcg(src + j * 32);
            };
            float4 cur[8], nxt[8];
            fetch(u_lo, cur);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
            for (int u = u_lo; u <= u_hi; ++u) {
              if (u < u_hi) fetch(u + 1, nxt);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                v[4 * j] += cur[j].x, v[4 * j + 1] += cur[j].y, v[4 * j + 2] += cur[j].z, v[4 * j + 3] += cur[j].w;
                cur[j] = nxt[j];
              }
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
      ++i;
    }
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();  // the single-thread roles rejoin their warps before the CTA barrier
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    // Loads the MMA thread never consumed may still be landing: wait (bounded)
    // for the last kStages the producer issued.
    const int64_t issued = *issued_slot;
    for (int64_t it = issued > St ? issued - St : 0; it < issued; ++it)
      mbar_wait_bounded_ns(full(static_cast<int>(it % St)), static_cast<uint32_t>(it / St) & 1u, g.err, 26,
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

// How a GEMM is spread over the persistent CTAs.
struct GemmPlan {
  int64_t tiles_m, tiles_n, k_chunks, tiles;
  int ctas;
  int64_t dp_tiles, sk_chunks;
  bool partials;  // some stream-K tile is cut between CTAs (workspace needed)
};

GemmPlan gemm_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
  GemmPlan pl;
  pl.tiles_m = (M + kGBM - 1) / kGBM;
  pl.tiles_n = (N + kGBN - 1) / kGBN;
  pl.k_chunks = (K + kGBK - 1) / kGBK;
  pl.tiles = pl.tiles_m * pl.tiles_n;
  const int64_t total = pl.tiles * pl.k_chunks;
  int64_t ctas = num_sms > 0 ? num_sms : 148;
  const int64_t by_work = total / kMinChunksPerCta;
  if (ctas > by_work) ctas = by_work > 0 ? by_work : 1;
  pl.ctas = static_cast<int>(ctas);
  // Whole tiles round-robin; a last wave that would leave most CTAs idle is
  // replaced by cutting the final one to two tiles a CTA along K into equal
  // runs (stream-K). The cut tiles cost up to about 3/4 of a wave (fp32
  // partials written, read back and summed), so K is cut only where that
  // saves more: measured on B200, out_proj at 2048 tokens (160 tiles on 148
  // SMs) 110 -> 93 us, while in_proj at 2048 tokens (6.5 waves) lost 7%.
  const int64_t whole_waves = (pl.tiles + ctas - 1) / ctas;
  const bool cut =
      static_cast<double>(pl.tiles) / static_cast<double>(ctas) + 0.75 <= static_cast<double>(whole_waves);
  const int64_t dp_waves = cut ? (pl.tiles >= ctas ? pl.tiles / ctas - 1 : 0) : whole_waves;
  pl.dp_tiles = dp_waves * ctas < pl.tiles ? dp_waves * ctas : pl.tiles;
  pl.sk_chunks = (pl.tiles - pl.dp_tiles) * pl.k_chunks;
  pl.partials = false;
  for (int64_t u = 1; u < ctas; ++u)
    if ((u * pl.sk_chunks / ctas) % pl.k_chunks != 0) pl.partials = true;
  return pl;
}

size_t partial_bytes(const GemmPlan& pl) { return static_cast<size_t>(pl.ctas) * 2 * kGBM * kGBN * 4; }

cudaError_t launch_gemm(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* ws,
                        size_t ws_bytes, int num_sms, int* err, cudaStream_t st) {
  using S = GemmSmem;
  const GemmPlan pl = gemm_plan(M, N, K, num_sms);
  if (pl.tiles >= (int64_t(1) << 30)) return cudaErrorInvalidConfiguration;
  CUtensorMap ma, mb, mc;
  if (!bf16_map2(&ma, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kGBK, kGBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mb, B, static_cast<uint64_t>(K), static_cast<uint64_t>(N), kGBK, kGBN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mc, C, static_cast<uint64_t>(N), static_cast<uint64_t>(M), 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  GemmArgs g;
  g.tiles_m = static_cast<int>(pl.tiles_m);
  g.tiles_n = static_cast<int>(pl.tiles_n);
  g.k_chunks = static_cast<int>(pl.k_chunks);
  g.group_m = static_cast<int>(pl.tiles_m < 16 ? pl.tiles_m : 16);
  g.ctas = pl.ctas;
  g.dp_tiles = static_cast<int>(pl.dp_tiles);
  g.sk_chunks = pl.sk_chunks;
  g.partial = nullptr;
  g.counters = nullptr;
  g.err = err;
  if (pl.partials) {
    if (!ws || ws_bytes < gemm_workspace_bytes(M, N, K, num_sms)) return cudaErrorInvalidValue;
    g.partial = static_cast<float*>(ws);
    g.counters = reinterpret_cast<int*>(static_cast<char*>(ws) + partial_bytes(pl));
    cudaError_t e = cudaMemsetAsync(g.counters, 0, static_cast<size_t>(pl.tiles) * sizeof(int), st);
    if (e != cudaSuccess) return e;
  }
  const int smem = S::kTotal + 1024;
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gemm_bf16_tn_kernel<<<static_cast<unsigned>(pl.ctas), kGThreads, smem, st>>>(ma, mb, mc, g);
  return cudaGetLastError();
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  const GemmPlan pl = gemm_plan(M, N, K, num_sms);
  if (!pl.partials) return 0;
  return partial_bytes(pl) + static_cast<size_t>(pl.tiles) * sizeof(int);
}

cudaError_t gemm_bf16_tn(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* ws,
                         size_t ws_bytes, int num_sms, int* err, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0 || N % 8 != 0) return cudaErrorInvalidValue;
  if (num_sms <= 0) num_sms = 148;
  return launch_gemm(A, B, C, M, N, K, ws, ws_bytes, num_sms, err, st);
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
