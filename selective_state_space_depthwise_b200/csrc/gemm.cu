// gemm.cu -- the block's dense projections on the tensor cores (sm_100a):
// in_proj (D -> 2E) and out_proj (E -> D) of "Axon-SSM: selective state space
// model", "Algorithm" diagram, as C[M][N] = A[M][K] . B[N][K]^T with A and B
// bf16 row-major (both K-major), fp32 accumulation and a bf16 C.
//
// CTA pairs. A cluster of two CTAs on two SMs computes 256 x 256 output
// tiles with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): each CTA
// stages 128 rows of A and 128 rows of B per K chunk, so an SM reads 32 KB of
// operands per 64-wide chunk instead of the 48 KB a one-SM 128 x 256 tile
// needs for the same MMA work (measured on B200: 4-10% faster than the
// one-SM tile at every projection shape). Six warps a CTA:
//   warp 0     TMA producer (both CTAs): its A and B halves of each chunk,
//              128-byte swizzled, into a 6-deep ring; the pair's completion
//              is counted on rank 0's full barrier (rank 0 expects the bytes
//              of both CTAs);
//   warp 1     MMA issuer (rank 0 only): four MMAs per chunk into a TMEM
//              accumulator, the slot's barrier tested inline and the abort
//              flag read only when the slot is not ready (a call and a
//              volatile read per chunk drained the tensor pipe: 62% -> 76%
//              busy once removed); each chunk's commit frees the ring slot in both
//              CTAs, each tile's commit hands both CTAs' accumulators to their
//              epilogues; two accumulators (2 x 256 of the 512 TMEM columns)
//              alternate, so the next tile's MMAs run while the epilogues
//              drain the last one;
//   warps 2-5  epilogue (both CTAs): warp w reads TMEM lanes 32 (w % 4)..+31
//              (its quarter of the CTA's 128 rows) 32 columns at a time,
//              rounds to bf16 into a [32][32] staging tile and stores it by
//              TMA, then counts itself in on rank 0's accumulator-free barrier.
// Schedule. Whole tiles run round-robin over the pairs, in a grouped raster
// (groups of 16 row blocks x every column block, row block fastest), so the
// pairs running together share A row blocks and B column blocks in L2. Where
// a partial last wave would idle most pairs (tiles / pairs + 3/4 <= whole
// waves), the final one to two tiles a pair are instead cut along K into
// equal runs of K chunks, one per pair (stream-K):
// a tile cut between pairs has every contributing CTA write its fp32 partial
// and count itself in; the one that completes the count adds the other's
// partial to its own accumulator (two contributors) or sums all partials in
// pair order (more), so the result does not depend on who came last, and
// stores the tile. No CTA waits on another pair.
// Tails: TMA loads past M, N or K read zeros; stores are clipped at M and N.
// Every mbarrier wait is bounded; a wait that gives up sets the device error
// word and the CTA's abort flag, every role leaves its loop, the waits that
// drain in-flight work give up after 0.2 s, an aborting CTA pauses 1 ms for
// loads still landing, and TMEM is freed once both CTAs are done.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "ssm.h"
#include "ssm_internal.h"
#include "tma_map.cuh"

namespace ssm {
namespace {

constexpr int kTileM = 256;  // tile rows per CTA pair: the MMA's M
constexpr int kHalfM = 128;  // rows per CTA: one TMEM lane per row
constexpr int kTileN = 256;  // tile columns: the MMA's N
constexpr int kHalfN = 128;  // B rows staged per CTA
constexpr int kGBK = 64;     // K chunk: 128 bytes of bf16, one swizzle row
constexpr int kStages = 6;
constexpr int kGThreads = 192;
constexpr int kMinChunksPerPair = 4;          // fewer pairs for tiny problems
constexpr uint64_t kDrainNs = 200000000ull;   // 0.2 s: drain waits
constexpr uint64_t kAbortPauseNs = 1000000ull;  // 1 ms: loads landing after an abort

struct GemmSmem {
  static constexpr int kABytes = kHalfM * 128;  // [128][64] bf16
  static constexpr int kBBytes = kHalfN * 128;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr uint32_t kTxPair = 2u * kStage;  // bytes of one chunk over both CTAs
  static constexpr int kOut = kStages * kStage;     // epilogue staging: 4 warps x 2 tiles of [32][32] bf16
  static constexpr int kOutBytes = 32 * 64;
  static constexpr int kBar = kOut + 8 * kOutBytes;  // full[S], empty[S], tfull[2], tempty[2], part, dec
  static constexpr int kTmemSlot = kBar + (2 * kStages + 6) * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kSplitFlag = kTmemSlot + 8;  // int: this CTA completed its half tile's count
  static constexpr int kTotal = kSplitFlag + 8;
  static constexpr uint32_t kTmemCols = 512;  // two accumulators of 256 columns
  static_assert(kStage % 1024 == 0, "swizzled operand tiles need 1 KB alignment");
};

struct GemmArgs {
  int tiles_m, tiles_n, k_chunks;
  int group_m;        // row blocks per raster group
  int pairs;          // CTA pairs launched
  int dp_waves;       // rounds of whole tiles before the stream-K part (the last one partial
                      // when nothing is cut)
  int64_t sk_chunks;  // K chunks of the stream-K part: (tiles - dp_waves * pairs) * k_chunks,
                      // 0 when nothing is cut
  float* partial;     // [pairs][2 slots][2 halves] fp32 half tiles of 128 x 256, each stored
                      // [warp quarter][32-column chunk][float4 slot][lane]: every warp
                      // instruction moves 512 contiguous bytes
  int* counters;      // [tiles][2 halves]: contributions counted so far, zero on entry; the
                      // contributor that completes a count sets it back to zero
  int* err;
};

// First stream-K chunk of pair p (p = pairs gives the end).
__device__ __forceinline__ int64_t sk_bound(const GemmArgs& g, int p) {
  return static_cast<int64_t>(p) * g.sk_chunks / g.pairs;
}

// The pair whose stream-K run holds chunk `pos`.
__device__ __forceinline__ int sk_pair_of(const GemmArgs& g, int64_t pos) {
  int p = static_cast<int>(pos * g.pairs / g.sk_chunks);
  while (p + 1 < g.pairs && sk_bound(g, p + 1) <= pos) ++p;
  while (p > 0 && sk_bound(g, p) > pos) --p;
  return p;
}

// Partial slot of stream-K tile `tl` in pair p's run: 0 if it is the run's
// first tile, else 1 (only a run's first and last tiles can be cut).
__device__ __forceinline__ int sk_slot(const GemmArgs& g, int p, int64_t tl) {
  return tl == sk_bound(g, p) / g.k_chunks ? 0 : 1;
}

// Float4 index of (pair, slot, half, warp quarter q, 32-column chunk c, slot
// j, lane) in the partials.
__device__ __forceinline__ int64_t partial_index(int p, int slot, int half, int q, int c, int j, int lane) {
  return ((((((static_cast<int64_t>(p) * 2 + slot) * 2 + half) * 4 + q) * 8 + c) * 8 + j) * 32) + lane;
}

// One tile's K range [k0, k1) in a pair's walk.
struct Seg {
  int tile, k0, k1;
};

// The sequence of segments pair p computes: its whole tiles, then its
// stream-K run. Every role of both CTAs walks the same sequence.
struct Walk {
  int p, w;
  int64_t pos, end;
  __device__ Walk(const GemmArgs& g, int p_) : p(p_), w(0), pos(sk_bound(g, p_)), end(sk_bound(g, p_ + 1)) {}
  __device__ bool next(const GemmArgs& g, Seg& s) {
    if (w < g.dp_waves && p + static_cast<int64_t>(w) * g.pairs < static_cast<int64_t>(g.tiles_m) * g.tiles_n) {
      s.tile = p + w * g.pairs;
      s.k0 = 0;
      s.k1 = g.k_chunks;
      ++w;
      return true;
    }
    if (pos >= end) return false;
    const int64_t kc = g.k_chunks, tl = pos / kc, rest = end - tl * kc;
    s.tile = static_cast<int>(static_cast<int64_t>(g.dp_waves) * g.pairs + tl);
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

// bf16 x bf16 -> fp32, M = 256 (over the pair), N = 256, A and B K-major.
__host__ __device__ constexpr uint32_t gemm_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kTileN >> 3) << 17) |
         (static_cast<uint32_t>(kTileM >> 4) << 24);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    gemm_bf16_tn_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        const __grid_constant__ CUtensorMap map_c, const GemmArgs g) {
  using S = GemmSmem;
  constexpr int St = kStages;
  extern __shared__ unsigned char smem_raw[];
  // Same offset in both CTAs (same kernel, same static layout): the MMA
  // descriptors of rank 0 address the peer's operands too.
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0), lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  auto full = [&](int s) { return sb + S::kBar + 8 * s; };
  auto empty = [&](int s) { return sb + S::kBar + 8 * (St + s); };
  auto tfull = [&](int b) { return sb + S::kBar + 8 * (2 * St + b); };
  auto tempty = [&](int b) { return sb + S::kBar + 8 * (2 * St + 2 + b); };
  const uint32_t part_bar = sb + S::kBar + 8 * (2 * St + 4), dec_bar = sb + S::kBar + 8 * (2 * St + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kAbort);
  volatile int* split_flag = reinterpret_cast<volatile int*>(smem + S::kSplitFlag);

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < St; ++s) {
      mbar_init(full(s), 1);   // rank 0's: its producer's expect_tx arrival
      mbar_init(empty(s), 1);  // one multicast commit per use
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull(b), 1);
      mbar_init(tempty(b), 8);  // rank 0's: one arrival per epilogue warp of each CTA
    }
    mbar_init(part_bar, 4);
    mbar_init(dec_bar, 1);
    mbar_fence_init();
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
    prefetch_tensormap(&map_c);
  }
  if (warp == 1) {
    tmem_alloc_pair(sb + S::kTmemSlot, S::kTmemCols);
    tmem_relinquish_pair();
  }
  tcgen05_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrival
  tcgen05_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + S::kTmemSlot);
  // Launched overlapped with the kernel before it (programmatic dependent
  // launch): the setup above ran during its tail; global memory is touched
  // only after it has finished. Without that launch attribute it returns at
  // once.
  griddep_wait();

  if (warp == 0) {
    // ---------------------------------------------------------- producer ---
    if (lane == 0) {
      int64_t it = 0;
      Walk wk(g, pair);
      Seg sg;
      while (!*abort_flag && wk.next(g, sg)) {
        int mb, nb;
        tile_coords(g, sg.tile, mb, nb);
        const int m0 = mb * kTileM + static_cast<int>(rank) * kHalfM;
        const int n0 = nb * kTileN + static_cast<int>(rank) * kHalfN;
        for (int kc = sg.k0; kc < sg.k1; ++kc, ++it) {
          const int s = static_cast<int>(it % St);
          const uint32_t round = static_cast<uint32_t>(it / St);
          if (!mbar_try_wait(empty(s), (round & 1u) ^ 1u) &&
              (*abort_flag || !mbar_wait_bounded_ns(empty(s), (round & 1u) ^ 1u, g.err, 21, 2000000000ull))) {
            *abort_flag = 1;
            break;
          }
          const uint32_t fb = mapa_shared(full(s), 0);
          if (rank == 0) mbar_arrive_expect_tx(full(s), S::kTxPair);
          tma_load_2d_pair(sb + s * S::kStage, &map_a, kc * kGBK, m0, fb);
          tma_load_2d_pair(sb + s * S::kStage + S::kABytes, &map_b, kc * kGBK, n0, fb);
        }
      }
      // The commits of the last chunks reach this CTA's empty barriers before
      // the CTA may leave (rank 0 commits them to both CTAs).
      for (int64_t j = it > St ? it - St : 0; j < it; ++j)
        mbar_wait_bounded_ns(empty(static_cast<int>(j % St)), static_cast<uint32_t>(j / St) & 1u, g.err, 29,
                             kDrainNs);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA ---
    if (rank == 0 && lane == 0) {
      int64_t it = 0;
      int last_slot = -1;
      uint32_t last_round = 0;
      int i = 0;
      Walk wk(g, pair);
      Seg sg;
      while (!*abort_flag && wk.next(g, sg)) {
        const int buf = i & 1;
        if (!mbar_wait_bounded(tempty(buf), (static_cast<uint32_t>(i >> 1) & 1u) ^ 1u, g.err, 22)) {
          *abort_flag = 1;
          break;
        }
        tcgen05_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * 256);
        bool ok = true;
        for (int kc = sg.k0; kc < sg.k1; ++kc, ++it) {
          const int s = static_cast<int>(it % St);
          const uint32_t round = static_cast<uint32_t>(it / St);
          if (!mbar_try_wait(full(s), round & 1u) &&
              (*abort_flag || !mbar_wait_bounded_ns(full(s), round & 1u, g.err, 23, 2000000000ull))) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tcgen05_fence_after();
          const uint64_t ad = umma_desc_k_sw128(sb + s * S::kStage);
          const uint64_t bd = umma_desc_k_sw128(sb + s * S::kStage + S::kABytes);
#pragma unroll
          for (int kk = 0; kk < kGBK / 16; ++kk)
            umma_f16_ss_pair(d, ad + 2 * kk, bd + 2 * kk, gemm_idesc(), kc > sg.k0 || kk > 0);
          umma_commit_pair(empty(s), 0x3);  // the slot is free in both CTAs once these MMAs have read it
          last_slot = s;
          last_round = round;
        }
        if (!ok) break;
        umma_commit_pair(tfull(buf), 0x3);
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
    const int half = static_cast<int>(rank);
    int ob = 0, i = 0, np = 0;
    Walk wk(g, pair);
    Seg sg;
    // Every decision below is warp-uniform: tcgen05.ld is a .sync.aligned
    // instruction that all 32 lanes must reach together.
    while (wk.next(g, sg)) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
      int mb, nb;
      tile_coords(g, sg.tile, mb, nb);
      const int m0 = mb * kTileM + half * kHalfM, n0 = nb * kTileN;
      const int buf = i & 1;
      const bool ok = mbar_wait_bounded(tfull(buf), static_cast<uint32_t>(i >> 1) & 1u, g.err, 24);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      tcgen05_fence_after();
      const uint32_t t_row = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * 256);
      const bool whole = sg.k0 == 0 && sg.k1 == g.k_chunks;
      bool store = true;
      int p_lo = pair, p_hi = pair;
      int64_t tl = 0;
      if (!whole) {
        // A tile cut between pairs: publish this CTA's partial half tile; the
        // contributor that completes the count sums them all.
        tl = sg.tile - static_cast<int64_t>(g.dp_waves) * g.pairs;
        p_lo = sk_pair_of(g, tl * g.k_chunks);
        p_hi = sk_pair_of(g, tl * g.k_chunks + g.k_chunks - 1);
        float4* mine = reinterpret_cast<float4*>(g.partial) + partial_index(pair, sk_slot(g, pair, tl), half, q, 0, 0, lane);
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
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
        // all four publish their rows, then one thread counts the half tile in.
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(part_bar);
        if (warp == 2 && lane == 0) {
          const bool okp = mbar_wait_bounded(part_bar, static_cast<uint32_t>(np) & 1u, g.err, 27);
          if (!okp) *abort_flag = 1;
          const bool last = okp && atomicAdd(g.counters + 2 * sg.tile + half, 1) == p_hi - p_lo;
          if (last) g.counters[2 * sg.tile + half] = 0;  // every contributor has counted: ready for the next launch
          *split_flag = last;
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
        for (int c = 0; c < 8; ++c) {
          float v[32];
          if (whole) {
            uint32_t r[32];
            tmem_ld_x32(t_row + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          } else if (p_hi - p_lo == 1) {
            // Two contributors: this CTA's own accumulator plus the other's
            // partial (a + b == b + a, so the sum does not depend on which
            // contributor came last), one partial read instead of two.
            const int other = pair == p_lo ? p_hi : p_lo;
            const float4* src = reinterpret_cast<const float4*>(g.partial) +
                                partial_index(other, sk_slot(g, other, tl), half, q, c, 0, lane);
            float4 pv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pv[j] = __ldcg(src + j * 32);
            uint32_t r[32];
            tmem_ld_x32(t_row + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              v[4 * j] = __uint_as_float(r[4 * j]) + pv[j].x;
              v[4 * j + 1] = __uint_as_float(r[4 * j + 1]) + pv[j].y;
              v[4 * j + 2] = __uint_as_float(r[4 * j + 2]) + pv[j].z;
              v[4 * j + 3] = __uint_as_float(r[4 * j + 3]) + pv[j].w;
            }
          } else {
            // Three or more: every partial, in pair order; the next
            // contributor's loads are in flight while the current one is added.
            auto fetch = [&](int p, float4 (&dst)[8]) {
              const float4* src =
                  reinterpret_cast<const float4*>(g.partial) + partial_index(p, sk_slot(g, p, tl), half, q, c, 0, lane);
#pragma unroll
              for (int j = 0; j < 8; ++j) dst[j] = __ldcg(src + j * 32);
            };
            float4 cur[8], nxt[8];
            fetch(p_lo, cur);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0f;
            for (int p = p_lo; p <= p_hi; ++p) {
              if (p < p_hi) fetch(p + 1, nxt);
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
      if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty(buf), 0));
      ++i;
    }
    if (lane == 0) bulk_wait<0>();
  }

  // The next kernel may now be launched (it waits for this one to finish
  // before it reads anything); signalled at the end, not the start, so its
  // waiting CTAs do not sit on the SMs while this kernel still runs (measured:
  // the block at 2048 tokens 1.3% faster than without the overlap, 2.8% slower
  // with the signal at the start).
  griddep_launch_dependents();
  __syncwarp();  // the single-thread roles rejoin their warps before the CTA barrier
  __syncthreads();
  // After an abort, loads issued by either CTA may still be landing and cannot
  // all be observed from here: pause before the pair may exit.
  if (tid == 0 && *abort_flag) spin_ns(kAbortPauseNs);
  tcgen05_fence_before();
  cluster_sync();  // no remote arrival or load targets a CTA that has left
  if (warp == 1) {
    tcgen05_fence_after();
    tmem_dealloc_pair(tmem, S::kTmemCols);
  }
}

bool bf16_map2(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
               uint32_t box_outer, CUtensorMapSwizzle swz) {
  const uint64_t dims[2] = {inner, outer}, strides[1] = {inner * 2};
  const uint32_t box[2] = {box_inner, box_outer};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, swz);
}

// How a GEMM is spread over the CTA pairs.
struct GemmPlan {
  int64_t tiles_m, tiles_n, k_chunks, tiles;
  int pairs, dp_waves;
  int64_t sk_chunks;
  bool partials;  // some stream-K tile is cut between pairs (workspace needed)
};

GemmPlan gemm_plan(int64_t M, int64_t N, int64_t K, int num_sms) {
  GemmPlan pl;
  pl.tiles_m = (M + kTileM - 1) / kTileM;
  pl.tiles_n = (N + kTileN - 1) / kTileN;
  pl.k_chunks = (K + kGBK - 1) / kGBK;
  pl.tiles = pl.tiles_m * pl.tiles_n;
  const int64_t total = pl.tiles * pl.k_chunks;
  int64_t pairs = (num_sms > 1 ? num_sms : 148) / 2;
  const int64_t by_work = total / kMinChunksPerPair;
  if (pairs > by_work) pairs = by_work > 0 ? by_work : 1;
  pl.pairs = static_cast<int>(pairs);
  // Whole tiles round-robin. A last wave that would leave most pairs idle is
  // replaced by cutting the final one to two tiles a pair along K (stream-K).
  // The cut tiles cost up to about 3/4 of a wave (fp32 partials written, read
  // back and summed at L2 latency), so K is cut only where that saves more:
  // measured on B200, out_proj at 2048 tokens (80 tiles on 74 pairs) gains,
  // in_proj at 2048 tokens (6.5 waves) loses 7%.
  const int64_t whole_waves = (pl.tiles + pairs - 1) / pairs;
  const bool cut =
      static_cast<double>(pl.tiles) / static_cast<double>(pairs) + 0.75 <= static_cast<double>(whole_waves);
  pl.dp_waves = static_cast<int>(cut ? (pl.tiles >= pairs ? pl.tiles / pairs - 1 : 0) : whole_waves);
  const int64_t dp_all = static_cast<int64_t>(pl.dp_waves) * pairs;
  const int64_t dp_tiles = dp_all < pl.tiles ? dp_all : pl.tiles;
  pl.sk_chunks = (pl.tiles - dp_tiles) * pl.k_chunks;
  pl.partials = false;
  for (int64_t p = 1; p < pairs; ++p)
    if ((p * pl.sk_chunks / pairs) % pl.k_chunks != 0) pl.partials = true;
  return pl;
}

size_t partial_bytes(const GemmPlan& pl) { return static_cast<size_t>(pl.pairs) * 4 * kHalfM * kTileN * 4; }
// The counters lead the workspace (so every GEMM finds its own at offset 0),
// the partials follow on a 512-byte boundary.
size_t counter_bytes(const GemmPlan& pl) { return (static_cast<size_t>(pl.tiles) * 2 * sizeof(int) + 511) / 512 * 512; }

cudaError_t launch_gemm(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* ws,
                        size_t ws_bytes, int num_sms, int* err, bool pdl, bool counters_zeroed, cudaStream_t st) {
  using S = GemmSmem;
  const GemmPlan pl = gemm_plan(M, N, K, num_sms);
  if (pl.tiles >= (int64_t(1) << 30)) return cudaErrorInvalidConfiguration;
  CUtensorMap ma, mb, mc;
  if (!bf16_map2(&ma, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), kGBK, kHalfM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mb, B, static_cast<uint64_t>(K), static_cast<uint64_t>(N), kGBK, kHalfN,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bf16_map2(&mc, C, static_cast<uint64_t>(N), static_cast<uint64_t>(M), 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  GemmArgs g;
  g.tiles_m = static_cast<int>(pl.tiles_m);
  g.tiles_n = static_cast<int>(pl.tiles_n);
  g.k_chunks = static_cast<int>(pl.k_chunks);
  g.group_m = static_cast<int>(pl.tiles_m < 16 ? pl.tiles_m : 16);
  g.pairs = pl.pairs;
  g.dp_waves = pl.dp_waves;
  g.sk_chunks = pl.sk_chunks;
  g.partial = nullptr;
  g.counters = nullptr;
  g.err = err;
  if (pl.partials) {
    if (!ws || ws_bytes < gemm_workspace_bytes(M, N, K, num_sms)) return cudaErrorInvalidValue;
    g.counters = static_cast<int*>(ws);
    g.partial = reinterpret_cast<float*>(static_cast<char*>(ws) + counter_bytes(pl));
    if (!counters_zeroed) {
      cudaError_t e = cudaMemsetAsync(g.counters, 0, counter_bytes(pl), st);
      if (e != cudaSuccess) return e;
    }
  }
  const int smem = S::kTotal + 1024;
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pl.pairs), 1, 1);
  cfg.blockDim = dim3(kGThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, gemm_bf16_tn_kernel, ma, mb, mc, g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  const GemmPlan pl = gemm_plan(M, N, K, num_sms);
  if (!pl.partials) return 0;
  return counter_bytes(pl) + partial_bytes(pl);
}

size_t gemm_counter_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  const GemmPlan pl = gemm_plan(M, N, K, num_sms);
  return pl.partials ? counter_bytes(pl) : 0;
}

cudaError_t gemm_bf16_tn(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* ws,
                         size_t ws_bytes, int num_sms, int* err, cudaStream_t st, bool pdl, bool counters_zeroed) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0 || N % 8 != 0) return cudaErrorInvalidValue;
  if (num_sms <= 1) num_sms = 148;
  return launch_gemm(A, B, C, M, N, K, ws, ws_bytes, num_sms, err, pdl, counters_zeroed, st);
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
