// ssd.cu -- the output of the Mamba-2 (SSD) chunk scan for sm_100a: "What is
// the Mamba model?" (velog, Texnee), "chunkscan" section. For batch b, chunk
// c, head h (group g) and position l of the chunk:
//
//   out[l] = sum_{s <= l} cb[l, s] exp(dA[l] - dA[s]) dt[s] x[s]     (intra-chunk)
//          + exp(dA[l]) C[l] . prev_states                          (carried state)
//          + D[h] x[l]                                              (skip)
//
// Both sums are dense contractions and run on the tensor cores, each into its
// own TMEM accumulator, so that the carried-state term needs no rescaled copy
// of C and starts as soon as its operands land. One CTA per (b, c, h) (two
// per chunk of 256, one per two chunks of 64): eight math warps (scores and
// epilogue) and a control warp, whose first thread issues the TMA loads and
// every MMA and waits on their barriers, so that the math warps wait only
// for their own data; ~75 KB of shared memory at chunk 128 lets three CTAs
// share an SM:
//  1. TMA brings, 128-byte swizzled, the cb tile [l][s] (128 columns, two
//     atoms) and the x tile [s][p] on one mbarrier, and the first 64-column
//     atom of the C tile [l][n] and of the prev_states tile [p][n] on a
//     second, while threads stage dA and dt;
//  2. as soon as that state atom is in, one thread issues its four tcgen05
//     MMAs C x prev_states^T into accumulator 1; their commit frees the
//     buffer, which takes the second atom (state dim 128) while the scores
//     are formed;
//  3. meanwhile thread s < 128 forms F[s] = exp(dA[s1] - dA[s]) dt[s], s1 the
//     last column of s's 8-column group (s1 = s | 7), and thread t turns the
//     64-column atom t / 128 of row l = t mod 128 of the cb tile, in place,
//     into the scores cb[l, s] exp(dA[l] - dA[s]) dt[s] for s <= l, zero above:
//     as cb exp(dA[l] - dA[s1]) F[s], one exponential per row and group. A
//     group wholly at or below the diagonal (s1 <= l) has both exponents <= 0
//     when dA_cumsum does not increase along the chunk (dt >= 0, A <= 0), so
//     no factor exceeds 1 however strong the decay, and a factor underflows
//     to 0 only where the exact product does. The group that holds the
//     diagonal has a row factor of at most exp(dA[s0] - dA[s1]) (s0 its first
//     column): below 80 nats it takes the same form, beyond that (where the
//     row factor could overflow) one exponential per element. The choice is
//     made per warp (over its 32 rows), so no branch diverges.
//     The TMA layout is already the MMA's K-major operand;
//  4. once the math warps have arrived at a named barrier, the control
//     thread issues eight MMAs scores x x (x as an MN-major B operand) into
//     accumulator 0. The second half of a 256-chunk has 256 score columns: it
//     runs steps 3-4 twice, on columns 0..127 then 128..255, the buffers
//     refilled once the first pass's MMAs have read them. Then the last state
//     atom's MMAs, and one commit for all;
//  5. warps w and w + 4 read lanes 32 (w mod 4) .. of columns 32 (w / 4) .. of
//     both accumulators, form acc0 + exp(dA[l]) acc1 + D x, and the bf16 tile
//     leaves by TMA store from the (now free) cb buffer.
// Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <initializer_list>

#include "sm100_ptx.cuh"
#include "ssm.h"
#include "ssm_internal.h"
#include "ssm_math.cuh"
#include "tma_map.cuh"

namespace ssm {
namespace {

constexpr int kCs = 128;  // rows of a CTA's tile: MMA M and the K of the intra-chunk term
constexpr int kHd = 64;   // head dim: MMA N
// Template parameters: the chunk length CS (64 or 128; a CTA's 128 rows hold
// 128 / CS consecutive chunks) and the state dim DS (64 or 128: the K of the
// carried-state term).
constexpr int kSsdMath = 256;                  // warps 0-7: scores and epilogue (a thread per row and atom)
constexpr int kSsdThreads = kSsdMath + 32;     // warp 8: TMA loads, TMEM, and every MMA issue and wait
constexpr int kCtlWarp = kSsdMath / 32;
constexpr int kBarScores = 1;                  // named barrier: the math warps' scores are in (arrive) -> MMAs (sync)
constexpr int kBarMath = 2;                    // named barrier among the math warps only
// Load order: 1 = cb and x first (the score math starts sooner; the
// carried-state MMAs go last), 0 = C and prev_states first (their MMAs are
// issued on arrival). Measured on B200 at b = 8, L = 4096, 80 heads: 364 us
// against 381 us.
#ifndef SSM_SSD_SCORES_FIRST
#define SSM_SSD_SCORES_FIRST 1
#endif
constexpr bool kScoresFirst = SSM_SSD_SCORES_FIRST;  // accumulator 0 (intra-chunk) at column 0, 1 (carried state) at 64

template <int CS, int DS>
struct SsdSmem {
  static_assert(DS == 64 || DS == 128, "state dim 64 or 128");
  static_assert(CS == 64 || CS == 128 || CS == 256, "chunk 64, 128 or 256");
  static constexpr int kNC = CS < kCs ? kCs / CS : 1;  // chunks per CTA (stacked on the tile diagonal)
  static constexpr int kHalves = CS > kCs ? CS / kCs : 1;  // CTAs per chunk (128-row halves)
  static constexpr int kCols = CS > kCs ? CS : kCs;    // most score columns = rows of x = K of the intra term
  static constexpr int kKS = kCs;                      // score columns (and rows of x) staged per pass
  static constexpr int kNA = DS / 64;                  // 64-column atoms across the state dim
  // State dim 128: the carried-state operands are loaded one 64-column atom
  // at a time into one buffer (the first atom's MMAs free it for the
  // second). With the 128-column score passes below, that brings a chunk-128
  // or chunk-256 CTA to ~75 KB (three CTAs per SM) and a chunk-64 CTA to
  // ~84 KB (two).
  static constexpr bool kReload = kNA == 2;
  static constexpr int kSA = kReload ? 1 : kNA;        // state atoms resident at once
  static constexpr int kAtomRows128 = kCs * 128;       // one 64-column atom of a 128-row tile
  static constexpr int kAtomRows64 = kHd * 128;        // one 64-column atom of a 64-row tile
  static constexpr int kCb = 0;                        // cb -> scores [128][kKS] (A of MMA 1) -> out tile
  static constexpr int kC = kCb + (kKS / 64) * kAtomRows128;  // C [128][DS] (A of MMA 2)
  static constexpr int kX = kC + kSA * kAtomRows128;   // x [kKS][p] (B of MMA 1, MN-major)
  static constexpr int kPrev = kX + kKS * 128;         // prev_states [chunk][p][n] (B of MMA 2, K-major)
  static constexpr int kDA = kPrev + kNC * kSA * kAtomRows64;
  static constexpr int kDt = kDA + kCols * 4;
  static constexpr int kF = kDt + kCols * 4;
  static constexpr int kBar = kF + kCols * 4;          // full_state, full_scores, done, state_free, pass_free
  static constexpr int kTmemSlot = kBar + 40;
  static constexpr int kTotal = kTmemSlot + 16;
  // C and prev_states bytes of one load round (all atoms, or one when reloading)
  static constexpr uint32_t kTxState = static_cast<uint32_t>(kSA * (kAtomRows128 + kNC * kAtomRows64));
  // cb and x of one score pass: stacked chunks load their [CS][CS] diagonal
  // blocks, otherwise 128 rows x 128 columns; x has 128 rows.
  static constexpr uint32_t kTxScores =
      static_cast<uint32_t>((kNC > 1 ? kNC * CS * CS * 2 : kCs * kKS * 2) + kKS * 128);
  static constexpr uint32_t kTmemCols = kNC == 1 ? 128u : 256u;  // intra + one carried-state term per chunk
  static_assert(kC % 1024 == 0 && kX % 1024 == 0 && kPrev % 1024 == 0, "swizzled tiles need 1 KB");
};

// bf16 x bf16 -> fp32, M = 128, N = 64, A K-major, B K-major or MN-major.
__host__ __device__ constexpr uint32_t ssd_idesc(bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(kHd >> 3) << 17) | (static_cast<uint32_t>(kCs >> 4) << 24);
}

struct SsdArgs {
  const float* dt;         // [b][H][nc][cs]
  const float* dA;         // [b][H][nc][cs]
  const float* D;          // [H] or null
  int64_t nheads, nchunks, ngroups;
  int* err;
};

// Byte offset of 16-byte chunk j (0..7) of row r in a 128-byte swizzled atom.
__device__ __forceinline__ int sw128(int r, int j) { return r * 128 + ((j ^ (r & 7)) << 4); }

__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 p;
    *reinterpret_cast<uint32_t*>(&p) = w[i];
    const float2 q = __bfloat1622float2(p);
    f[2 * i] = q.x, f[2 * i + 1] = q.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int CS, int DS>
__global__ void __launch_bounds__(kSsdThreads) ssd_chunk_scan_kernel(
    const __grid_constant__ CUtensorMap map_cb, const __grid_constant__ CUtensorMap map_x,
    const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_prev,
    const __grid_constant__ CUtensorMap map_out, const SsdArgs a) {
  using S = SsdSmem<CS, DS>;
  constexpr int NC = S::kNC;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
  const int l = tid & (kCs - 1), at = tid >> 7;  // this thread's tile row and first 64-column atom
  const int h = blockIdx.x, b = blockIdx.z;
  // This CTA: chunk c (the first of NC stacked ones), rows r0 .. r0 + 127 of
  // it (r0 > 0 only for the second half of a 256-chunk), ks score columns.
  const int c = S::kHalves > 1 ? static_cast<int>(blockIdx.y) / S::kHalves : static_cast<int>(blockIdx.y) * NC;
  const int r0 = S::kHalves > 1 ? (static_cast<int>(blockIdx.y) % S::kHalves) * kCs : 0;
  const int ks = r0 + kCs;
  const int64_t t_chunk = static_cast<int64_t>(c) * CS;  // first token of chunk c
  const int g = static_cast<int>(h / (a.nheads / a.ngroups));
  const uint32_t full_state = sb + S::kBar, full_scores = sb + S::kBar + 8, done = sb + S::kBar + 16;
  const uint32_t state_free = sb + S::kBar + 24, pass_free = sb + S::kBar + 32;
  const int np = ks / kCs;  // score passes: 2 for the second half of a 256-chunk, else 1
  const int64_t zp0 = (static_cast<int64_t>(b) * a.nchunks + c) * a.nheads + h;
  // State atoms [t0, t0 + kSA) of C and prev_states into the state buffers.
  auto load_state = [&](int t0) {
#pragma unroll
    for (int i = 0; i < S::kSA; ++i) {
      const int t = t0 + i;
      tma_load_4d(sb + S::kC + i * S::kAtomRows128, &map_c, 64 * t, g, static_cast<int>(t_chunk + r0), b, full_state);
#pragma unroll
      for (int k = 0; k < NC; ++k)
        tma_load_3d(sb + S::kPrev + (k * S::kSA + i) * S::kAtomRows64, &map_prev, 64 * t, 0,
                    static_cast<int>(zp0 + k * a.nheads), full_state);
    }
  };
  // A second stacked chunk past the last one (odd chunk count) reads zeros
  // or a neighbouring sequence's chunk; its rows lie past L and are never stored.
  const int64_t zc0 = (static_cast<int64_t>(b) * a.nchunks + c) * a.ngroups + g;
  // Score pass p: cb columns 128 p .. 128 p + 127 of this CTA's 128 rows and
  // x rows 128 p .. of the chunk into the score buffers.
  auto load_scores = [&](int p) {
    if constexpr (NC == 1) {
#pragma unroll
      for (int t = 0; t < S::kKS / 64; ++t)  // rows r0 .. r0 + 127, columns 128 p + 64 t ..
        tma_load_3d(sb + S::kCb + t * S::kAtomRows128, &map_cb, kCs * p + 64 * t, r0, static_cast<int>(zc0),
                    full_scores);
    } else {
      // chunk k's [CS][CS] block on the diagonal: atom k, rows CS k ..
#pragma unroll
      for (int k = 0; k < NC; ++k)
        tma_load_3d(sb + S::kCb + k * S::kAtomRows128 + k * CS * 128, &map_cb, 0, 0,
                    static_cast<int>(zc0 + k * a.ngroups), full_scores);
    }
    tma_load_4d(sb + S::kX, &map_x, 0, h, static_cast<int>(t_chunk + kCs * p), b, full_scores);
  };
  const bool ctl = tid == kSsdMath;  // the control thread: lane 0 of warp 8
  if (ctl) {
    mbar_init(full_state, 1);
    mbar_init(full_scores, 1);
    mbar_init(done, 1);
    mbar_init(state_free, 1);
    mbar_init(pass_free, 1);
    mbar_fence_init();
    prefetch_tensormap(&map_cb);
    prefetch_tensormap(&map_x);
    prefetch_tensormap(&map_c);
    prefetch_tensormap(&map_prev);
    mbar_arrive_expect_tx(full_state, S::kTxState);
    mbar_arrive_expect_tx(full_scores, S::kTxScores);
    if (kScoresFirst) {
      load_scores(0);
      load_state(0);
    } else {
      load_state(0);
      load_scores(0);
    }
  }
  if (warp == kCtlWarp) {
    tmem_alloc(sb + S::kTmemSlot, S::kTmemCols);
    tmem_relinquish();
  }
  float* sdA = reinterpret_cast<float*>(smem + S::kDA);
  float* sdt = reinterpret_cast<float*>(smem + S::kDt);
  float* F = reinterpret_cast<float*>(smem + S::kF);
  {  // the score columns' dA and dt: positions 0 .. ks - 1 from chunk c on ([b][H][nc][CS], chunks adjacent)
    const int64_t row = ((static_cast<int64_t>(b) * a.nheads + h) * a.nchunks + c) * CS;
    for (int i = tid; i < ks; i += kSsdThreads) {
      const bool in = c + i / CS < a.nchunks;
      sdA[i] = in ? a.dA[row + i] : 0.0f;
      sdt[i] = in ? a.dt[row + i] : 0.0f;
    }
  }
  const float Dh = a.D ? a.D[h] : 0.0f;
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + S::kTmemSlot);
  // Accumulators: the intra-chunk term at column 0, the carried-state term of
  // stacked chunk k at 64 (k + 1) (C x prev_states(k)^T over all 128 rows;
  // rows of chunk k read it).
  const uint32_t acc_intra = tmem;
  // MMAs of the resident state atoms, the first of which is state atom t0
  // (a K of 16 per MMA, four per 64-column atom).
  auto state_mmas = [&](int t0) {
#pragma unroll
    for (int k = 0; k < NC; ++k)
#pragma unroll
      for (int kk = 0; kk < 4 * S::kSA; ++kk)
        umma_f16_ss(tmem + kHd * (k + 1),
                    umma_desc_k_sw128(sb + S::kC + (kk >> 2) * S::kAtomRows128 + (kk & 3) * 32),
                    umma_desc_k_sw128(sb + S::kPrev + (k * S::kSA + (kk >> 2)) * S::kAtomRows64 + (kk & 3) * 32),
                    ssd_idesc(false), t0 > 0 || kk > 0);
  };
  if (warp == kCtlWarp) {
    // The control warp: the MMAs and the waits they need, so that the math
    // warps wait only for their data.
    if (ctl) {
      // 2. Carried-state term, as soon as its operands are in: C[l][n] x prev_states[p][n]^T.
      //    Reloading: the first atom here, then the buffer is refilled with the
      //    second while the scores are formed.
      if (S::kReload || !kScoresFirst) {
        mbar_wait_bounded(full_state, 0u, a.err, 7);
        tcgen05_fence_after();
        state_mmas(0);
        if constexpr (S::kReload) {
          umma_commit(state_free);
          mbar_wait_bounded(state_free, 0u, a.err, 10);  // the MMAs have read the buffer
          mbar_arrive_expect_tx(full_state, S::kTxState);
          load_state(1);
        }
      }
    }
    // 4. Intra-chunk term of each pass: scores[l][s] x x[s][p], s in steps of
    //    16 rows of x, once the math warps have formed the pass's scores.
    //    Before a second pass the buffers are refilled once these MMAs have
    //    read them. (The warp reconverges before each barrier: bar.sync is
    //    executed by whole warps.)
    for (int pass = 0; pass < np; ++pass) {
      __syncwarp();
      named_bar_sync(kBarScores, kSsdThreads);
      if (ctl) {
        tcgen05_fence_after();
#pragma unroll
        for (int kk = 0; kk < S::kKS / 16; ++kk)
          umma_f16_ss(acc_intra, umma_desc_k_sw128(sb + S::kCb + (kk >> 2) * S::kAtomRows128 + (kk & 3) * 32),
                      umma_desc_k_sw128(sb + S::kX + kk * 16 * 128), ssd_idesc(true), pass > 0 || kk > 0);
        if (pass + 1 < np) {
          umma_commit(pass_free);
          mbar_wait_bounded(pass_free, static_cast<uint32_t>(pass) & 1u, a.err, 11);
          mbar_arrive_expect_tx(full_scores, S::kTxScores);
          load_scores(pass + 1);
        }
      }
    }
    // The carried-state term (its last atom) and one commit for everything.
    if (ctl) {
      if constexpr (S::kReload) {  // the second state atom
        mbar_wait_bounded(full_state, 1u, a.err, 7);
        tcgen05_fence_after();
        state_mmas(1);
      } else if (kScoresFirst) {  // carried-state term last: its operands were loaded second
        mbar_wait_bounded(full_state, 0u, a.err, 7);
        tcgen05_fence_after();
        state_mmas(0);
      }
      umma_commit(done);
    }
    __syncwarp();
  } else {
    for (int i = tid; i < ks; i += kSsdMath) F[i] = ex2_approx((sdA[i | 7] - sdA[i]) * kLog2e) * sdt[i];
    const int lg = r0 + l;  // this thread's row within its chunk pair / chunk
    const float dAl = sdA[lg];
    mbar_wait_bounded(full_scores, 0u, a.err, 8);
    named_bar_sync(kBarMath, kSsdMath);  // F complete

    // 3. Row l of the cb tile -> scores (in place), one pass of 128 columns at a
    //    time (two passes only for the second half of a 256-chunk), this
    //    thread's 64-column atom `at` of each. A warp's 32 rows lie in one chunk, starting at column
    //    warp_min_s. Groups are classified against the warp's whole row span,
    //    so every branch below is warp-uniform: groups wholly at or below all 32
    //    rows take the two-factor product with no masking; the four groups the
    //    span straddles mask per element, in the two-factor form unless the
    //    diagonal group of some row of the warp decays by 80 nats or more
    //    across its 8 columns (then its row factor could overflow, and each
    //    decay is formed on its own).
    const int warp_min_l = r0 + 32 * (warp & 3), warp_max_l = warp_min_l + 31;
    const int warp_min_s = CS < kCs ? (32 * (warp & 3)) & ~(CS - 1) : 0;
    const int sd = lg & ~7;
    const bool strong = __any_sync(0xffffffffu, sdA[sd] - sdA[sd + 7] >= 80.0f);
    for (int pass = 0; pass < np; ++pass) {
      if (pass > 0) mbar_wait_bounded(full_scores, static_cast<uint32_t>(pass) & 1u, a.err, 8);
      // This thread's 64-column atom of the pass: columns 128 pass + 64 at ..
      {
        const int aa = 2 * pass + at;  // atom index over the chunk's columns
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int s0 = 64 * aa + 8 * j;
          uint4* p = reinterpret_cast<uint4*>(smem + S::kCb + at * S::kAtomRows128 + sw128(l, j));
          if (s0 > warp_max_l || s0 < warp_min_s) {  // above the diagonal or outside the chunk, every row
            *p = make_uint4(0u, 0u, 0u, 0u);
            continue;
          }
          float f[8];
          unpack8(*p, f);
          if (s0 + 7 <= warp_min_l) {  // wholly at or below the diagonal for every row: row factor x column factor
            const float e = ex2_approx((dAl - sdA[s0 + 7]) * kLog2e);
#pragma unroll
            for (int q = 0; q < 8; ++q) f[q] *= e * F[s0 + q];
          } else if (!strong) {  // straddled by the warp's rows: masked two-factor form
            const float e = s0 <= lg ? ex2_approx((dAl - sdA[s0 + 7]) * kLog2e) : 0.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) f[q] = s0 + q <= lg ? f[q] * e * F[s0 + q] : 0.0f;
          } else {  // masked, each decay on its own
#pragma unroll
            for (int q = 0; q < 8; ++q)
              f[q] = s0 + q <= lg ? f[q] * ex2_approx((dAl - sdA[s0 + q]) * kLog2e) * sdt[s0 + q] : 0.0f;
          }
          *p = pack8(f);
        }
      }
      fence_proxy_async_smem();  // generic-proxy writes become visible to the tensor core
      tcgen05_fence_before();
      named_bar_arrive(kBarScores, kSsdThreads);  // the pass's scores are in: the control warp issues its MMAs
    }
    mbar_wait_bounded(done, 0u, a.err, 9);
    tcgen05_fence_after();

    // 5. Lanes 32 (w mod 4) .., columns 32 (w / 4) ..: acc0 + exp(dA[l]) acc1 + D x, bf16,
    //    into the out tile (the cb buffer, free now), then out by TMA.
    {
      const int q4 = warp & 3, col0 = 32 * (warp >> 2);
      const int row = 32 * q4 + (tid & 31);
      const float el = ex2_approx(sdA[r0 + row] * kLog2e);
      const uint32_t acc_state = tmem + kHd * (1 + (CS < kCs ? (32 * q4) / CS : 0));  // this warp's chunk
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        uint32_t r0v[16], r1v[16];
        const uint32_t lane_col = (static_cast<uint32_t>(32 * q4) << 16) + col0 + 16 * jj;
        tmem_ld_x16(acc_intra + lane_col, r0v);
        tmem_ld_x16(acc_state + lane_col, r1v);
        tmem_ld_wait();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int j = (col0 + 16 * jj) / 8 + half;  // 16-byte chunk of the row: p = 8 j .. 8 j + 7
          float xv[8], o[8];
          unpack8(*reinterpret_cast<const uint4*>(smem + S::kX + sw128(row, j)), xv);  // the last pass's x rows
#pragma unroll
          for (int q = 0; q < 8; ++q)
            o[q] = fmaf(Dh, xv[q], fmaf(el, __uint_as_float(r1v[8 * half + q]), __uint_as_float(r0v[8 * half + q])));
          *reinterpret_cast<uint4*>(smem + S::kCb + sw128(row, j)) = pack8(o);
        }
      }
    }
  }  // math warps
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
    tma_store_4d(&map_out, sb + S::kCb, 0, h, static_cast<int>(t_chunk + r0), b);
    bulk_commit();
    bulk_wait_read<0>();  // the tile stays in shared memory until the store has read it
  }
  tcgen05_fence_before();
  __syncthreads();
  if (warp == kCtlWarp) {
    tcgen05_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

bool bf16_map(CUtensorMap* m, int rank, const void* base, std::initializer_list<uint64_t> dims,
              std::initializer_list<uint64_t> strides, std::initializer_list<uint32_t> box) {
  uint64_t d[5], s[4];
  uint32_t bx[5];
  int i = 0;
  for (uint64_t v : dims) d[i++] = v;
  i = 0;
  for (uint64_t v : strides) s[i++] = v;
  i = 0;
  for (uint32_t v : box) bx[i++] = v;
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, d, s, bx, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int CS, int DS>
cudaError_t launch_ssd(int64_t H, int64_t nc, int64_t b, const CUtensorMap& mcb, const CUtensorMap& mx,
                       const CUtensorMap& mc, const CUtensorMap& mp, const CUtensorMap& mo, const SsdArgs& a,
                       cudaStream_t st) {
  using S = SsdSmem<CS, DS>;
  const int smem = S::kTotal + 1024;
  auto kern = ssd_chunk_scan_kernel<CS, DS>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const dim3 grid(static_cast<unsigned>(H), static_cast<unsigned>((nc + S::kNC - 1) / S::kNC * S::kHalves),
                  static_cast<unsigned>(b));
  kern<<<grid, kSsdThreads, smem, st>>>(mcb, mx, mc, mp, mo, a);
  return cudaGetLastError();
}

}  // namespace
}  // namespace ssm

extern "C" ssm_status ssm_ssd_chunk_scan(const ssm_ssd_dims* dims, const void* cb, const void* x, const float* dt,
                                         const float* dA_cumsum, const void* C, const void* prev_states,
                                         const float* D, void* out, void* stream) {
  using ssm::fail;
  if (!dims) return fail(SSM_ERR_INVALID_ARG, "dims is NULL");
  const int64_t b = dims->batch, L = dims->seqlen, H = dims->nheads, P = dims->headdim, G = dims->ngroups;
  const int64_t N = dims->dstate, cs = dims->chunk_size;
  if ((cs != 64 && cs != 128 && cs != 256) || P != ssm::kHd || (N != 64 && N != 128))
    return fail(SSM_ERR_UNSUPPORTED,
                "chunk_size %lld, headdim %lld, dstate %lld: the built shapes are chunk 64, 128 or 256, headdim 64, "
                "dstate 64 or 128",
                (long long)cs, (long long)P, (long long)N);
  if (b <= 0 || b > 65535 || H <= 0 || H > 0x7fffffff || G <= 0 || H % G != 0)
    return fail(SSM_ERR_INVALID_ARG, "need 0 < batch <= 65535, nheads > 0 and nheads a multiple of ngroups");
  if (L <= 0 || L % cs != 0 || L / cs > 32767)
    return fail(SSM_ERR_INVALID_ARG, "seqlen must be a positive multiple of chunk_size, at most 32767 chunks");
  const void* ptrs[8] = {cb, x, dt, dA_cumsum, C, prev_states, out, D};
  const char* names[8] = {"cb", "x", "dt", "dA_cumsum", "C", "prev_states", "out", "D"};
  for (int i = 0; i < 8; ++i) {
    if (!ptrs[i] && i < 7) return fail(SSM_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (ptrs[i] && !ssm::aligned(ptrs[i], 16)) return fail(SSM_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (out == x || out == cb || out == C || out == prev_states)
    return fail(SSM_ERR_INVALID_ARG, "out must not alias an input");
  const int64_t nc = L / cs;
  CUtensorMap mcb, mx, mc, mp, mo;
  const uint64_t e2 = 2;
  const bool ok =
      ssm::bf16_map(&mcb, 3, cb, {uint64_t(cs), uint64_t(cs), uint64_t(b * nc * G)}, {cs * e2, cs * cs * e2},
                    {64, uint32_t(cs < 128 ? cs : 128), 1}) &&
      ssm::bf16_map(&mx, 4, x, {uint64_t(P), uint64_t(H), uint64_t(L), uint64_t(b)},
                    {P * e2, H * P * e2, L * H * P * e2}, {64, 1, 128, 1}) &&
      ssm::bf16_map(&mc, 4, C, {uint64_t(N), uint64_t(G), uint64_t(L), uint64_t(b)},
                    {N * e2, G * N * e2, L * G * N * e2}, {64, 1, 128, 1}) &&
      ssm::bf16_map(&mp, 3, prev_states, {uint64_t(N), uint64_t(P), uint64_t(b * nc * H)}, {N * e2, P * N * e2},
                    {64, 64, 1}) &&
      ssm::bf16_map(&mo, 4, out, {uint64_t(P), uint64_t(H), uint64_t(L), uint64_t(b)},
                    {P * e2, H * P * e2, L * H * P * e2}, {64, 1, 128, 1});
  if (!ok) return fail(SSM_ERR_CUDA, "tensor map encoding failed");
  ssm::SsdArgs a{dt, dA_cumsum, D, H, nc, G, ssm::device_error_ptr()};
  if (!a.err) return fail(SSM_ERR_CUDA, "device error word: %s", cudaGetErrorString(cudaGetLastError()));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (cs == 256)
    err = N == 128 ? ssm::launch_ssd<256, 128>(H, nc, b, mcb, mx, mc, mp, mo, a, st)
                   : ssm::launch_ssd<256, 64>(H, nc, b, mcb, mx, mc, mp, mo, a, st);
  else if (cs == 128)
    err = N == 128 ? ssm::launch_ssd<128, 128>(H, nc, b, mcb, mx, mc, mp, mo, a, st)
                   : ssm::launch_ssd<128, 64>(H, nc, b, mcb, mx, mc, mp, mo, a, st);
  else
    err = N == 128 ? ssm::launch_ssd<64, 128>(H, nc, b, mcb, mx, mc, mp, mo, a, st)
                   : ssm::launch_ssd<64, 64>(H, nc, b, mcb, mx, mc, mp, mo, a, st);
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "chunk-scan launch: %s", cudaGetErrorString(err));
  return fail(SSM_OK, "");
}
