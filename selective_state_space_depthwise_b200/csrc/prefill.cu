// prefill.cu -- full-sequence selective scan for sm_100a.
//
// One fused kernel computes, for a tile of NCH channels of one sequence and
// the whole length L, the block core of "Axon-SSM: selective state space
// model" ("Algorithm" diagram): causal depthwise conv (K=4) + SiLU, dt =
// clip(softplus(dt_raw*w_dt + dt_bias)), dA = exp(dt*A) with A = -exp(A_log),
// the scan h = dA*h + dt*B*u (the _ssm_fma leaf of "JIT-compiled kernels"),
// y = C.h + D*u and the gate y*SiLU(z). dA, dB and h never reach HBM: the 16
// states of a channel live in registers for the whole walk over L.
//
// Pipeline. L is walked in stages of kTok tokens through a kStages-deep ring
// in shared memory filled by TMA tile loads: the x tile carries a 3-row halo
// for the conv (rows before token 0 come back zero-filled and are replaced by
// conv_cache_in when one is given), B and C (shared by all channels) come as
// [token][16] tiles, and warp 0 stages dt_raw one stage ahead. Thread 0
// re-arms a slot right after the CTA has finished with it; every wait on the
// ring's mbarriers is bounded.
//
// Work split. G threads share a channel and hold 16/G states each (G is
// chosen from b*E so that small batches still fill the GPU without splitting
// L). With G == 1 one thread does everything for its channel token by token.
// With G > 1 each stage runs three phases:
//  A. per-token work for a contiguous run of kTok/G tokens of the thread's
//     channel (conv with a sliding window of x, SiLU, dt), written to shared
//     memory as (dt, dt, dt*u, dt*u); D*u and SiLU(z) stay in registers;
//  B. every thread advances its states through all kTok tokens (packed f32x2
//     multiplies/FMAs, SFU exp2 for the decays) and writes the partial
//     readout C.h of each token -- a stream whose only carried dependency is
//     the state;
//  C. each thread sums the G partials of its phase-A tokens, applies the D
//     skip and the gate, and fills an output tile that leaves by TMA store.
//
// Kernels. 1: channel tiles (a thread holds all 16/G states of a channel for
// NCH channels per CTA). 2: state slices (a CTA is G warps over 32 channels;
// warp j holds state slice j of every channel, lane = channel). 3 (default):
// kernel 2 software-pipelined, phase A of stage s + 1 fused into phase B of
// stage s, two barriers per stage instead of three. 4 (default when the grid
// needs at most two CTAs per SM): kernel 3 built with the register budget of
// two CTAs per SM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "ssm_internal.h"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kTok = 32;    // tokens per pipeline stage (= lanes of the dt_raw stager)
// Phase-B tokens computed between partial-readout stores, per states-per-warp
// K (measured on B200: longer unrolled runs hide more latency until registers
// run out; 32 for K = 4, 16 for K = 8, 4 for K = 2).
template <int K>
constexpr int phase_b_chunk() {
  return K == 4 ? 32 : (K == 8 ? 16 : 4);
}
constexpr int kStages = 3;  // ring depth

struct Maps {
  CUtensorMap x, z, B, C, y;
};

constexpr int align128(int v) { return (v + 127) / 128 * 128; }

// Shared-memory layout (byte offsets from a 128-aligned base).
template <typename T, int NCH, int G>
struct Smem {
  static constexpr int kEs = static_cast<int>(sizeof(T));
  static constexpr int kXBytes = (kTok + 3) * NCH * kEs;  // TMA box {NCH, kTok + 3}
  static constexpr int kZBytes = kTok * NCH * kEs;        // TMA box {NCH, kTok}
  static constexpr int kBCBytes = kTok * 16 * 4;          // TMA box {16, kTok}
  static constexpr int kX = 0;
  static constexpr int kZ = align128(kX + kXBytes);
  static constexpr int kB = align128(kZ + kZBytes);
  static constexpr int kC = kB + kBCBytes;
  static constexpr int kSlot = kC + kBCBytes;
  // Phase-A outputs (G > 1): a row per channel, one pad entry after every
  // thread's run of kTok/G tokens so that the runs of a warp hit distinct banks.
  static constexpr int kRow = kTok + G;
  // Partial readouts (G > 1): [channel][state slice][token], rows padded by 4
  // floats and channels by a further 4 x G floats for bank spread.
  static constexpr int kPRow = kTok + 4;
  static constexpr int kPCh = G * kPRow + 4 * G;
  static constexpr int kDT = kStages * kSlot;                           // float4 (dt, dt, dt*u, dt*u)
  static constexpr int kP = kDT + (G > 1 ? NCH * kRow * 16 : 0);       // float partials
  static constexpr int kDr = kP + (G > 1 ? NCH * kPCh * 4 : 0);        // dt_raw, 2 stages
  static constexpr int kY = align128(kDr + 2 * kTok * 4);              // output tiles (G > 1)
  static constexpr int kYBytes = G > 1 ? align128(kTok * NCH * kEs) : 0;
  static constexpr int kBar = kY + 2 * kYBytes;
  static constexpr int kTotal = kBar + kStages * 8;
  static constexpr uint32_t kTxBytes = static_cast<uint32_t>(kXBytes + kZBytes + 2 * kBCBytes);
  static_assert((NCH * kEs) % 16 == 0, "TMA rows must be whole 16-byte chunks");
};

// Advance KP packed state pairs through one token; returns C.h over the pairs.
// dt2 = {dt, dt}, inj2 = {dt*u, dt*u}; B, C point at this thread's states.
template <int KP, int NPOLY = 0>
__device__ __forceinline__ float scan_token(uint64_t dt2, uint64_t inj2, const float* a2, float* h, const float* Bp,
                                            const float* Cp) {
  uint64_t acc = 0;
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    float b0, b1, c0, c1;
    if constexpr (KP >= 2) {
      const float4 bq = *reinterpret_cast<const float4*>(Bp + 4 * (q / 2));
      const float4 cq = *reinterpret_cast<const float4*>(Cp + 4 * (q / 2));
      b0 = (q & 1) ? bq.z : bq.x, b1 = (q & 1) ? bq.w : bq.y;
      c0 = (q & 1) ? cq.z : cq.x, c1 = (q & 1) ? cq.w : cq.y;
    } else {
      const float2 bq = *reinterpret_cast<const float2*>(Bp);
      const float2 cq = *reinterpret_cast<const float2*>(Cp);
      b0 = bq.x, b1 = bq.y, c0 = cq.x, c1 = cq.y;
    }
    float x0, x1;
    upk2(fmul2(dt2, pk2(a2[2 * q], a2[2 * q + 1])), x0, x1);
    // the last NPOLY pairs take the FMA-pipe exp2, the others the SFU
    const uint64_t dA = q >= KP - NPOLY ? ex2_poly2(x0, x1) : pk2(ex2_approx(x0), ex2_approx(x1));
    const uint64_t hb = ffma2(dA, pk2(h[2 * q], h[2 * q + 1]), fmul2(inj2, pk2(b0, b1)));
    upk2(hb, h[2 * q], h[2 * q + 1]);
    acc = q == 0 ? fmul2(pk2(c0, c1), hb) : ffma2(pk2(c0, c1), hb, acc);
  }
  float lo, hi;
  upk2(acc, lo, hi);
  return lo + hi;
}

// Zero-order-hold variant (scalar): h = e^{dt A} h + (e^{dt A} - 1)/A * u * B.
template <int K>
__device__ __forceinline__ float scan_token_zoh(float dt, float u, const float* Av, float* h, const float* Bp,
                                                const float* Cp) {
  float acc = 0.0f;
#pragma unroll
  for (int q = 0; q < K; ++q) {
    const float xa = dt * Av[q];
    const float dA = ex2_approx(xa * kLog2e);
    h[q] = fmaf(dA, h[q], expm1_nonpos(xa, dA) / Av[q] * u * Bp[q]);
    acc = fmaf(Cp[q], h[q], acc);
  }
  return acc;
}

template <typename T, int G, int NCH, bool ZOH, int NPOLY>
__global__ void __launch_bounds__(NCH* G) prefill_kernel(const __grid_constant__ Maps maps, const KernelArgs a) {
  constexpr int NT = NCH * G;  // threads
  constexpr int K = 16 / G;    // states per thread
  constexpr int KP = K / 2;    // packed state pairs
  constexpr int TA = kTok / G;  // phase-A tokens per thread (G > 1)
  using S = Smem<T, NCH, G>;
  static_assert(kTok % G == 0 && NT % 32 == 0 && K >= 2, "bad shape");

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  const uint32_t sb = smem_u32(smem);
  const uint32_t full0 = sb + S::kBar;
  float* Dr = reinterpret_cast<float*>(smem + S::kDr);  // [2][kTok]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int64_t tiles = (a.E + NCH - 1) / NCH;
  const int seq = static_cast<int>(blockIdx.x / tiles);
  const int e0 = static_cast<int>(blockIdx.x % tiles) * NCH;
  const int64_t L = a.L;
  const int64_t n_stages = (L + kTok - 1) / kTok;
  const float* dtr = a.dt_raw + static_cast<int64_t>(seq) * a.s.dt_seq;

  auto issue_stage = [&](int64_t st_idx) {  // thread 0 only
    const int slot = static_cast<int>(st_idx % kStages);
    const uint32_t base = sb + slot * S::kSlot, bar = full0 + 8 * slot;
    const int t0 = static_cast<int>(st_idx * kTok);
    mbar_arrive_expect_tx(bar, S::kTxBytes);
    tma_load_3d(base + S::kX, &maps.x, e0, t0 - 3, seq, bar);
    tma_load_3d(base + S::kZ, &maps.z, e0, t0, seq, bar);
    tma_load_3d(base + S::kB, &maps.B, 0, t0, seq, bar);
    tma_load_3d(base + S::kC, &maps.C, 0, t0, seq, bar);
  };

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(full0 + 8 * i, 1);
    mbar_fence_init();
    prefetch_tensormap(&maps.x);
    prefetch_tensormap(&maps.z);
    prefetch_tensormap(&maps.B);
    prefetch_tensormap(&maps.C);
    for (int64_t i = 0; i < kStages && i < n_stages; ++i) issue_stage(i);
  }
  float d_next = 0.0f;  // warp 0 stages dt_raw one stage ahead
  if (tid < 32) {
    Dr[lane] = lane < L ? dtr[lane] : 0.0f;
    d_next = kTok + lane < L ? dtr[kTok + lane] : 0.0f;
  }
  __syncthreads();

  const int c = tid / G;  // channel within the tile
  const int j = tid % G;  // state slice; also the token this lane owns in a round
  const int e = e0 + c;
  const bool ch_ok = e < a.E;
  const int64_t ec = ch_ok ? e : a.E - 1;  // clamped index for parameter loads

  const float cw0 = a.conv_w[ec * 4 + 0], cw1 = a.conv_w[ec * 4 + 1];
  const float cw2 = a.conv_w[ec * 4 + 2], cw3 = a.conv_w[ec * 4 + 3];
  const float cb = a.conv_b[ec], wdt = a.w_dt[ec], dtb = a.dt_bias[ec], Dd = a.D[ec];
  const float lo = a.dt_min, hi = a.dt_max;
  float hx0 = 0.0f, hx1 = 0.0f, hx2 = 0.0f;  // conv history before token 0
  if (a.conv_cache_in) {
    const T* hist = static_cast<const T*>(a.conv_cache_in) + static_cast<int64_t>(seq) * 3 * a.E + ec;
    hx0 = IO<T>::to_f(hist[0]);
    hx1 = IO<T>::to_f(hist[a.E]);
    hx2 = IO<T>::to_f(hist[2 * a.E]);
  }
  float a2[K];  // A_n * log2(e): exp(dt*A_n) = 2^(dt*a2_n)
  float Av[K];  // A_n (ZOH only)
  float h[K];
#pragma unroll
  for (int q = 0; q < K; ++q) {
    const float A = -expf(a.A_log[ec * 16 + j * K + q]);
    Av[q] = A;
    a2[q] = A * kLog2e;
    h[q] = a.ssm_state_in ? a.ssm_state_in[(static_cast<int64_t>(seq) * a.E + ec) * 16 + j * K + q] : 0.0f;
  }
  (void)Av;

  for (int64_t s = 0; s < n_stages; ++s) {
    const int slot = static_cast<int>(s % kStages);
    const unsigned char* st = smem + slot * S::kSlot;
    mbar_wait_bounded(full0 + 8 * slot, static_cast<uint32_t>((s / kStages) & 1), a.err, 1);
    const T* X = reinterpret_cast<const T*>(st + S::kX);
    const T* Z = reinterpret_cast<const T*>(st + S::kZ);
    const float* Bt = reinterpret_cast<const float*>(st + S::kB);
    const float* Ct = reinterpret_cast<const float*>(st + S::kC);
    const float* D_ = Dr + (s & 1) * kTok;
    const int64_t t0 = s * kTok;
    const bool first = s == 0;
    // Tile row r of x holds token t0 + r - 3.
    auto xrow = [&](int r) {
      if (first && r < 3) return r == 0 ? hx0 : (r == 1 ? hx1 : hx2);
      return IO<T>::to_f(X[r * NCH + c]);
    };

    if constexpr (G == 1) {
      // One thread owns every token of its channel: per-token work and the
      // scan fuse; y goes straight to global memory (a warp writes 32
      // consecutive channels of a token).
      T* yrow = static_cast<T*>(a.y) + static_cast<int64_t>(seq) * a.s.y_seq + e;
      float w0 = xrow(0), w1 = xrow(1), w2 = xrow(2);
      constexpr int kChunk = 8;  // tokens computed before their outputs are stored
#pragma unroll 1
      for (int tc = 0; tc < kTok; tc += kChunk) {
        float yv[kChunk];
#pragma unroll
        for (int k = 0; k < kChunk; ++k) {
          const int tl = tc + k;
          const float w3 = xrow(tl + 3);
          const float conv = fmaf(cw3, w3, fmaf(cw2, w2, fmaf(cw1, w1, fmaf(cw0, w0, cb))));
          w0 = w1;
          w1 = w2;
          w2 = w3;
          const float u = silu(conv);
          float dt = dt_of(fmaf(D_[tl], wdt, dtb), lo, hi);
          if (t0 + tl >= L) dt = 0.0f;  // past the end: keep the state
          const float zg = silu(IO<T>::to_f(Z[tl * NCH + c]));
          float yc;
          if constexpr (ZOH)
            yc = scan_token_zoh<K>(dt, u, Av, h, Bt + tl * 16, Ct + tl * 16);
          else
            yc = scan_token<KP, NPOLY>(pk2(dt, dt), pk2(dt * u, dt * u), a2, h, Bt + tl * 16, Ct + tl * 16);
          yv[k] = (yc + Dd * u) * zg;
        }
        if (ch_ok) {
#pragma unroll
          for (int k = 0; k < kChunk; ++k)
            if (t0 + tc + k < L) yrow[(t0 + tc + k) * a.s.y_tok] = IO<T>::from_f(yv[k]);
        }
      }
    } else {
      float4* DT = reinterpret_cast<float4*>(smem + S::kDT) + c * S::kRow;
      float* P = reinterpret_cast<float*>(smem + S::kP) + c * S::kPCh;
      auto pos = [](int tl) { return tl + tl / TA; };
      // Phase A: tokens [j*TA, (j+1)*TA) of channel c. All inputs are read
      // first and the (dt, dt, dt*u, dt*u) rows written last; D*u and SiLU(z)
      // stay in registers for phase C.
      float du[TA], zg[TA];
      {
        const int tb = j * TA;
        float xw[TA + 3], zr[TA], dr[TA];
#pragma unroll
        for (int i = 0; i < TA + 3; ++i) xw[i] = xrow(tb + i);
#pragma unroll
        for (int i = 0; i < TA; ++i) {
          zr[i] = IO<T>::to_f(Z[(tb + i) * NCH + c]);
          dr[i] = D_[tb + i];
        }
        float4 dtv[TA];
#pragma unroll
        for (int i = 0; i < TA; ++i) {
          const float conv = fmaf(cw3, xw[i + 3], fmaf(cw2, xw[i + 2], fmaf(cw1, xw[i + 1], fmaf(cw0, xw[i], cb))));
          const float u = silu(conv);
          float dt = dt_of(fmaf(dr[i], wdt, dtb), lo, hi);
          if (t0 + tb + i >= L) dt = 0.0f;  // past the end: keep the state
          const float inj = ZOH ? u : dt * u;
          dtv[i] = make_float4(dt, dt, inj, inj);
          du[i] = Dd * u;
          zg[i] = silu(zr[i]);
        }
#pragma unroll
        for (int i = 0; i < TA; ++i) DT[pos(tb + i)] = dtv[i];
      }
      if (tid == 0) bulk_wait_read<1>();  // output tile (s & 1) no longer read by the store of stage s - 2
      named_bar_sync(1, NT);

      // Phase B: this thread's K states through all kTok tokens of the stage.
      // Partial readouts C.h stay in registers until the stream is done.
      float pr[kTok];
#pragma unroll
      for (int tl = 0; tl < kTok; ++tl) {
        const float4 dd = DT[pos(tl)];
        const float* Bp = Bt + tl * 16 + j * K;
        const float* Cp = Ct + tl * 16 + j * K;
        if constexpr (ZOH)
          pr[tl] = scan_token_zoh<K>(dd.x, dd.z, Av, h, Bp, Cp);
        else
          pr[tl] = scan_token<KP>(pk2(dd.x, dd.y), pk2(dd.z, dd.w), a2, h, Bp, Cp);
      }
      {
        float* Pj = P + j * S::kPRow;
#pragma unroll
        for (int tl = 0; tl < kTok; tl += 4)
          *reinterpret_cast<float4*>(Pj + tl) = make_float4(pr[tl], pr[tl + 1], pr[tl + 2], pr[tl + 3]);
      }
      __syncwarp();  // the G slices of a channel live in one warp

      // Phase C: sum the G partials of this thread's phase-A tokens, gate, write the tile.
      {
        const int tb = j * TA;
        float ys[TA];
#pragma unroll
        for (int q = 0; q < TA; q += 4) {
          float4 acc = *reinterpret_cast<const float4*>(P + tb + q);
#pragma unroll
          for (int jj = 1; jj < G; ++jj) {
            const float4 v = *reinterpret_cast<const float4*>(P + jj * S::kPRow + tb + q);
            acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
          }
          ys[q + 0] = (acc.x + du[q + 0]) * zg[q + 0];
          ys[q + 1] = (acc.y + du[q + 1]) * zg[q + 1];
          ys[q + 2] = (acc.z + du[q + 2]) * zg[q + 2];
          ys[q + 3] = (acc.w + du[q + 3]) * zg[q + 3];
        }
        T* Y = reinterpret_cast<T*>(smem + S::kY + (s & 1) * S::kYBytes);
#pragma unroll
        for (int i = 0; i < TA; ++i) Y[(tb + i) * NCH + c] = IO<T>::from_f(ys[i]);
      }
      fence_proxy_async_smem();
    }

    // End of stage: stage dt_raw two ahead, then release the ring slot.
    if (tid < 32) {
      Dr[((s + 1) & 1) * kTok + lane] = d_next;
      const int64_t tn = t0 + 2 * kTok + lane;
      d_next = tn < L ? dtr[tn] : 0.0f;
    }
    named_bar_sync(1, NT);
    if (tid == 0) {
      if constexpr (G > 1) {
        tma_store_3d(&maps.y, sb + S::kY + (s & 1) * S::kYBytes, e0, static_cast<int>(t0), seq);
        bulk_commit();
      }
      if (s + kStages < n_stages) issue_stage(s + kStages);
    }
  }
  if constexpr (G > 1) {
    if (tid == 0) bulk_wait<0>();
  }

  if (ch_ok) {
#pragma unroll
    for (int q = 0; q < K; ++q) a.ssm_state_out[(static_cast<int64_t>(seq) * a.E + e) * 16 + j * K + q] = h[q];
    if (j == 0) {
      // conv_cache_out = last 3 raw rows of [history, x]; read all before
      // writing (the output may alias conv_cache_in).
      const T* x = static_cast<const T*>(a.x);
      const T* hist = static_cast<const T*>(a.conv_cache_in);
      T keep[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int64_t t = L - 3 + k;
        if (t >= 0)
          keep[k] = x[seq * a.s.x_seq + t * a.s.x_tok + e];
        else
          keep[k] = hist ? hist[(static_cast<int64_t>(seq) * 3 + (3 + t)) * a.E + e] : IO<T>::from_f(0.0f);
      }
      T* out = static_cast<T*>(a.conv_cache_out);
#pragma unroll
      for (int k = 0; k < 3; ++k) out[(static_cast<int64_t>(seq) * 3 + k) * a.E + e] = keep[k];
    }
  }
}

// ------------------------------------------------ slice-per-warp kernel ---
// G > 1: a CTA covers 32 channels with G warps; warp J owns states
// [J*16/G, (J+1)*16/G) of every channel (lane = channel). B and C are then
// identical across a warp (broadcast loads), and x, z, the phase-A rows, the
// partial readouts and y are all lane-contiguous (conflict-free).
template <typename T, int G>
struct SliceSmem {
  static constexpr int kEs = static_cast<int>(sizeof(T));
  static constexpr int kXBytes = (kTok + 3) * 32 * kEs;
  static constexpr int kZBytes = kTok * 32 * kEs;
  static constexpr int kBCBytes = kTok * 16 * 4;
  static constexpr int kX = 0;
  static constexpr int kZ = align128(kX + kXBytes);
  static constexpr int kB = align128(kZ + kZBytes);
  static constexpr int kC = kB + kBCBytes;
  static constexpr int kSlot = kC + kBCBytes;
  static constexpr int kDT = kStages * kSlot;               // float2 (dt, dt*u) [token][channel]
  static constexpr int kPR = kTok + 4;                      // partial row (padded)
  static constexpr int kP = kDT + kTok * 32 * 8;            // float [slice][channel][kPR]
  static constexpr int kDr = kP + G * 32 * kPR * 4;         // dt_raw, 2 stages
  static constexpr int kY = align128(kDr + 2 * kTok * 4);   // output tiles [token][channel]
  static constexpr int kYBytes = align128(kTok * 32 * kEs);
  static constexpr int kBar = kY + 2 * kYBytes;
  static constexpr int kTotal = kBar + kStages * 8;
  static constexpr uint32_t kTxBytes = static_cast<uint32_t>(kXBytes + kZBytes + 2 * kBCBytes);
};

// Phase B for one state slice: advance the slice's K states through kTok
// tokens, writing the partial readouts C.h to P[slice][lane][*] kBChunk
// tokens at a time (registers hold a chunk's readouts between stores). The pointers do not alias (distinct shared-memory regions).
template <int K, bool ZOH, int NPOLY, int kBChunk = phase_b_chunk<K>()>
__device__ __forceinline__ void slice_phase_b(const float2* __restrict__ DT, const float* __restrict__ Bs,
                                              const float* __restrict__ Cs, const float* a2, const float* Av, float* h,
                                              float* __restrict__ Pj, int lane) {
#pragma unroll 1
  for (int tc = 0; tc < kTok; tc += kBChunk) {
    float pr[kBChunk];
#pragma unroll
    for (int k = 0; k < kBChunk; ++k) {
      const int tl = tc + k;
      const float2 dd = DT[tl * 32 + lane];
      if constexpr (ZOH)
        pr[k] = scan_token_zoh<K>(dd.x, dd.y, Av, h, Bs + tl * 16, Cs + tl * 16);
      else
        pr[k] = scan_token<K / 2, NPOLY>(pk2(dd.x, dd.x), pk2(dd.y, dd.y), a2, h, Bs + tl * 16, Cs + tl * 16);
    }
#pragma unroll
    for (int k = 0; k < kBChunk; k += 4)
      *reinterpret_cast<float4*>(Pj + tc + k) = make_float4(pr[k], pr[k + 1], pr[k + 2], pr[k + 3]);
  }
}

template <typename T, int G, bool ZOH, int NPOLY>
__global__ void __launch_bounds__(32 * G) prefill_slice_kernel(const __grid_constant__ Maps maps, const KernelArgs a) {
  constexpr int NT = 32 * G;
  constexpr int K = 16 / G;
  constexpr int TA = kTok / G;  // phase-A and phase-C tokens per warp
  using S = SliceSmem<T, G>;
  static_assert(TA % 4 == 0 && K >= 2, "bad slice shape");

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  const uint32_t sb = smem_u32(smem);
  const uint32_t full0 = sb + S::kBar;
  float* Dr = reinterpret_cast<float*>(smem + S::kDr);
  float2* DT = reinterpret_cast<float2*>(smem + S::kDT);
  float* P = reinterpret_cast<float*>(smem + S::kP);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t tiles = (a.E + 31) / 32;
  const int seq = static_cast<int>(blockIdx.x / tiles);
  const int e0 = static_cast<int>(blockIdx.x % tiles) * 32;
  const int64_t L = a.L;
  const int64_t n_stages = (L + kTok - 1) / kTok;
  const float* dtr = a.dt_raw + static_cast<int64_t>(seq) * a.s.dt_seq;

  auto issue_stage = [&](int64_t st_idx) {  // thread 0 only
    const int slot = static_cast<int>(st_idx % kStages);
    const uint32_t base = sb + slot * S::kSlot, bar = full0 + 8 * slot;
    const int t0 = static_cast<int>(st_idx * kTok);
    mbar_arrive_expect_tx(bar, S::kTxBytes);
    tma_load_3d(base + S::kX, &maps.x, e0, t0 - 3, seq, bar);
    tma_load_3d(base + S::kZ, &maps.z, e0, t0, seq, bar);
    tma_load_3d(base + S::kB, &maps.B, 0, t0, seq, bar);
    tma_load_3d(base + S::kC, &maps.C, 0, t0, seq, bar);
  };
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(full0 + 8 * i, 1);
    mbar_fence_init();
    prefetch_tensormap(&maps.x);
    prefetch_tensormap(&maps.z);
    prefetch_tensormap(&maps.B);
    prefetch_tensormap(&maps.C);
    for (int64_t i = 0; i < kStages && i < n_stages; ++i) issue_stage(i);
  }
  float d_next = 0.0f;
  if (tid < 32) {
    Dr[lane] = lane < L ? dtr[lane] : 0.0f;
    d_next = kTok + lane < L ? dtr[kTok + lane] : 0.0f;
  }
  __syncthreads();

  const int e = e0 + lane;
  const bool ch_ok = e < a.E;
  const int64_t ec = ch_ok ? e : a.E - 1;
  const float cw0 = a.conv_w[ec * 4 + 0], cw1 = a.conv_w[ec * 4 + 1];
  const float cw2 = a.conv_w[ec * 4 + 2], cw3 = a.conv_w[ec * 4 + 3];
  const float cb = a.conv_b[ec], wdt = a.w_dt[ec], dtb = a.dt_bias[ec], Dd = a.D[ec];
  const float lo = a.dt_min, hi = a.dt_max;
  float hx0 = 0.0f, hx1 = 0.0f, hx2 = 0.0f;
  if (a.conv_cache_in) {
    const T* hist = static_cast<const T*>(a.conv_cache_in) + static_cast<int64_t>(seq) * 3 * a.E + ec;
    hx0 = IO<T>::to_f(hist[0]);
    hx1 = IO<T>::to_f(hist[a.E]);
    hx2 = IO<T>::to_f(hist[2 * a.E]);
  }
  float a2[K], Av[K], h[K];
#pragma unroll
  for (int q = 0; q < K; ++q) {
    const float A = -expf(a.A_log[ec * 16 + warp * K + q]);
    Av[q] = A;
    a2[q] = A * kLog2e;
    h[q] = a.ssm_state_in ? a.ssm_state_in[(static_cast<int64_t>(seq) * a.E + ec) * 16 + warp * K + q] : 0.0f;
  }

  for (int64_t s = 0; s < n_stages; ++s) {
    const int slot = static_cast<int>(s % kStages);
    const unsigned char* st = smem + slot * S::kSlot;
    mbar_wait_bounded(full0 + 8 * slot, static_cast<uint32_t>((s / kStages) & 1), a.err, 1);
    const T* X = reinterpret_cast<const T*>(st + S::kX);
    const T* Z = reinterpret_cast<const T*>(st + S::kZ);
    const float* Bt = reinterpret_cast<const float*>(st + S::kB);
    const float* Ct = reinterpret_cast<const float*>(st + S::kC);
    const float* D_ = Dr + (s & 1) * kTok;
    const int64_t t0 = s * kTok;
    const bool first = s == 0;
    const int tb = warp * TA;

    // Phase A: tokens [tb, tb + TA) of this lane's channel. Inputs first, then
    // the (dt, dt*u) rows; D*u and SiLU(z) stay in registers for phase C.
    float du[TA], zg[TA];
    {
      float xw[TA + 3], zr[TA], dr[TA];
#pragma unroll
      for (int i = 0; i < TA + 3; ++i) {
        const int r = tb + i;
        xw[i] = (first && r < 3) ? (r == 0 ? hx0 : (r == 1 ? hx1 : hx2)) : IO<T>::to_f(X[r * 32 + lane]);
      }
#pragma unroll
      for (int i = 0; i < TA; ++i) {
        zr[i] = IO<T>::to_f(Z[(tb + i) * 32 + lane]);
        dr[i] = D_[tb + i];
      }
      float2 dtv[TA];
#pragma unroll
      for (int i = 0; i < TA; ++i) {
        const float conv = fmaf(cw3, xw[i + 3], fmaf(cw2, xw[i + 2], fmaf(cw1, xw[i + 1], fmaf(cw0, xw[i], cb))));
        const float u = silu(conv);
        float dt = dt_of(fmaf(dr[i], wdt, dtb), lo, hi);
        if (t0 + tb + i >= L) dt = 0.0f;  // past the end: keep the state
        dtv[i] = make_float2(dt, ZOH ? u : dt * u);
        du[i] = Dd * u;
        zg[i] = silu(zr[i]);
      }
#pragma unroll
      for (int i = 0; i < TA; ++i) DT[(tb + i) * 32 + lane] = dtv[i];
    }
    if (tid == 0) bulk_wait_read<1>();  // output tile (s & 1) no longer read by the store of stage s - 2
    named_bar_sync(1, NT);

    // Phase B: this warp's state slice through all kTok tokens.
    slice_phase_b<K, ZOH, NPOLY>(DT, Bt + warp * K, Ct + warp * K, a2, Av, h, P + (warp * 32 + lane) * S::kPR, lane);
    named_bar_sync(1, NT);

    // Phase C: tokens [tb, tb + TA): sum the G slices, skip, gate, output tile.
    {
      float ys[TA];
#pragma unroll
      for (int q = 0; q < TA; q += 4) {
        float4 acc = *reinterpret_cast<const float4*>(P + lane * S::kPR + tb + q);
#pragma unroll
        for (int jj = 1; jj < G; ++jj) {
          const float4 v = *reinterpret_cast<const float4*>(P + (jj * 32 + lane) * S::kPR + tb + q);
          acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
        }
        ys[q + 0] = (acc.x + du[q + 0]) * zg[q + 0];
        ys[q + 1] = (acc.y + du[q + 1]) * zg[q + 1];
        ys[q + 2] = (acc.z + du[q + 2]) * zg[q + 2];
        ys[q + 3] = (acc.w + du[q + 3]) * zg[q + 3];
      }
      T* Y = reinterpret_cast<T*>(smem + S::kY + (s & 1) * S::kYBytes);
#pragma unroll
      for (int i = 0; i < TA; ++i) Y[(tb + i) * 32 + lane] = IO<T>::from_f(ys[i]);
      fence_proxy_async_smem();
    }

    if (tid < 32) {
      Dr[((s + 1) & 1) * kTok + lane] = d_next;
      const int64_t tn = t0 + 2 * kTok + lane;
      d_next = tn < L ? dtr[tn] : 0.0f;
    }
    named_bar_sync(1, NT);
    if (tid == 0) {
      tma_store_3d(&maps.y, sb + S::kY + (s & 1) * S::kYBytes, e0, static_cast<int>(t0), seq);
      bulk_commit();
      if (s + kStages < n_stages) issue_stage(s + kStages);
    }
  }
  if (tid == 0) bulk_wait<0>();

  if (ch_ok) {
#pragma unroll
    for (int q = 0; q < K; ++q) a.ssm_state_out[(static_cast<int64_t>(seq) * a.E + e) * 16 + warp * K + q] = h[q];
    if (warp == 0) {
      const T* x = static_cast<const T*>(a.x);
      const T* hist = static_cast<const T*>(a.conv_cache_in);
      T keep[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int64_t t = L - 3 + k;
        if (t >= 0)
          keep[k] = x[seq * a.s.x_seq + t * a.s.x_tok + e];
        else
          keep[k] = hist ? hist[(static_cast<int64_t>(seq) * 3 + (3 + t)) * a.E + e] : IO<T>::from_f(0.0f);
      }
      T* out = static_cast<T*>(a.conv_cache_out);
#pragma unroll
      for (int k = 0; k < 3; ++k) out[(static_cast<int64_t>(seq) * 3 + k) * a.E + e] = keep[k];
    }
  }
}

// ---------------------------------------- pipelined state-slice kernel ---
// Kernel 3: the state-slice layout of kernel 2 with the phases software-
// pipelined across stages. While a warp streams its state slice through
// stage s (phase B), it also does the per-token work of stage s+1 (phase A)
// in the same unrolled block, so the two independent instruction streams hide
// each other's latency. The (dt, dt*u) rows are double-buffered; warp 0 copies
// the dt_raw row of stage s + 2 to shared memory with cp.async at the top of
// stage s and waits for it at the end, so no register waits on that load.
#ifndef SSM_PIPE_STAGES
#define SSM_PIPE_STAGES 3
#endif
// Ring depth of kernel 3 (depths 3 to 5 time the same on long sequences).
constexpr int kPipeStages = SSM_PIPE_STAGES;

template <typename T, int G>
struct PipeSmem {
  static constexpr int kEs = static_cast<int>(sizeof(T));
  static constexpr int kXBytes = (kTok + 3) * 32 * kEs;
  static constexpr int kZBytes = kTok * 32 * kEs;
  static constexpr int kBCBytes = kTok * 16 * 4;
  static constexpr int kX = 0;
  static constexpr int kZ = align128(kX + kXBytes);
  static constexpr int kB = align128(kZ + kZBytes);
  static constexpr int kC = kB + kBCBytes;
  static constexpr int kSlot = kC + kBCBytes;
  static constexpr int kDT = kPipeStages * kSlot;             // float4 [2][token pair][channel]
  static constexpr int kPR = kTok + 4;
  static constexpr int kDr = kDT + 2 * kTok * 32 * 8;         // dt_raw float [2][token]
  static constexpr int kP = kDr + 2 * kTok * 4;               // float [slice][channel][kPR]
  static constexpr int kY = align128(kP + G * 32 * kPR * 4);  // output tiles [2][token][channel]
  static constexpr int kYBytes = align128(kTok * 32 * kEs);
  static constexpr int kBar = kY + 2 * kYBytes;
  static constexpr int kTotal = kBar + kPipeStages * 8;
  static constexpr uint32_t kTxBytes = static_cast<uint32_t>(kXBytes + kZBytes + 2 * kBCBytes);
};

// Per-token work of TA tokens [tb, tb+TA) of this lane's channel for one stage:
// (dt, dt*u) of token pairs, D*u and SiLU(z) to registers. Dr is the stage's
// dt_raw row. The caller stores the pairs (store_rows) after the scan, so no
// shared-memory store sits between the scan's loads in program order.
template <typename T, int TA, bool ZOH>
__device__ __forceinline__ void pipe_phase_a(const T* __restrict__ X, const T* __restrict__ Z, const float* __restrict__ Dr,
                                             int64_t t0, int64_t L, int tb, int lane,
                                             bool first, float hx0, float hx1, float hx2, float cw0, float cw1,
                                             float cw2, float cw3, float cb, float wdt, float dtb, float Dd, float lo,
                                             float hi, float4* rows, float* du, float* zg) {
  float xw[TA + 3], zr[TA], dr[TA];
#pragma unroll
  for (int i = 0; i < TA + 3; ++i) {
    const int r = tb + i;
    xw[i] = (first && r < 3) ? (r == 0 ? hx0 : (r == 1 ? hx1 : hx2)) : IO<T>::to_f(X[r * 32 + lane]);
  }
#pragma unroll
  for (int i = 0; i < TA; ++i) {
    zr[i] = IO<T>::to_f(Z[(tb + i) * 32 + lane]);
  }
#pragma unroll
  for (int i = 0; i < TA; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(Dr + tb + i);  // broadcast
    dr[i] = v.x, dr[i + 1] = v.y, dr[i + 2] = v.z, dr[i + 3] = v.w;
  }
  float2 dtv[TA];
#pragma unroll
  for (int i = 0; i < TA; ++i) {
    const float conv = fmaf(cw3, xw[i + 3], fmaf(cw2, xw[i + 2], fmaf(cw1, xw[i + 1], fmaf(cw0, xw[i], cb))));
    const float u = silu(conv);
    float dt = dt_of(fmaf(dr[i], wdt, dtb), lo, hi);
    if (t0 + tb + i >= L) dt = 0.0f;  // past the end: keep the state
    dtv[i] = make_float2(dt, ZOH ? u : dt * u);
    du[i] = Dd * u;
    zg[i] = silu(zr[i]);
  }
#pragma unroll
  for (int i = 0; i < TA; i += 2) rows[i / 2] = make_float4(dtv[i].x, dtv[i].y, dtv[i + 1].x, dtv[i + 1].y);
}

// Rows as [token pair][channel] (dt, inj, dt', inj'): one 16-byte load per two
// tokens in phase B.
template <int TA>
__device__ __forceinline__ void store_rows(float2* DTo, int tb, int lane, const float4* rows) {
  float4* DT4 = reinterpret_cast<float4*>(DTo);
#pragma unroll
  for (int i = 0; i < TA; i += 2) DT4[((tb + i) >> 1) * 32 + lane] = rows[i / 2];
}

// Phase B over tokens [T0, T1) of one stage: this thread's K states; pr gets
// the partial readouts.
template <int K, bool ZOH, int T0 = 0, int T1 = kTok>
__device__ __forceinline__ void scan_stage(const float2* __restrict__ DTc, int lane, const float* Av, const float* a2,
                                           float* h, const float* __restrict__ Bs, const float* __restrict__ Cs,
                                           float* pr) {
#pragma unroll
  for (int tl = T0; tl < T1; ++tl) {
    const float4 d4 = reinterpret_cast<const float4*>(DTc)[(tl >> 1) * 32 + lane];
    const float2 dd = (tl & 1) ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
    if constexpr (ZOH)
      pr[tl] = scan_token_zoh<K>(dd.x, dd.y, Av, h, Bs + tl * 16, Cs + tl * 16);
    else
      pr[tl] = scan_token<K / 2>(pk2(dd.x, dd.x), pk2(dd.y, dd.y), a2, h, Bs + tl * 16, Cs + tl * 16);
  }
}

// MINB 0 leaves the register budget to the compiler (3 CTAs of 4 warps fit an
// SM); MINB 1 lets it use up to 255 registers a thread (2 CTAs fit), which it
// spends on a deeper schedule of the fused block: measured 7% faster when the
// grid needs at most two CTAs per SM, slower when it needs more.
template <typename T, int G, bool ZOH, int MINB>
__global__ void __launch_bounds__(32 * G, MINB) prefill_pipe_kernel(const __grid_constant__ Maps maps, const KernelArgs a) {
  constexpr int NT = 32 * G;
  constexpr int K = 16 / G;
  constexpr int TA = kTok / G;
  using S = PipeSmem<T, G>;
  static_assert(TA % 4 == 0 && K >= 2, "bad pipelined-slice shape");

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  const uint32_t sb = smem_u32(smem);
  const uint32_t full0 = sb + S::kBar;
  float2* DT = reinterpret_cast<float2*>(smem + S::kDT);
  float* Dr = reinterpret_cast<float*>(smem + S::kDr);
  float* P = reinterpret_cast<float*>(smem + S::kP);

  const int tid = threadIdx.x;
  // A warp index the compiler can prove uniform puts the B/C row addresses of
  // the scan in uniform registers (measured: 6% faster than tid >> 5 here).
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0), lane = tid & 31;
  const int64_t tiles = (a.E + 31) / 32;
  const int seq = static_cast<int>(blockIdx.x / tiles);
  const int e0 = static_cast<int>(blockIdx.x % tiles) * 32;
  const int64_t L = a.L;
  const int64_t n_stages = (L + kTok - 1) / kTok;
  const float* dtr = a.dt_raw + static_cast<int64_t>(seq) * a.s.dt_seq;

  auto issue_stage = [&](int64_t st_idx) {  // thread 0 only
    const int slot = static_cast<int>(st_idx % kPipeStages);
    const uint32_t base = sb + slot * S::kSlot, bar = full0 + 8 * slot;
    const int t0 = static_cast<int>(st_idx * kTok);
    mbar_arrive_expect_tx(bar, S::kTxBytes);
    tma_load_3d(base + S::kX, &maps.x, e0, t0 - 3, seq, bar);
    tma_load_3d(base + S::kZ, &maps.z, e0, t0, seq, bar);
    tma_load_3d(base + S::kB, &maps.B, 0, t0, seq, bar);
    tma_load_3d(base + S::kC, &maps.C, 0, t0, seq, bar);
  };
  if (tid == 0) {
    for (int i = 0; i < kPipeStages; ++i) mbar_init(full0 + 8 * i, 1);
    mbar_fence_init();
    prefetch_tensormap(&maps.x);
    prefetch_tensormap(&maps.z);
    prefetch_tensormap(&maps.B);
    prefetch_tensormap(&maps.C);
    for (int64_t i = 0; i < kPipeStages && i < n_stages; ++i) issue_stage(i);
  }
  // dt_raw of stage st_idx (one token per lane of warp 0) into its buffer; zero past the end
  auto copy_dt_raw = [&](int64_t st_idx) {
    const int64_t t = st_idx * kTok + lane;
    cp_async_4(smem_u32(Dr + (st_idx & 1) * kTok + lane), dtr + (t < L ? t : 0), t < L ? 4u : 0u);
    cp_async_commit();
  };
  if (warp == 0) {
    copy_dt_raw(0);
    copy_dt_raw(1);
    cp_async_wait_all();
  }
  __syncthreads();

  const int e = e0 + lane;
  const bool ch_ok = e < a.E;
  const int64_t ec = ch_ok ? e : a.E - 1;
  const float cw0 = a.conv_w[ec * 4 + 0], cw1 = a.conv_w[ec * 4 + 1];
  const float cw2 = a.conv_w[ec * 4 + 2], cw3 = a.conv_w[ec * 4 + 3];
  const float cb = a.conv_b[ec], wdt = a.w_dt[ec], dtb = a.dt_bias[ec], Dd = a.D[ec];
  const float lo = a.dt_min, hi = a.dt_max;
  float hx0 = 0.0f, hx1 = 0.0f, hx2 = 0.0f;
  if (a.conv_cache_in) {
    const T* hist = static_cast<const T*>(a.conv_cache_in) + static_cast<int64_t>(seq) * 3 * a.E + ec;
    hx0 = IO<T>::to_f(hist[0]);
    hx1 = IO<T>::to_f(hist[a.E]);
    hx2 = IO<T>::to_f(hist[2 * a.E]);
  }
  float a2[K], Av[K], h[K];
#pragma unroll
  for (int q = 0; q < K; ++q) {
    const float A = -expf(a.A_log[ec * 16 + warp * K + q]);
    Av[q] = A;
    a2[q] = A * kLog2e;
    h[q] = a.ssm_state_in ? a.ssm_state_in[(static_cast<int64_t>(seq) * a.E + ec) * 16 + warp * K + q] : 0.0f;
  }
  const int tb = warp * TA;

  // Prologue: phase A of stage 0.
  float du[TA], zg[TA];
  {
    float4 rows0[TA / 2];
    mbar_wait_bounded(full0, 0u, a.err, 1);
    pipe_phase_a<T, TA, ZOH>(reinterpret_cast<const T*>(smem + S::kX), reinterpret_cast<const T*>(smem + S::kZ), Dr, 0,
                             L, tb, lane, true, hx0, hx1, hx2, cw0, cw1, cw2, cw3, cb, wdt, dtb, Dd, lo, hi, rows0, du, zg);
    store_rows<TA>(DT, tb, lane, rows0);
  }
  named_bar_sync(1, NT);

  for (int64_t s = 0; s < n_stages; ++s) {
    const int slot = static_cast<int>(s % kPipeStages);
    const unsigned char* st = smem + slot * S::kSlot;
    const float* Bs = reinterpret_cast<const float*>(st + S::kB) + warp * K;
    const float* Cs = reinterpret_cast<const float*>(st + S::kC) + warp * K;
    const float2* DTc = DT + (s & 1) * kTok * 32;
    float2* DTn = DT + ((s + 1) & 1) * kTok * 32;
    const int64_t t0 = s * kTok;
    const bool has_next = s + 1 < n_stages;
    float duN[TA], zgN[TA];
    // dt_raw of stage s + 2 into the buffer that phase A of stage s (block s - 1) has finished with
    if (warp == 0) copy_dt_raw(s + 2);

    // Phase B of stage s fused with phase A of stage s + 1.
    float pr[kTok];
    if (has_next) {
      const int nslot = static_cast<int>((s + 1) % kPipeStages);
      mbar_wait_bounded(full0 + 8 * nslot, static_cast<uint32_t>(((s + 1) / kPipeStages) & 1), a.err, 1);
      const unsigned char* nst = smem + nslot * S::kSlot;
      // Source order: first half of the scan, the next stage's per-token work,
      // second half of the scan (measured 2% faster than either block first).
      float4 rows[TA / 2];
      scan_stage<K, ZOH, 0, kTok / 2>(DTc, lane, Av, a2, h, Bs, Cs, pr);
      pipe_phase_a<T, TA, ZOH>(reinterpret_cast<const T*>(nst + S::kX), reinterpret_cast<const T*>(nst + S::kZ),
                               Dr + ((s + 1) & 1) * kTok,
                               t0 + kTok, L, tb, lane, false, hx0, hx1, hx2, cw0, cw1, cw2, cw3, cb, wdt, dtb, Dd, lo,
                               hi, rows, duN, zgN);
      scan_stage<K, ZOH, kTok / 2, kTok>(DTc, lane, Av, a2, h, Bs, Cs, pr);
      store_rows<TA>(DTn, tb, lane, rows);
    } else {
      scan_stage<K, ZOH>(DTc, lane, Av, a2, h, Bs, Cs, pr);
    }
    {
      float* Pj = P + (warp * 32 + lane) * S::kPR;
#pragma unroll
      for (int tl = 0; tl < kTok; tl += 4)
        *reinterpret_cast<float4*>(Pj + tl) = make_float4(pr[tl], pr[tl + 1], pr[tl + 2], pr[tl + 3]);
    }
    if (tid == 0) bulk_wait_read<1>();  // output tile (s & 1) no longer read by the store of stage s - 2
    named_bar_sync(1, NT);              // partials of stage s and rows of stage s + 1 visible

    // Phase C of stage s: tokens [tb, tb + TA).
    {
      float ys[TA];
#pragma unroll
      for (int q = 0; q < TA; q += 4) {
        float4 acc = *reinterpret_cast<const float4*>(P + lane * S::kPR + tb + q);
#pragma unroll
        for (int jj = 1; jj < G; ++jj) {
          const float4 v = *reinterpret_cast<const float4*>(P + (jj * 32 + lane) * S::kPR + tb + q);
          acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
        }
        ys[q + 0] = (acc.x + du[q + 0]) * zg[q + 0];
        ys[q + 1] = (acc.y + du[q + 1]) * zg[q + 1];
        ys[q + 2] = (acc.z + du[q + 2]) * zg[q + 2];
        ys[q + 3] = (acc.w + du[q + 3]) * zg[q + 3];
      }
      T* Y = reinterpret_cast<T*>(smem + S::kY + (s & 1) * S::kYBytes);
#pragma unroll
      for (int i = 0; i < TA; ++i) Y[(tb + i) * 32 + lane] = IO<T>::from_f(ys[i]);
      fence_proxy_async_smem();
    }
    if (has_next) {
#pragma unroll
      for (int i = 0; i < TA; ++i) {
        du[i] = duN[i];
        zg[i] = zgN[i];
      }
    }
    if (warp == 0) cp_async_wait_all();  // dt_raw of stage s + 2 lands before the barrier
    named_bar_sync(1, NT);  // output tile complete; slot of stage s and its partials free
    if (tid == 0) {
      tma_store_3d(&maps.y, sb + S::kY + (s & 1) * S::kYBytes, e0, static_cast<int>(t0), seq);
      bulk_commit();
      if (s + kPipeStages < n_stages) issue_stage(s + kPipeStages);
    }
  }
  if (tid == 0) bulk_wait<0>();

  if (ch_ok) {
#pragma unroll
    for (int q = 0; q < K; ++q) a.ssm_state_out[(static_cast<int64_t>(seq) * a.E + e) * 16 + warp * K + q] = h[q];
    if (warp == 0) {
      const T* x = static_cast<const T*>(a.x);
      const T* hist = static_cast<const T*>(a.conv_cache_in);
      T keep[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int64_t t = L - 3 + k;
        if (t >= 0)
          keep[k] = x[seq * a.s.x_seq + t * a.s.x_tok + e];
        else
          keep[k] = hist ? hist[(static_cast<int64_t>(seq) * 3 + (3 + t)) * a.E + e] : IO<T>::from_f(0.0f);
      }
      T* out = static_cast<T*>(a.conv_cache_out);
#pragma unroll
      for (int k = 0; k < 3; ++k) out[(static_cast<int64_t>(seq) * 3 + k) * a.E + e] = keep[k];
    }
  }
}

// L == 0: the outputs are the incoming caches (or zeros).
template <typename T>
__global__ void caches_only_kernel(const KernelArgs a) {
  const int64_t ch = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (ch >= a.batch * a.E) return;
  const int64_t seq = ch / a.E, e = ch - seq * a.E;
  for (int n = 0; n < 16; ++n) a.ssm_state_out[ch * 16 + n] = a.ssm_state_in ? a.ssm_state_in[ch * 16 + n] : 0.0f;
  const T* hist = static_cast<const T*>(a.conv_cache_in);
  T* out = static_cast<T*>(a.conv_cache_out);
  T keep[3];
  for (int k = 0; k < 3; ++k) keep[k] = hist ? hist[(seq * 3 + k) * a.E + e] : IO<T>::from_f(0.0f);
  for (int k = 0; k < 3; ++k) out[(seq * 3 + k) * a.E + e] = keep[k];
}

// ------------------------------------------------------------------ host ---
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// Rank-3 tiled map over (inner, rows, seqs) with element strides in bytes.
bool map3(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
          uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0, uint32_t b1) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1_bytes, s2_bytes ? s2_bytes : s1_bytes * d1};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int NCH>
bool make_maps(const KernelArgs& a, Maps* m) {
  const CUtensorMapDataType dt =
      sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint64_t es = sizeof(T), E = a.E, L = a.L, b = a.batch;
  return map3(&m->x, dt, a.x, E, L, b, a.s.x_tok * es, a.s.x_seq * es, NCH, kTok + 3) &&
         map3(&m->z, dt, a.z, E, L, b, a.s.z_tok * es, a.s.z_seq * es, NCH, kTok) &&
         map3(&m->y, dt, a.y, E, L, b, a.s.y_tok * es, a.s.y_seq * es, NCH, kTok) &&
         map3(&m->B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.B, 16, L, b, a.s.bc_tok * 4, a.s.bc_seq * 4, 16, kTok) &&
         map3(&m->C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.C, 16, L, b, a.s.bc_tok * 4, a.s.bc_seq * 4, 16, kTok);
}

template <typename T, int G, int NCH, bool ZOH, int NPOLY>
cudaError_t launch_one(const KernelArgs& a, cudaStream_t st) {
  using S = Smem<T, NCH, G>;
  Maps maps;
  if (!make_maps<T, NCH>(a, &maps)) return cudaErrorInvalidValue;
  auto kern = prefill_kernel<T, G, NCH, ZOH, NPOLY>;
  const int smem = S::kTotal + 128;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int64_t grid = a.batch * ((a.E + NCH - 1) / NCH);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), NCH * G, smem, st>>>(maps, a);
  return cudaGetLastError();
}

template <typename T, int G, bool ZOH, int NPOLY>
cudaError_t launch_slice(const KernelArgs& a, cudaStream_t st) {
  using S = SliceSmem<T, G>;
  Maps maps;
  if (!make_maps<T, 32>(a, &maps)) return cudaErrorInvalidValue;
  auto kern = prefill_slice_kernel<T, G, ZOH, NPOLY>;
  const int smem = S::kTotal + 128;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int64_t grid = a.batch * ((a.E + 31) / 32);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), 32 * G, smem, st>>>(maps, a);
  return cudaGetLastError();
}

template <typename T, int G, bool ZOH, int MINB>
cudaError_t launch_pipe(const KernelArgs& a, cudaStream_t st) {
  using S = PipeSmem<T, G>;
  Maps maps;
  if (!make_maps<T, 32>(a, &maps)) return cudaErrorInvalidValue;
  auto kern = prefill_pipe_kernel<T, G, ZOH, MINB>;
  const int smem = S::kTotal + 128;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int64_t grid = a.batch * ((a.E + 31) / 32);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), 32 * G, smem, st>>>(maps, a);
  return cudaGetLastError();
}

// Every instantiated launch shape. ZOH runs its scalar scan (npoly 0 only).
template <typename T, bool ZOH>
cudaError_t dispatch(const KernelArgs& a, PrefillShape sh, cudaStream_t st) {
#define SSM_SLICE(G_, P_) \
  if (sh.kernel == 2 && sh.G == G_ && sh.npoly == P_) return launch_slice<T, G_, ZOH, P_>(a, st);
#define SSM_TILE(G_, N_, P_) \
  if (sh.kernel == 1 && sh.G == G_ && sh.NCH == N_ && sh.npoly == P_) return launch_one<T, G_, N_, ZOH, P_>(a, st);
  SSM_SLICE(2, 0)
  SSM_SLICE(4, 0)
  SSM_SLICE(8, 0)
  if (sh.kernel == 3 && sh.npoly == 0) {
    if (sh.G == 4) return launch_pipe<T, 4, ZOH, 0>(a, st);
    if (sh.G == 8) return launch_pipe<T, 8, ZOH, 0>(a, st);
  }
  if (sh.kernel == 4 && sh.npoly == 0 && sh.G == 4) return launch_pipe<T, 4, ZOH, 1>(a, st);
  SSM_TILE(1, 32, 0)
  SSM_TILE(1, 64, 0)
  SSM_TILE(1, 128, 0)
  SSM_TILE(2, 16, 0)
  SSM_TILE(2, 32, 0)
  SSM_TILE(2, 64, 0)
  SSM_TILE(4, 8, 0)
  SSM_TILE(4, 16, 0)
  SSM_TILE(4, 32, 0)
  SSM_TILE(8, 8, 0)
  SSM_TILE(8, 16, 0)
  SSM_TILE(8, 32, 0)
  if constexpr (!ZOH) {
    SSM_SLICE(2, 1)
    SSM_SLICE(2, 2)
    SSM_SLICE(4, 1)
    SSM_TILE(1, 32, 1)
    SSM_TILE(1, 32, 2)
    SSM_TILE(1, 32, 3)
    SSM_TILE(1, 64, 1)
    SSM_TILE(1, 64, 2)
    SSM_TILE(1, 128, 1)
    SSM_TILE(1, 128, 2)
  }
#undef SSM_SLICE
#undef SSM_TILE
  return cudaErrorInvalidValue;
}

}  // namespace

bool prefill_shape_supported(PrefillShape sh) {
  const int g = sh.G, n = sh.NCH, p = sh.npoly;
  if (sh.kernel == 2) return (g == 2 && p >= 0 && p <= 2) || (g == 4 && p >= 0 && p <= 1) || (g == 8 && p == 0);
  if (sh.kernel == 3) return (g == 4 || g == 8) && p == 0;
  if (sh.kernel == 4) return g == 4 && p == 0;
  if (sh.kernel != 1) return false;
  if (p != 0) {  // FMA-pipe exp2 variants exist for G == 1 tiles only
    if (g != 1 || p < 0) return false;
    return n == 32 ? p <= 3 : ((n == 64 || n == 128) && p <= 2);
  }
  if (g == 1) return n == 32 || n == 64 || n == 128;
  if (g == 2) return n == 16 || n == 32 || n == 64;
  if (g == 4 || g == 8) return n == 8 || n == 16 || n == 32;
  return false;
}

// Default launch shape: state slices of 4 warps (measured best on B200 for the
// long-context, layer-shape and batched workloads once phase B streams 32
// tokens per chunk). The SFU carries every exp2 (npoly 0): the FMA-pipe
// polynomial measured slower in every shape.
// Pipelined state slices, G = 4 (measured best for every prefill workload);
// the register-rich build when the grid needs at most two CTAs per SM.
PrefillShape choose_prefill_shape(int64_t batch, int64_t E, int64_t /*L*/, int num_sms) {
  const int64_t ctas = batch * ((E + 31) / 32);
  return PrefillShape{4, 32, ctas <= 2 * static_cast<int64_t>(num_sms > 0 ? num_sms : 148) ? 4 : 3, 0};
}

cudaError_t launch_prefill(const KernelArgs& a, bool io_bf16, bool zoh, PrefillShape sh, cudaStream_t st) {
  if (a.L == 0) {
    const int64_t n = a.batch * a.E;
    const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
    if (io_bf16)
      caches_only_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(a);
    else
      caches_only_kernel<float><<<blocks, 256, 0, st>>>(a);
    return cudaGetLastError();
  }
  if (!prefill_shape_supported(sh)) return cudaErrorInvalidValue;
  if (io_bf16) return zoh ? dispatch<__nv_bfloat16, true>(a, sh, st) : dispatch<__nv_bfloat16, false>(a, sh, st);
  return zoh ? dispatch<float, true>(a, sh, st) : dispatch<float, false>(a, sh, st);
}

}  // namespace ssm
