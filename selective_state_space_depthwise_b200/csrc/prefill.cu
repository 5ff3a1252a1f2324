// prefill.cu -- full-sequence selective scan for sm_100a.
//
// One fused kernel computes, for a tile of 32 channels of one sequence and the
// whole length L, the block core of "Axon-SSM: selective state space model"
// ("Algorithm" diagram): causal depthwise conv (K=4) + SiLU, dt =
// clip(softplus(dt_raw*w_dt + dt_bias)), dA = exp(dt*A) with A = -exp(A_log),
// the scan h = dA*h + dt*B*u (the _ssm_fma leaf of "JIT-compiled kernels"),
// y = C.h + D*u and the gate y*SiLU(z). dA, dB and h never reach HBM: the 16
// states of a channel live in registers for the whole walk over L.
//
// Pipeline. L is walked in stages of kTok tokens through a ring in shared
// memory filled by TMA tile loads: the x tile carries a 3-row halo for the
// conv (rows before token 0 come back zero-filled and are replaced by
// conv_cache_in when one is given), B and C (shared by all channels) come as
// [token][16] tiles, and warp 0 copies dt_raw two stages ahead with cp.async.
// Thread 0 re-arms a slot right after the CTA has finished with it; every
// wait on the ring's mbarriers is bounded.
//
// Work split (state slices). A CTA is G = 4 warps over 32 channels
// (lane = channel); warp j holds states 16j/G .. 16(j+1)/G - 1 of every
// channel, so B and C are warp-broadcast loads and x, z, y are lane-contiguous.
// Each 32-token stage:
//  A. warp j does the per-token work of tokens [32j/G, 32(j+1)/G) of its
//     lane's channel (conv from a sliding window of x, SiLU, dt, D*u,
//     SiLU(z)) two tokens at a time on f32x2 operations; the per-token decay
//     operand and dt*u go to shared memory as token-pair rows, D*u and
//     SiLU(z) stay in registers;
//  B. every warp streams its state slice through all 32 tokens (packed f32x2
//     multiplies and FMAs) and keeps the partial readouts C.h in registers;
//  C. warp j sums the G partials of its phase-A tokens, applies the skip and
//     the gate (again two tokens per f32x2 operation), and fills an output
//     tile that leaves by TMA store.
// Phase A of stage s+1 runs inside phase B of stage s (software pipelining),
// so every warp has two independent instruction streams.
//
// Decays. The generic path computes each state's decay on the SFU, dA_n =
// 2^(dt A_n log2 e): 16 exponentials per channel-token. "Axon-SSM", "State
// initialization" sets A_log so that the diagonal of A is -1, -2, ..., -16,
// i.e. A_n = (n+1) A_0. For such a channel exp(dt A_n) = q^(n+1) with
// q = exp(dt A_0): one exponential per channel-token (in phase A) and a few
// multiplications per state slice. At the start each CTA tests its channels'
// A (|A_n - (n+1) A_0| <= 2^-20 |A_n| for every n, on the fp32 values the
// kernel computes); it takes the power path only if all 32 pass, so every
// other channel keeps the generic path. The power path changes each decay
// exponent by at most that 2^-20 relative, far inside the fp32 parity bar.
//
// Kernels. 3: G = 4 with the register budget of three CTAs per SM; 4: G = 4
// built for two CTAs per SM, whose larger register budget buys a deeper
// schedule; 5: the same state slices with phases A and C in four more warps
// of the CTA, handing over through mbarriers (ws_run). Measured alternatives
// at the long-context shape: G = 2 (8 states a thread) executes ~13% fewer
// instructions per channel-token but runs 1.28x slower (one warp per SM sub-partition leaves dependency latencies exposed);
// G = 8 (2 states a thread, 16 warps per SM) runs 1.36x slower: with two
// states a thread the power path saves nothing, and the 16 per-state
// exponentials and the B/C loads then saturate the shared MIO queue. A power
// path forming each slice's first two decays as exponentials (two per slice
// and token, no power chain) ran 1.14x slower: SFU latency on the scan chain.
// Doing phases A and C on token pairs (f32x2) cut the executed instructions
// by 12%: 8% off the batched shape and 5% off the per-state path, but under 1%
// off the long-context power path, which is bound by dependency latency at
// two warps per SM sub-partition, not by issue slots. One-warp CTAs over 8
// channels (960 CTAs for E = 7680, six or seven warps on every SM instead of
// kernel 4's eight or four) ran 5% slower there: per-lane slice arithmetic
// adds 9% instructions and the warps' latency is no better hidden.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "ssm_internal.h"
#include "ssm_math.cuh"

namespace ssm {
namespace {

constexpr int kTok = 32;  // tokens per pipeline stage (= lanes of the dt_raw stager)
// G warps per CTA = state slices; each thread holds 16 / G states of its lane's
// channel and does the per-token work of kTok / G tokens per stage.
#ifndef SSM_PIPE_STAGES
#define SSM_PIPE_STAGES 3
#endif
// Ring depth (depths 3 to 5 time the same on long sequences).
constexpr int kPipeStages = SSM_PIPE_STAGES;
// Power-path test: |A_n - (n+1) A_0| <= kPowTol |A_n|.
constexpr float kPowTol = 9.5367431640625e-07f;  // 2^-20

struct Maps {
  CUtensorMap x, z, B, C, y;
};

constexpr int align128(int v) { return (v + 127) / 128 * 128; }

// Shared-memory layout (byte offsets from a 128-aligned base). SPLIT: the
// partial readouts alternate between two buffers by stage parity (the split
// end-of-stage barrier needs them; see pipe_run).
template <typename T, int G, bool SPLIT>
struct PipeSmem {
  static constexpr int kEs = static_cast<int>(sizeof(T));
  static constexpr int kXBytes = (kTok + 3) * 32 * kEs;  // TMA box {32, kTok + 3}
  static constexpr int kZBytes = kTok * 32 * kEs;        // TMA box {32, kTok}
  static constexpr int kBCBytes = kTok * 16 * 4;         // TMA box {16, kTok}
  static constexpr int kX = 0;
  static constexpr int kZ = align128(kX + kXBytes);
  static constexpr int kB = align128(kZ + kZBytes);
  static constexpr int kC = kB + kBCBytes;
  static constexpr int kSlot = kC + kBCBytes;
  static constexpr int kDT = kPipeStages * kSlot;             // float4 [2][token pair][channel]
  static constexpr int kPR = kTok + 4;                        // partial row (padded)
  static constexpr int kDr = kDT + 2 * kTok * 32 * 8;         // dt_raw float [2][token]
  static constexpr int kPBytes = G * 32 * kPR * 4;            // float [slice][channel][kPR]
  static constexpr int kP = kDr + 2 * kTok * 4;               // partials, double-buffered by stage parity
  static constexpr int kY = align128(kP + (SPLIT ? 2 : 1) * kPBytes);  // output tiles [2][token][channel]
  static constexpr int kYBytes = align128(kTok * 32 * kEs);
  static constexpr int kBar = kY + 2 * kYBytes;
  static constexpr int kTotal = kBar + kPipeStages * 8;
  static constexpr uint32_t kTxBytes = static_cast<uint32_t>(kXBytes + kZBytes + 2 * kBCBytes);
  static_assert((32 * kEs) % 16 == 0, "TMA rows must be whole 16-byte chunks");
};

// Generic decays: advance the thread's 2 KP states (KP packed pairs) through
// one token; returns C.h over them. dt2 = {dt, dt}, inj2 = {dt*u, dt*u}.
template <int KP>
__device__ __forceinline__ float scan_token(uint64_t dt2, uint64_t inj2, const float* a2, float* h, const float* Bp,
                                            const float* Cp) {
  uint64_t acc = 0;
#pragma unroll
  for (int q = 0; q < KP; q += 2) {
    const float4 bq = *reinterpret_cast<const float4*>(Bp + 2 * q);
    const float4 cq = *reinterpret_cast<const float4*>(Cp + 2 * q);
    float x0, x1, x2, x3;
    upk2(fmul2(dt2, pk2(a2[2 * q], a2[2 * q + 1])), x0, x1);
    upk2(fmul2(dt2, pk2(a2[2 * q + 2], a2[2 * q + 3])), x2, x3);
    const uint64_t hb0 =
        ffma2(pk2(ex2_approx(x0), ex2_approx(x1)), pk2(h[2 * q], h[2 * q + 1]), fmul2(inj2, pk2(bq.x, bq.y)));
    const uint64_t hb1 =
        ffma2(pk2(ex2_approx(x2), ex2_approx(x3)), pk2(h[2 * q + 2], h[2 * q + 3]), fmul2(inj2, pk2(bq.z, bq.w)));
    upk2(hb0, h[2 * q], h[2 * q + 1]);
    upk2(hb1, h[2 * q + 2], h[2 * q + 3]);
    acc = q == 0 ? fmul2(pk2(cq.x, cq.y), hb0) : ffma2(pk2(cq.x, cq.y), hb0, acc);
    acc = ffma2(pk2(cq.z, cq.w), hb1, acc);
  }
  float lo, hi;
  upk2(acc, lo, hi);
  return lo + hi;
}

// Zero-order-hold decays, in state pairs: h = e^{dt A} h + (e^{dt A} - 1)/A
// * u * B, the input scale as zoh_scale_pair forms it (rA = 1 / A).
template <int K>
__device__ __forceinline__ float scan_token_zoh(float dt, float u, const float* Av, const float* rA, float* h,
                                                const float* Bp, const float* Cp) {
  static_assert(K % 4 == 0, "states in groups of 4");
  const uint64_t dt2 = pk2(dt, dt), u2 = pk2(u, u);
  uint64_t acc = 0;
#pragma unroll
  for (int q = 0; q < K; q += 4) {
    const float4 bq = *reinterpret_cast<const float4*>(Bp + q);
    const float4 cq = *reinterpret_cast<const float4*>(Cp + q);
#pragma unroll
    for (int r = 0; r < 4; r += 2) {
      const int i = q + r;
      const uint64_t x = fmul2(dt2, pk2(Av[i], Av[i + 1]));
      float l0, l1;
      upk2(fmul2(x, pk2(kLog2e, kLog2e)), l0, l1);
      const uint64_t ex = pk2(ex2_approx(l0), ex2_approx(l1));
      const uint64_t c = zoh_scale_pair(x, dt2, ex, pk2(rA[i], rA[i + 1]));
      const uint64_t b2 = r == 0 ? pk2(bq.x, bq.y) : pk2(bq.z, bq.w);
      const uint64_t c2 = r == 0 ? pk2(cq.x, cq.y) : pk2(cq.z, cq.w);
      const uint64_t hh = ffma2(ex, pk2(h[i], h[i + 1]), fmul2(fmul2(c, u2), b2));
      upk2(hh, h[i], h[i + 1]);
      acc = i == 0 ? fmul2(c2, hh) : ffma2(c2, hh, acc);
    }
  }
  float lo, hi;
  upk2(acc, lo, hi);
  return lo + hi;
}

// Decay operand stored per token: dt (generic), q = e^{dt A_0} (power path),
// dt (ZOH, with u instead of dt*u as the second value).
enum class Path { kGeneric, kPow, kZoh };

// Two tokens per f32x2 operation. The packed forms round exactly as the scalar
// ones (same operations in the same order), so both give the same bits.
__device__ __forceinline__ uint64_t splat2(float v) { return pk2(v, v); }

__device__ __forceinline__ uint64_t ex2_pair(uint64_t x) {
  float x0, x1;
  upk2(x, x0, x1);
  return pk2(ex2_approx(x0), ex2_approx(x1));
}

// SiLU of both halves: v / (1 + 2^(-v log2 e)).
__device__ __forceinline__ uint64_t silu_pair(uint64_t v) {
  const uint64_t e = ex2_pair(fmul2(v, splat2(-kLog2e)));
  float d0, d1;
  upk2(fadd2(e, splat2(1.0f)), d0, d1);
  return fmul2(v, pk2(rcp_approx(d0), rcp_approx(d1)));
}

// clip(softplus(v), lo, hi) of both halves (softplus as in dt_of).
__device__ __forceinline__ uint64_t dt_pair(uint64_t v, float lo, float hi) {
  float v0, v1;
  upk2(v, v0, v1);
  const uint64_t e = pk2(ex2_approx(-fabsf(v0) * kLog2e), ex2_approx(-fabsf(v1) * kLog2e));
  uint64_t q = ffma2(e, splat2(log1p_q(0)), splat2(log1p_q(1)));
#pragma unroll
  for (int k = 2; k <= kLog1pDeg; ++k) q = ffma2(e, q, splat2(log1p_q(k)));
  float s0, s1;
  upk2(fadd2(pk2(fmaxf(v0, 0.0f), fmaxf(v1, 0.0f)), fmul2(e, q)), s0, s1);
  return pk2(fminf(fmaxf(s0, lo), hi), fminf(fmaxf(s1, lo), hi));
}

// Rows of tokens at or past L (last stage only) become the row of a token that
// keeps the state: decay 1 (or dt 0) and no injection.
template <Path P, int kTA>
__device__ __forceinline__ void fix_rows(float4* rows, int64_t t0, int64_t L, int tb) {
  if (t0 + tb + kTA > L) {
    constexpr float kKeep = P == Path::kPow ? 1.0f : 0.0f;  // q = 1, or dt = 0
#pragma unroll
    for (int p = 0; p < kTA / 2; ++p) {
      const int64_t t = t0 + tb + 2 * p;
      if (t >= L) rows[p].x = kKeep, rows[p].z = 0.0f;
      if (t + 1 >= L) rows[p].y = kKeep, rows[p].w = 0.0f;
    }
  }
}

// Per-token work of tokens [tb, tb + kTA) of this lane's channel for one
// stage, as kTA / 2 token pairs that share each f32x2 operation. Outputs per
// pair: the row (d, d', inj, inj') of decay operands and injections, D*u and
// SiLU(z). Tokens at or past L get the row of a
// token that changes nothing (decay 1, no injection). The caller stores the
// rows (store_rows) after the scan, so no shared-memory store sits between
// the scan's loads in program order.
struct PhaseAConsts {
  float cw0, cw1, cw2, cw3, cb, wdt, dtb, Dd, lo, hi, a20;
};

// The x rows of tokens tb - 3 .. tb + kTA - 1 (the conv window of the
// thread's phase-A tokens); rows before the sequence start come from the
// incoming conv cache (first stage).
template <typename T, int kTA>
__device__ __forceinline__ void phase_a_window(const T* __restrict__ X, int tb, int lane, bool first, float hx0,
                                               float hx1, float hx2, float* xw) {
#pragma unroll
  for (int i = 0; i < kTA + 3; ++i) {
    const int r = tb + i;
    xw[i] = (first && r < 3) ? (r == 0 ? hx0 : (r == 1 ? hx1 : hx2)) : IO<T>::to_f(X[r * 32 + lane]);
  }
}

// Token pair t, t + 1 (t from the stage start; x = its conv window, 5 rows).
template <typename T, Path P>
__device__ __forceinline__ void phase_a_pair(const float* x, const T* __restrict__ Z, float2 dr, int t, int lane,
                                             const PhaseAConsts& k, float4& row, uint64_t& du2, uint64_t& zg2) {
  const float c0 = fmaf(k.cw3, x[3], fmaf(k.cw2, x[2], fmaf(k.cw1, x[1], fmaf(k.cw0, x[0], k.cb))));
  const float c1 = fmaf(k.cw3, x[4], fmaf(k.cw2, x[3], fmaf(k.cw1, x[2], fmaf(k.cw0, x[1], k.cb))));
  const float z0 = IO<T>::to_f(Z[t * 32 + lane]), z1 = IO<T>::to_f(Z[(t + 1) * 32 + lane]);
  const uint64_t u2 = silu_pair(pk2(c0, c1));
  const uint64_t dt2 = dt_pair(ffma2(pk2(dr.x, dr.y), splat2(k.wdt), splat2(k.dtb)), k.lo, k.hi);
  uint64_t r1, r2;
  if constexpr (P == Path::kPow)
    r1 = ex2_pair(fmul2(dt2, splat2(k.a20)));
  else
    r1 = dt2;
  if constexpr (P == Path::kZoh)
    r2 = u2;
  else
    r2 = fmul2(dt2, u2);
  float a0, a1, b0, b1;
  upk2(r1, a0, a1);
  upk2(r2, b0, b1);
  row = make_float4(a0, a1, b0, b1);
  du2 = fmul2(splat2(k.Dd), u2);
  zg2 = silu_pair(pk2(z0, z1));
}

template <typename T, Path P, int kTA>
__device__ __forceinline__ void phase_a(const T* __restrict__ X, const T* __restrict__ Z, const float* __restrict__ Dr,
                                        int64_t t0, int64_t L, int tb, int lane, bool first, float hx0, float hx1,
                                        float hx2, float cw0, float cw1, float cw2, float cw3, float cb, float wdt,
                                        float dtb, float Dd, float lo, float hi, float a20, float4* rows, uint64_t* du2,
                                        uint64_t* zg2) {
  float xw[kTA + 3];
  phase_a_window<T, kTA>(X, tb, lane, first, hx0, hx1, hx2, xw);
  const PhaseAConsts k{cw0, cw1, cw2, cw3, cb, wdt, dtb, Dd, lo, hi, a20};
#pragma unroll
  for (int p = 0; p < kTA / 2; ++p)
    phase_a_pair<T, P>(xw + 2 * p, Z, *reinterpret_cast<const float2*>(Dr + tb + 2 * p), tb + 2 * p, lane, k, rows[p],
                       du2[p], zg2[p]);  // dt_raw: a broadcast load
  fix_rows<P, kTA>(rows, t0, L, tb);
}

// Rows as [token pair][channel] (d, d', inj, inj'): one 16-byte load per two
// tokens in phase B.
template <int kTA>
__device__ __forceinline__ void store_rows(float2* DTo, int tb, int lane, const float4* rows) {
  float4* DT4 = reinterpret_cast<float4*>(DTo);
#pragma unroll
  for (int p = 0; p < kTA / 2; ++p) DT4[((tb >> 1) + p) * 32 + lane] = rows[p];
}

// Power decays, 4 states a thread: states 4j .. 4j + 3 decay by q^(4j+1) ..
// q^(4j+4) = base * (q, q^2, q^3, q^4) with base = q^(4j); hi1 / hi2
// (warp-uniform) are the bits of j, so base = (q^4)^(j&1) (q^8)^(j>>1 & 1).
// pow_prep forms everything of token tl that does not depend on the state:
// its decays, its injections dt*u*B (row values q and dt*u) and its C.
struct TokPrep {
  uint64_t d01, d23, b01, b23, c01, c23;
};
__device__ __forceinline__ TokPrep pow_prep(const float2* __restrict__ DTc, int lane, int tl, bool hi1, bool hi2,
                                            const float* __restrict__ Bs, const float* __restrict__ Cs) {
  const float4 d4 = reinterpret_cast<const float4*>(DTc)[(tl >> 1) * 32 + lane];
  const float q = (tl & 1) ? d4.y : d4.x, inj = (tl & 1) ? d4.w : d4.z;
  const float4 bq = *reinterpret_cast<const float4*>(Bs + tl * 16);
  const float4 cq = *reinterpret_cast<const float4*>(Cs + tl * 16);
  const float q2 = q * q;
  const uint64_t p0 = pk2(q, q2);
  const uint64_t p1 = fmul2(p0, pk2(q2, q2));
  float q3, q4;
  upk2(p1, q3, q4);
  float base = hi1 ? q4 : 1.0f;
  if (hi2) base *= q4 * q4;
  const uint64_t bb = pk2(base, base), i2 = pk2(inj, inj);
  TokPrep r;
  r.d01 = fmul2(bb, p0);
  r.d23 = fmul2(bb, p1);
  r.b01 = fmul2(i2, pk2(bq.x, bq.y));
  r.b23 = fmul2(i2, pk2(bq.z, bq.w));
  r.c01 = pk2(cq.x, cq.y);
  r.c23 = pk2(cq.z, cq.w);
  return r;
}

// Phase B over tokens [T0, T1) with each token's state-independent part
// prepared kScanLA tokens ahead of its state update. Measured on the power
// path at L = 16384: E = 7680 0.903 ms with 4 ahead, 0.905 with 2, 0.93-0.94
// with 1 and 0.94 with none (the same arithmetic in every case); 4 ahead was
// also best or within 0.4% of best at E = 4736 and on 8 x 4096 x 5120. The
// same for the per-state path made the batched shape 4% slower.
constexpr int kScanLA = 4;
template <int T0, int T1, typename Prep>
__device__ __forceinline__ void scan_stage_la(Prep prep, float* h, float* pr) {
  constexpr int LA = kScanLA;
  uint64_t h01 = pk2(h[0], h[1]), h23 = pk2(h[2], h[3]);
  TokPrep buf[LA + 1];
#pragma unroll
  for (int j = 0; j < LA; ++j)
    if (T0 + j < T1) buf[j] = prep(T0 + j);
#pragma unroll
  for (int tl = T0; tl < T1; ++tl) {
    const TokPrep cu = buf[(tl - T0) % (LA + 1)];
    if (tl + LA < T1) buf[(tl - T0 + LA) % (LA + 1)] = prep(tl + LA);
    h01 = ffma2(cu.d01, h01, cu.b01);
    h23 = ffma2(cu.d23, h23, cu.b23);
    float lo, hi;
    upk2(ffma2(cu.c23, h23, fmul2(cu.c01, h01)), lo, hi);
    pr[tl] = lo + hi;
  }
  upk2(h01, h[0], h[1]);
  upk2(h23, h[2], h[3]);
}

// Phase B over tokens [T0, T1) of one stage: this thread's 4 states; pr gets
// the partial readouts.
template <Path P, int K, int T0 = 0, int T1 = kTok>
__device__ __forceinline__ void scan_stage(const float2* __restrict__ DTc, int lane, const float* Av, const float* rA,
                                           const float* a2, bool hi1, bool hi2, float* h, const float* __restrict__ Bs,
                                           const float* __restrict__ Cs, float* pr) {
  if constexpr (P == Path::kPow) {
    static_assert(K == 4, "power decays are built for 4 states per thread");
    scan_stage_la<T0, T1>([&](int tl) { return pow_prep(DTc, lane, tl, hi1, hi2, Bs, Cs); }, h, pr);
  } else {
#pragma unroll
    for (int tl = T0; tl < T1; ++tl) {
      const float4 d4 = reinterpret_cast<const float4*>(DTc)[(tl >> 1) * 32 + lane];
      const float2 dd = (tl & 1) ? make_float2(d4.y, d4.w) : make_float2(d4.x, d4.z);
      if constexpr (P == Path::kZoh)
        pr[tl] = scan_token_zoh<K>(dd.x, dd.y, Av, rA, h, Bs + tl * 16, Cs + tl * 16);
      else
        pr[tl] = scan_token<K / 2>(pk2(dd.x, dd.x), pk2(dd.y, dd.y), a2, h, Bs + tl * 16, Cs + tl * 16);
    }
  }
}

// Phase C for 4 consecutive tokens of one channel: the sum of the NS slices'
// partial readouts (slice j at Pj + j * stride), plus D*u, times SiLU(z).
template <int NS, int stride>
__device__ __forceinline__ void gate_pairs(const float* Pj, const uint64_t* du, const uint64_t* zg, float* ys) {
  const float4 a4 = *reinterpret_cast<const float4*>(Pj);
  uint64_t lo = pk2(a4.x, a4.y), hi = pk2(a4.z, a4.w);
#pragma unroll
  for (int j = 1; j < NS; ++j) {
    const float4 v = *reinterpret_cast<const float4*>(Pj + j * stride);
    lo = fadd2(lo, pk2(v.x, v.y));
    hi = fadd2(hi, pk2(v.z, v.w));
  }
  upk2(fmul2(fadd2(lo, du[0]), zg[0]), ys[0], ys[1]);
  upk2(fmul2(fadd2(hi, du[1]), zg[1]), ys[2], ys[3]);
}

// The whole walk over L for one CTA of G warps, on the decay path P. Two
// barriers per stage: barrier 1 after the scan (partials, next rows and dt_raw
// visible; ring slot s free) and barrier 2 after phase C (output tile
// complete). SPLIT: at barrier 2 only warp 0, which stores the tile, waits;
// the others arrive and run on, which needs the partials double-buffered.
template <typename T, int G, Path P, bool SPLIT>
__device__ __forceinline__ void pipe_run(const Maps& maps, const KernelArgs& a) {
  constexpr int NT = 32 * G;
  constexpr int kK = 16 / G;     // states per thread
  constexpr int kTA = kTok / G;  // phase-A and phase-C tokens per warp and stage
  using S = PipeSmem<T, G, SPLIT>;

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  const uint32_t sb = smem_u32(smem);
  const uint32_t full0 = sb + S::kBar;
  float2* DT = reinterpret_cast<float2*>(smem + S::kDT);
  float* Dr = reinterpret_cast<float*>(smem + S::kDr);

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
  float a2[kK], Av[kK], rA[kK], h[kK];
#pragma unroll
  for (int q = 0; q < kK; ++q) {
    const float A = -expf(a.A_log[ec * 16 + warp * kK + q]);
    Av[q] = A;
    rA[q] = 1.0f / A;  // ZOH only
    a2[q] = A * kLog2e;
    h[q] = a.ssm_state_in ? a.ssm_state_in[(static_cast<int64_t>(seq) * a.E + ec) * 16 + warp * kK + q] : 0.0f;
  }
  const float a20 = -expf(a.A_log[ec * 16]) * kLog2e;  // A_0 log2(e): q = 2^(dt a20) on the power path
  const bool hi1 = (warp & 1) != 0, hi2 = (warp & 2) != 0;  // bits of the slice index (power path)
  const int tb = warp * kTA;

  // Prologue: phase A of stage 0.
  uint64_t du[kTA / 2], zg[kTA / 2];  // D*u and SiLU(z) of token pairs
  {
    float4 rows0[kTA / 2];
    mbar_wait_bounded(full0, 0u, a.err, 1);
    phase_a<T, P, kTA>(reinterpret_cast<const T*>(smem + S::kX), reinterpret_cast<const T*>(smem + S::kZ), Dr, 0, L,
                       tb, lane, true, hx0, hx1, hx2, cw0, cw1, cw2, cw3, cb, wdt, dtb, Dd, lo, hi, a20, rows0, du, zg);
    store_rows<kTA>(DT, tb, lane, rows0);
  }
  named_bar_sync(1, NT);

  for (int64_t s = 0; s < n_stages; ++s) {
    const int slot = static_cast<int>(s % kPipeStages);
    const unsigned char* st = smem + slot * S::kSlot;
    const float* Bs = reinterpret_cast<const float*>(st + S::kB) + warp * kK;
    const float* Cs = reinterpret_cast<const float*>(st + S::kC) + warp * kK;
    const float2* DTc = DT + (s & 1) * kTok * 32;
    float2* DTn = DT + ((s + 1) & 1) * kTok * 32;
    const int64_t t0 = s * kTok;
    const bool has_next = s + 1 < n_stages;
    uint64_t duN[kTA / 2], zgN[kTA / 2];
    float* P_ = reinterpret_cast<float*>(smem + S::kP + (SPLIT ? (s & 1) * S::kPBytes : 0));
    // dt_raw of stage s + 2 into the buffer that phase A of stage s (block s - 1) has finished with
    if (warp == 0) copy_dt_raw(s + 2);

    // Phase B of stage s fused with phase A of stage s + 1.
    float pr[kTok];
    float* Pj = P_ + (warp * 32 + lane) * S::kPR;  // this thread's partial readouts
    if (has_next) {
      const int nslot = static_cast<int>((s + 1) % kPipeStages);
      mbar_wait_bounded(full0 + 8 * nslot, static_cast<uint32_t>(((s + 1) / kPipeStages) & 1), a.err, 1);
      const unsigned char* nst = smem + nslot * S::kSlot;
      // Source order: first half of the scan, the next stage's per-token work,
      // second half of the scan (measured 2% faster than either block first,
      // and 5% faster on the power path than one token pair of the next
      // stage after every 8 tokens of the scan).
      float4 rows[kTA / 2];
      scan_stage<P, kK, 0, kTok / 2>(DTc, lane, Av, rA, a2, hi1, hi2, h, Bs, Cs, pr);
      phase_a<T, P, kTA>(reinterpret_cast<const T*>(nst + S::kX), reinterpret_cast<const T*>(nst + S::kZ),
                         Dr + ((s + 1) & 1) * kTok, t0 + kTok, L, tb, lane, false, hx0, hx1, hx2, cw0, cw1, cw2, cw3,
                         cb, wdt, dtb, Dd, lo, hi, a20, rows, duN, zgN);
      scan_stage<P, kK, kTok / 2, kTok>(DTc, lane, Av, rA, a2, hi1, hi2, h, Bs, Cs, pr);
      store_rows<kTA>(DTn, tb, lane, rows);
    } else {
      scan_stage<P, kK>(DTc, lane, Av, rA, a2, hi1, hi2, h, Bs, Cs, pr);
    }
#pragma unroll
    for (int tl = 0; tl < kTok; tl += 4)
      *reinterpret_cast<float4*>(Pj + tl) = make_float4(pr[tl], pr[tl + 1], pr[tl + 2], pr[tl + 3]);
    if (warp == 0) cp_async_wait_all();  // dt_raw of stage s + 2 lands before the barrier
    if (tid == 0) bulk_wait_read<1>();    // output tile (s & 1) no longer read by the store of stage s - 2
    // Partials of stage s, rows of stage s + 1 and dt_raw of stage s + 2
    // visible; every warp is done with ring slot s (phase A of s ran in the
    // previous block, phase B of s just now), so it is re-armed at once.
    named_bar_sync(1, NT);
    if (tid == 0 && s + kPipeStages < n_stages) issue_stage(s + kPipeStages);

    // Phase C of stage s: tokens [tb, tb + kTA).
    {
      float ys[kTA];
#pragma unroll
      for (int q = 0; q < kTA; q += 4)
        gate_pairs<G, 32 * S::kPR>(P_ + lane * S::kPR + tb + q, du + q / 2, zg + q / 2, ys + q);
      T* Y = reinterpret_cast<T*>(smem + S::kY + (s & 1) * S::kYBytes);
#pragma unroll
      for (int i = 0; i < kTA; ++i) Y[(tb + i) * 32 + lane] = IO<T>::from_f(ys[i]);
      fence_proxy_async_smem();
    }
    if (has_next) {
#pragma unroll
      for (int i = 0; i < kTA / 2; ++i) {
        du[i] = duN[i];
        zg[i] = zgN[i];
      }
    }
    // The output tile is complete once every warp has written its tokens.
    // SPLIT: warp 0 waits for that and stores it; the other warps only arrive
    // and go on to the next stage (no other buffer needs this barrier: the
    // partials alternate by stage parity, and the next writer of any buffer
    // read in phase C passes barrier 1 of the next stage first). Otherwise
    // every warp waits, which also frees the single partials buffer.
    if (!SPLIT || warp == 0) {
      named_bar_sync(2, NT);
      if (tid == 0) {
        tma_store_3d(&maps.y, sb + S::kY + (s & 1) * S::kYBytes, e0, static_cast<int>(t0), seq);
        bulk_commit();
      }
    } else {
      named_bar_arrive(2, NT);
    }
  }
  griddep_launch_dependents();  // the next kernel may be launched (it waits for this one to finish)
  if (tid == 0) bulk_wait<0>();

  if (ch_ok) {
#pragma unroll
    for (int q = 0; q < kK; ++q) a.ssm_state_out[(static_cast<int64_t>(seq) * a.E + e) * 16 + warp * kK + q] = h[q];
    if (warp == 0) {
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

// ------------------------------------------- warp-specialised CTA (kernel 5) ---
// The same state slices as pipe_run (state warp j holds states 4j .. 4j + 3 of
// its lane's channel), with the per-token work moved to four more warps of the
// CTA: token warp k does phase A of tokens [8k, 8k + 8) of stage s + 1 and then
// phase C of the same tokens of stage s, while the state warps scan stage s.
// The two groups hand over through mbarriers, each a double buffer: rows of
// decay operands and injections (token -> state warps) and partial readouts
// (state -> token warps). No warp waits at a CTA-wide barrier, and with two
// CTAs of eight warps every SM sub-partition holds four warps instead of two.
// Token warp 0's lane 0 keeps the TMA ring of x, z, B and C filled; the gated
// outputs leave by direct stores (each token a 32-channel row, one per lane).
constexpr int kWsSlots = 4;     // ring depth (stage s + 4 is loaded once stage s is scanned)
constexpr int kWsThreads = 256;  // 4 state warps, then 4 token warps
constexpr int kWsTA = kTok / 4;  // phase-A and phase-C tokens per token warp and stage

template <typename T>
struct WsSmem {
  static constexpr int kEs = static_cast<int>(sizeof(T));
  static constexpr int kXBytes = (kTok + 3) * 32 * kEs;  // TMA box {32, kTok + 3}
  static constexpr int kZBytes = kTok * 32 * kEs;        // TMA box {32, kTok}
  static constexpr int kBCBytes = kTok * 16 * 4;         // TMA box {16, kTok}
  static constexpr int kX = 0;
  static constexpr int kZ = align128(kX + kXBytes);
  static constexpr int kB = align128(kZ + kZBytes);
  static constexpr int kC = kB + kBCBytes;
  static constexpr int kSlot = align128(kC + kBCBytes);
  static constexpr int kRowBytes = (kTok / 2) * 32 * 16;  // float4 [token pair][channel]
  static constexpr int kRows = kWsSlots * kSlot;         // [2] row buffers
  static constexpr int kPR = kTok + 4;                   // partial row (padded)
  static constexpr int kPBytes = 4 * 32 * kPR * 4;       // float [slice][channel][kPR]
  static constexpr int kP = kRows + 2 * kRowBytes;       // [2] partial buffers
  static constexpr int kBar = kP + 2 * kPBytes;          // full[kWsSlots], then 4 pairs (below)
  static constexpr int kTotal = kBar + (kWsSlots + 8) * 8;
  static constexpr uint32_t kTxBytes = static_cast<uint32_t>(kXBytes + kZBytes + 2 * kBCBytes);
};

template <typename T, Path P>
__device__ __forceinline__ void ws_run(const Maps& maps, const KernelArgs& a) {
  using S = WsSmem<T>;
  constexpr int kTA = kWsTA;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  const uint32_t sb = smem_u32(smem);
  const uint32_t full0 = sb + S::kBar;                 // ring slot landed (TMA transaction count)
  const uint32_t rows_full = full0 + 8 * kWsSlots;     // rows of a stage written (128 token threads)
  const uint32_t rows_free = rows_full + 16;           // rows of a stage read (128 state threads)
  const uint32_t part_full = rows_free + 16;           // partials of a stage written (state threads)
  const uint32_t part_free = part_full + 16;           // partials of a stage read (token threads)
  float4* R = reinterpret_cast<float4*>(smem + S::kRows);
  float* PB = reinterpret_cast<float*>(smem + S::kP);

  const int tid = threadIdx.x;
  const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0), lane = tid & 31;
  const int64_t tiles = (a.E + 31) / 32;
  const int seq = static_cast<int>(blockIdx.x / tiles);
  const int e0 = static_cast<int>(blockIdx.x % tiles) * 32;
  const int64_t L = a.L;
  const int64_t n_stages = (L + kTok - 1) / kTok;
  const int e = e0 + lane;
  const bool ch_ok = e < a.E;
  const int64_t ec = ch_ok ? e : a.E - 1;
  // A thread whose wait gave up (error word set) waits no more, so a broken
  // hand-over ends the kernel after one time-out per thread, not one per stage.
  bool live = true;
  auto wait = [&](uint32_t bar, uint32_t parity) {
    if (live) live = mbar_wait_bounded(bar, parity, a.err, 2);
  };

  if (tid == 0) {
    for (int i = 0; i < kWsSlots; ++i) mbar_init(full0 + 8 * i, 1);
    for (int i = 0; i < 8; ++i) mbar_init(rows_full + 8 * i, 128);
    mbar_fence_init();
  }
  __syncthreads();

  if (warp >= 4) {
    // ---------------- token warps: phases A and C, and the TMA ring.
    const int k = warp - 4, tb = k * kTA;
    const bool issuer = tid == 128;
    auto issue_stage = [&](int64_t st_idx) {
      const int slot = static_cast<int>(st_idx % kWsSlots);
      const uint32_t base = sb + slot * S::kSlot, bar = full0 + 8 * slot;
      const int t0 = static_cast<int>(st_idx * kTok);
      mbar_arrive_expect_tx(bar, S::kTxBytes);
      tma_load_3d(base + S::kX, &maps.x, e0, t0 - 3, seq, bar);
      tma_load_3d(base + S::kZ, &maps.z, e0, t0, seq, bar);
      tma_load_3d(base + S::kB, &maps.B, 0, t0, seq, bar);
      tma_load_3d(base + S::kC, &maps.C, 0, t0, seq, bar);
    };
    if (issuer) {
      prefetch_tensormap(&maps.x);
      prefetch_tensormap(&maps.z);
      prefetch_tensormap(&maps.B);
      prefetch_tensormap(&maps.C);
      for (int64_t i = 0; i < kWsSlots && i < n_stages; ++i) issue_stage(i);
    }
    const PhaseAConsts kc{a.conv_w[ec * 4 + 0], a.conv_w[ec * 4 + 1], a.conv_w[ec * 4 + 2], a.conv_w[ec * 4 + 3],
                          a.conv_b[ec], a.w_dt[ec], a.dt_bias[ec], a.D[ec], a.dt_min, a.dt_max,
                          -expf(a.A_log[ec * 16]) * kLog2e};
    float hx0 = 0.0f, hx1 = 0.0f, hx2 = 0.0f;
    if (a.conv_cache_in) {
      const T* hist = static_cast<const T*>(a.conv_cache_in) + static_cast<int64_t>(seq) * 3 * a.E + ec;
      hx0 = IO<T>::to_f(hist[0]);
      hx1 = IO<T>::to_f(hist[a.E]);
      hx2 = IO<T>::to_f(hist[2 * a.E]);
    }
    // dt_raw: lane i holds token tb + (i & 7) of a stage, loaded a stage before its use.
    const float* dtr = a.dt_raw + static_cast<int64_t>(seq) * a.s.dt_seq;
    auto load_dr = [&](int64_t st_idx) -> float {
      const int64_t t = st_idx * kTok + tb + (lane & 7);
      return t < L ? __ldg(dtr + t) : 0.0f;
    };
    // Phase A of stage st_idx: rows to row buffer (st_idx & 1) once the state
    // warps have read its previous contents (stage st_idx - 2).
    auto phase_a_ws = [&](int64_t st_idx, float dr, uint64_t* du2, uint64_t* zg2) {
      const int slot = static_cast<int>(st_idx % kWsSlots);
      wait(full0 + 8 * slot, static_cast<uint32_t>((st_idx / kWsSlots) & 1));
      const unsigned char* st = smem + slot * S::kSlot;
      float xw[kTA + 3];
      phase_a_window<T, kTA>(reinterpret_cast<const T*>(st + S::kX), tb, lane, st_idx == 0, hx0, hx1, hx2, xw);
      float4 rows[kTA / 2];
#pragma unroll
      for (int p = 0; p < kTA / 2; ++p) {
        const float2 d2 = make_float2(__shfl_sync(0xffffffffu, dr, 2 * p), __shfl_sync(0xffffffffu, dr, 2 * p + 1));
        phase_a_pair<T, P>(xw + 2 * p, reinterpret_cast<const T*>(st + S::kZ), d2, tb + 2 * p, lane, kc, rows[p],
                           du2[p], zg2[p]);
      }
      fix_rows<P, kTA>(rows, st_idx * kTok, L, tb);
      const int b = static_cast<int>(st_idx & 1);
      if (st_idx >= 2) wait(rows_free + 8 * b, static_cast<uint32_t>(((st_idx - 2) >> 1) & 1));
      store_rows<kTA>(reinterpret_cast<float2*>(R + b * (kTok / 2) * 32), tb, lane, rows);
      mbar_arrive(rows_full + 8 * b);
    };

    uint64_t du[kTA / 2], zg[kTA / 2], duN[kTA / 2], zgN[kTA / 2];
    float dr_next = load_dr(0);
    {
      const float dr = dr_next;
      dr_next = load_dr(1);
      phase_a_ws(0, dr, du, zg);
    }
    T* Y = static_cast<T*>(a.y) + static_cast<int64_t>(seq) * a.s.y_seq + e;
    for (int64_t s = 0; s < n_stages; ++s) {
      const bool has_next = s + 1 < n_stages;
      if (has_next) {
        const float dr = dr_next;
        dr_next = load_dr(s + 2);
        phase_a_ws(s + 1, dr, duN, zgN);
      }
      // Phase C of stage s.
      const int b = static_cast<int>(s & 1);
      wait(part_full + 8 * b, static_cast<uint32_t>((s >> 1) & 1));
      // Stage s is scanned and its phase A is long done: its slot takes stage s + kWsSlots.
      if (issuer && s + kWsSlots < n_stages) issue_stage(s + kWsSlots);
      float ys[kTA];
      const float* Pp = PB + b * (S::kPBytes / 4) + lane * S::kPR + tb;
#pragma unroll
      for (int q = 0; q < kTA; q += 4) gate_pairs<4, 32 * S::kPR>(Pp + q, du + q / 2, zg + q / 2, ys + q);
      mbar_arrive(part_free + 8 * b);
      const int64_t t0 = s * kTok + tb;
#pragma unroll
      for (int i = 0; i < kTA; ++i)
        if (ch_ok && t0 + i < L) Y[(t0 + i) * a.s.y_tok] = IO<T>::from_f(ys[i]);
      if (has_next) {
#pragma unroll
        for (int i = 0; i < kTA / 2; ++i) {
          du[i] = duN[i];
          zg[i] = zgN[i];
        }
      }
    }
    if (k == 0 && ch_ok) {
      // conv_cache_out = last 3 raw rows of [history, x]; read all before
      // writing (the output may alias conv_cache_in).
      const T* x = static_cast<const T*>(a.x);
      const T* hist = static_cast<const T*>(a.conv_cache_in);
      T keep[3];
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int64_t t = L - 3 + j;
        if (t >= 0)
          keep[j] = x[seq * a.s.x_seq + t * a.s.x_tok + e];
        else
          keep[j] = hist ? hist[(static_cast<int64_t>(seq) * 3 + (3 + t)) * a.E + e] : IO<T>::from_f(0.0f);
      }
      T* out = static_cast<T*>(a.conv_cache_out);
#pragma unroll
      for (int j = 0; j < 3; ++j) out[(static_cast<int64_t>(seq) * 3 + j) * a.E + e] = keep[j];
    }
  } else {
    // ---------------- state warps: phase B.
    float a2[4], Av[4], rA[4], h[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float A = -expf(a.A_log[ec * 16 + warp * 4 + q]);
      Av[q] = A;
      rA[q] = 1.0f / A;  // ZOH only
      a2[q] = A * kLog2e;
      h[q] = a.ssm_state_in ? a.ssm_state_in[(static_cast<int64_t>(seq) * a.E + ec) * 16 + warp * 4 + q] : 0.0f;
    }
    const bool hi1 = (warp & 1) != 0, hi2 = (warp & 2) != 0;
    float* Pj = PB + (warp * 32 + lane) * S::kPR;
    for (int64_t s = 0; s < n_stages; ++s) {
      const int slot = static_cast<int>(s % kWsSlots), b = static_cast<int>(s & 1);
      wait(full0 + 8 * slot, static_cast<uint32_t>((s / kWsSlots) & 1));
      wait(rows_full + 8 * b, static_cast<uint32_t>((s >> 1) & 1));
      const unsigned char* st = smem + slot * S::kSlot;
      const float* Bs = reinterpret_cast<const float*>(st + S::kB) + warp * 4;
      const float* Cs = reinterpret_cast<const float*>(st + S::kC) + warp * 4;
      float pr[kTok];
      scan_stage<P, 4>(reinterpret_cast<const float2*>(R + b * (kTok / 2) * 32), lane, Av, rA, a2, hi1, hi2, h, Bs,
                       Cs, pr);
      mbar_arrive(rows_free + 8 * b);
      if (s >= 2) wait(part_free + 8 * b, static_cast<uint32_t>(((s - 2) >> 1) & 1));
      float* Pw = Pj + b * (S::kPBytes / 4);
#pragma unroll
      for (int tl = 0; tl < kTok; tl += 4)
        *reinterpret_cast<float4*>(Pw + tl) = make_float4(pr[tl], pr[tl + 1], pr[tl + 2], pr[tl + 3]);
      mbar_arrive(part_full + 8 * b);
    }
    if (ch_ok) {
#pragma unroll
      for (int q = 0; q < 4; ++q) a.ssm_state_out[(static_cast<int64_t>(seq) * a.E + e) * 16 + warp * 4 + q] = h[q];
    }
  }
  griddep_launch_dependents();  // the next kernel may be launched (it waits for this one to finish)
}

// True when every channel of this CTA has A_n = (n+1) A_0 to within kPowTol
// (on the fp32 A = -expf(A_log) the kernel uses). Called by all NT threads of
// the CTA; warp j < G checks states 16j/G .. 16(j+1)/G - 1 of its lane's
// channel (warps past G only vote).
template <int G, int NT = 32 * G>
__device__ __forceinline__ bool cta_has_power_decays(const KernelArgs& a) {
  const int64_t tiles = (a.E + 31) / 32;
  const int64_t e = (blockIdx.x % tiles) * 32 + (threadIdx.x & 31);
  const int64_t ec = e < a.E ? e : a.E - 1;
  const float4* row = reinterpret_cast<const float4*>(a.A_log + ec * 16);  // 16-byte aligned rows
  const float A0 = -expf(a.A_log[ec * 16]);
  const int j = static_cast<int>(threadIdx.x >> 5);
  bool ok = true;
#pragma unroll
  for (int v4 = 0; v4 < 4 / G; ++v4) {
    if (NT > 32 * G && j >= G) break;
    const int q4 = j * (4 / G) + v4;
    const float4 v = row[q4];
    const float al[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = 4 * q4 + i;
      const float An = -expf(al[i]);
      ok = ok && fabsf(An - static_cast<float>(n + 1) * A0) <= kPowTol * fabsf(An);
    }
  }
  return __syncthreads_and(ok) != 0;
}

// MINB 0 leaves the register budget to the compiler (3 CTAs of 4 warps fit an
// SM); MINB 1 lets it use up to 255 registers a thread (2 CTAs fit), which it
// spends on a deeper schedule of the fused block (see choose_prefill_shape).
// The split end-of-stage barrier (double-buffered partials) is used where
// the shared memory allows: not in the three-CTAs-per-SM build. The build
// switch turns it off everywhere (for side-by-side measurements).
#ifndef SSM_PREFILL_SPLIT_BARRIER
#define SSM_PREFILL_SPLIT_BARRIER 1
#endif
template <int MINB>
__host__ __device__ constexpr bool split_barrier() {
  return MINB == 1 && SSM_PREFILL_SPLIT_BARRIER;
}

template <typename T, int G, bool ZOH, int MINB>
__global__ void __launch_bounds__(32 * G, MINB) prefill_pipe_kernel(const __grid_constant__ Maps maps,
                                                                     const KernelArgs a) {
  constexpr bool SPLIT = split_barrier<MINB>();
  // Launched overlapped with the kernel before it (programmatic dependent
  // launch, in the block forward): nothing in global memory is touched before
  // that kernel has finished. Without that launch attribute it returns at once.
  griddep_wait();
  if constexpr (ZOH) {
    pipe_run<T, G, Path::kZoh, SPLIT>(maps, a);
  } else {
    const bool pw = a.decay_path == 0 && cta_has_power_decays<G>(a);
    if (pw)
      pipe_run<T, G, Path::kPow, SPLIT>(maps, a);
    else
      pipe_run<T, G, Path::kGeneric, SPLIT>(maps, a);
  }
}

template <typename T, bool ZOH>
__global__ void __launch_bounds__(kWsThreads, 2) prefill_ws_kernel(const __grid_constant__ Maps maps,
                                                                    const KernelArgs a) {
  griddep_wait();  // as in prefill_pipe_kernel
  if constexpr (ZOH) {
    ws_run<T, Path::kZoh>(maps, a);
  } else {
    const bool pw = a.decay_path == 0 && cta_has_power_decays<4, kWsThreads>(a);
    if (pw)
      ws_run<T, Path::kPow>(maps, a);
    else
      ws_run<T, Path::kGeneric>(maps, a);
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

template <typename T>
bool make_maps(const KernelArgs& a, Maps* m) {
  const CUtensorMapDataType dt =
      sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint64_t es = sizeof(T), E = a.E, L = a.L, b = a.batch;
  return map3(&m->x, dt, a.x, E, L, b, a.s.x_tok * es, a.s.x_seq * es, 32, kTok + 3) &&
         map3(&m->z, dt, a.z, E, L, b, a.s.z_tok * es, a.s.z_seq * es, 32, kTok) &&
         map3(&m->y, dt, a.y, E, L, b, a.s.y_tok * es, a.s.y_seq * es, 32, kTok) &&
         map3(&m->B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.B, 16, L, b, a.s.bc_tok * 4, a.s.bc_seq * 4, 16, kTok) &&
         map3(&m->C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.C, 16, L, b, a.s.bc_tok * 4, a.s.bc_seq * 4, 16, kTok);
}

template <typename T, int G, bool ZOH, int MINB>
cudaError_t launch_pipe(const KernelArgs& a, cudaStream_t st, bool pdl) {
  using S = PipeSmem<T, G, split_barrier<MINB>()>;
  Maps maps;
  if (!make_maps<T>(a, &maps)) return cudaErrorInvalidValue;
  auto kern = prefill_pipe_kernel<T, G, ZOH, MINB>;
  const int smem = S::kTotal + 128;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int64_t grid = a.batch * ((a.E + 31) / 32);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(32 * G, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  err = cudaLaunchKernelEx(&cfg, kern, maps, a);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

template <typename T, bool ZOH>
cudaError_t launch_ws(const KernelArgs& a, cudaStream_t st, bool pdl) {
  Maps maps;
  if (!make_maps<T>(a, &maps)) return cudaErrorInvalidValue;
  auto kern = prefill_ws_kernel<T, ZOH>;
  const int smem = WsSmem<T>::kTotal + 128;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int64_t grid = a.batch * ((a.E + 31) / 32);
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kWsThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  err = cudaLaunchKernelEx(&cfg, kern, maps, a);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

template <typename T, bool ZOH>
cudaError_t dispatch(const KernelArgs& a, PrefillShape sh, cudaStream_t st, bool pdl) {
  if (sh.kernel == 3) return launch_pipe<T, 4, ZOH, 0>(a, st, pdl);
  if (sh.kernel == 4) return launch_pipe<T, 4, ZOH, 1>(a, st, pdl);
  if (sh.kernel == 5) return launch_ws<T, ZOH>(a, st, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace

bool prefill_shape_supported(PrefillShape sh) { return sh.kernel >= 3 && sh.kernel <= 5; }

// Measured on B200 (L = 16384 unless stated): with at most one CTA per SM
// the warp-specialised kernel 5 was 4% faster than kernel 4 on the power path
// and 20% faster on the per-state path (32 to 148 CTAs). From two CTAs per SM
// on it was 8% slower on the power path (160 to 296 CTAs), so the
// register-rich kernel 4 takes those grids, unless every CTA is known to run
// per-state exponentials (ZOH, or per-state decays forced): there kernel 5
// was level at 240 CTAs and 2-8% faster from 480 to 15360 CTAs. Kernel 4
// matched or beat kernel 3 from 80 to 5120 CTAs (by 1-27%); at 61440 CTAs
// (256 sequences of 7680 channels) kernel 3 was 2.6% faster.
PrefillShape choose_prefill_shape(int64_t batch, int64_t E, int64_t /*L*/, int num_sms, bool per_state) {
  const int64_t ctas = batch * ((E + 31) / 32), sms = num_sms > 0 ? num_sms : 148;
  if (ctas <= sms) return PrefillShape{5};
  if (ctas > 64 * sms) return PrefillShape{3};
  return PrefillShape{per_state ? 5 : 4};
}

cudaError_t launch_prefill(const KernelArgs& a, bool io_bf16, bool zoh, PrefillShape sh, cudaStream_t st, bool pdl) {
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
  if (io_bf16)
    return zoh ? dispatch<__nv_bfloat16, true>(a, sh, st, pdl) : dispatch<__nv_bfloat16, false>(a, sh, st, pdl);
  return zoh ? dispatch<float, true>(a, sh, st, pdl) : dispatch<float, false>(a, sh, st, pdl);
}

}  // namespace ssm
