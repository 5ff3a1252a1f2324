/*
 * ssm_oracle.c -- plain, slow, double-precision CPU definition of the
 * selective state-space block core (Mamba-style, diagonal A, one B/C group).
 *
 * TEST INFRASTRUCTURE. This file is the parity oracle for the CUDA path.
 * Only the test suite, the package smoke check and the benchmark's CPU
 * baseline leg may load it. The product path never calls it, and it shares
 * no code, header, table or constant with the CUDA sources.
 *
 * Sources (web pages, cited by title and section):
 *  [AX]  "Axon-SSM: selective state space model" (Bit-Axon architecture docs):
 *        the block diagram under "Algorithm" (conv1d causal kernel=4 groups=E,
 *        SiLU, x_proj -> B, C, dt_raw, dt_proj 1->E + softplus + clip, SSM scan,
 *        y * SiLU(z)); "State initialization" (A = -exp(A_log), diagonals
 *        -1 .. -d_state); "JIT-compiled kernels" (_ssm_fma: dA*h + dB*x_t,
 *        _compute_dt: clip(softplus(dt + dt_bias), lo, hi)); "Autoregressive
 *        decoding" (prefill with cache=None starts from a zero state and builds
 *        conv_cache from the last K-1 positions; decode concatenates conv_cache
 *        with the new token and runs one scan step from the carried state).
 *  [SSM] "Mamba/SSM basics" (molayo insights), "Technical details": the
 *        zero-order-hold discretisation Abar = exp(dA), Bbar = (dA)^-1 (exp(dA) - I) dB.
 *  [UL]  "State Space Models (SSM)" (Ultralytics glossary), "How SSMs work":
 *        a fixed-parameter scan equals convolution with K_k = C . (Abar^k Bbar).
 *  [TX]  "What is the Mamba model?" (velog, Texnee), "Mamba computation":
 *        unrolled form h_t = (prod A) h_0 + sum_j (prod_{i>j} A_i) B_j x_j;
 *        "chunkscan": the output adds the skip D . x of the scan input.
 *
 * Readings where the pages are silent or lost in extraction (each is listed
 * in the design notes):
 *  - The recurrence and discretisation display equations of [AX] did not
 *    survive extraction. Default discretisation is the "Euler-B" form that the
 *    _ssm_fma leaf and [TX]'s dt[s]*x[s] factor imply: dA = exp(dt*A),
 *    dB*x = dt*B*x. ORACLE_ZOH selects [SSM]'s zero-order-hold form instead.
 *  - The scan input and the D skip both use u = SiLU(conv(x)) (the order of
 *    [AX]'s diagram; [TX] adds D times the scan input).
 *  - Causal conv = cross-correlation over [K-1 history rows, x], weight K-1
 *    multiplies the current token.
 *  - softplus has no threshold (exact log1p form); clip(.) = min(max(.,lo),hi).
 *  - conv_cache holds the raw (pre-conv) x rows; with L < K-1 the older rows
 *    come from the incoming history (zeros for a fresh prefill).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_EULER_B 0
#define ORACLE_ZOH 1

/* [AX] "Algorithm": causal depthwise conv1d of one channel.
 * xh = [hist[0..K-2], x[0..L-1]];  c_t = bias + sum_{k<K} w[k] * xh[t + k]. */
void oracle_causal_conv(int64_t L, int K, const double *hist, const double *x,
                        const double *w, double bias, double *c) {
  for (int64_t t = 0; t < L; ++t) {
    double acc = bias;
    for (int k = 0; k < K; ++k) {
      int64_t j = t + k - (K - 1); /* index into x; negative = history row */
      double v;
      if (j >= 0)
        v = x[j];
      else
        v = hist ? hist[(K - 1) + j] : 0.0;
      acc += w[k] * v;
    }
    c[t] = acc;
  }
}

/* [AX] "Algorithm": SiLU(v) = v * sigmoid(v). */
double oracle_silu(double v) { return v / (1.0 + exp(-v)); }

/* [AX] "JIT-compiled kernels" (_compute_dt): softplus, written in the
 * overflow-free form log(1 + e^v) = max(v, 0) + log1p(e^-|v|). */
double oracle_softplus(double v) { return fmax(v, 0.0) + log1p(exp(-fabs(v))); }

/* [AX] "Algorithm" (dt_proj 1 -> E, no bias of its own) and _compute_dt:
 * dt = clip(softplus(dt_raw * w_dt + dt_bias), lo, hi). */
double oracle_dt(double dt_raw, double w_dt, double dt_bias, double lo, double hi) {
  double sp = oracle_softplus(dt_raw * w_dt + dt_bias);
  return fmin(fmax(sp, lo), hi);
}

/* [AX] "State initialization": A = -exp(A_log). */
double oracle_A(double A_log) { return -exp(A_log); }

/* The selective scan of one channel with a diagonal A (N states):
 *   [AX] _ssm_fma:  h_n <- dA_n * h_n + dB_n * u_t,  dA_n = exp(dt_t * A_n)
 *   Euler-B:        dB_n * u_t = dt_t * B_{t,n} * u_t
 *   ZOH ([SSM]):    dB_n * u_t = (exp(dt_t A_n) - 1) / A_n * B_{t,n} * u_t
 *   readout:        y_t = sum_n C_{t,n} h_n + D * u_t   ([TX] "chunkscan")
 * B, C are [L][N] row-major; h0 may be NULL (zero state, [AX] prefill).
 * y[t] receives the pre-gate output; h_out the state after the last token. */
void oracle_scan(int64_t L, int N, int disc, const double *u, const double *dt,
                 const double *A, const double *B, const double *C, double D,
                 const double *h0, double *y, double *h_out) {
  double *h = (double *)malloc(sizeof(double) * (size_t)N);
  for (int n = 0; n < N; ++n) h[n] = h0 ? h0[n] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    double acc = 0.0;
    for (int n = 0; n < N; ++n) {
      double a = dt[t] * A[n];
      double dA = exp(a);
      double inj;
      if (disc == ORACLE_ZOH)
        inj = (A[n] != 0.0 ? expm1(a) / A[n] : dt[t]) * B[t * N + n] * u[t];
      else
        inj = dt[t] * B[t * N + n] * u[t];
      h[n] = dA * h[n] + inj;
      acc += C[t * N + n] * h[n];
    }
    y[t] = acc + D * u[t];
  }
  for (int n = 0; n < N; ++n) h_out[n] = h[n];
  free(h);
}

/* One channel of the block core, in [AX]'s order:
 *   conv -> SiLU -> dt -> A -> scan (+ D skip) -> gate y * SiLU(z).
 * Inputs are the stored values of one channel, widened exactly to double.
 * hist (K-1 raw x rows) and h0 (N) may be NULL (fresh prefill).
 * Outputs: out[L] (gated), h_out[N], hist_out[K-1] (last K-1 raw rows of
 * [hist, x]; the conv_cache of [AX] "Autoregressive decoding"). */
void oracle_channel(int64_t L, int N, int K, int disc, double lo, double hi,
                    const double *x, const double *z, const double *B,
                    const double *C, const double *dt_raw, const double *conv_w,
                    double conv_b, double w_dt, double dt_bias,
                    const double *A_log, double D, const double *hist,
                    const double *h0, double *out, double *h_out,
                    double *hist_out) {
  double *c = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  double *u = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  double *dt = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  double *A = (double *)malloc(sizeof(double) * (size_t)N);
  oracle_causal_conv(L, K, hist, x, conv_w, conv_b, c);
  for (int64_t t = 0; t < L; ++t) {
    u[t] = oracle_silu(c[t]);
    dt[t] = oracle_dt(dt_raw[t], w_dt, dt_bias, lo, hi);
  }
  for (int n = 0; n < N; ++n) A[n] = oracle_A(A_log[n]);
  oracle_scan(L, N, disc, u, dt, A, B, C, D, h0, out, h_out);
  for (int64_t t = 0; t < L; ++t) out[t] = out[t] * oracle_silu(z[t]);
  /* last K-1 rows of xh = [hist, x] */
  for (int k = 0; k < K - 1; ++k) {
    int64_t j = L - (K - 1) + k; /* index into x */
    hist_out[k] = j >= 0 ? x[j] : (hist ? hist[(K - 1) + j] : 0.0);
  }
  free(c);
  free(u);
  free(dt);
  free(A);
}

/* Many channels, one call. Channel i reads its own columns x[i*L..], z[i*L..],
 * its parameters at index i, and the B/C/dt_raw of sequence bidx[i]
 * (B, C: [nseq][L][N]; dt_raw: [nseq][L]). hist / h0 may be NULL.
 * Channels are independent, so the loop may run on several threads
 * (n_threads <= 0: leave the OpenMP default). */
void oracle_channels(int64_t n_ch, int64_t L, int N, int K, int disc, double lo,
                     double hi, const double *x, const double *z,
                     const double *B, const double *C, const double *dt_raw,
                     const int64_t *bidx, const double *conv_w,
                     const double *conv_b, const double *w_dt,
                     const double *dt_bias, const double *A_log,
                     const double *D, const double *hist, const double *h0,
                     double *out, double *h_out, double *hist_out,
                     int n_threads) {
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t i = 0; i < n_ch; ++i) {
    int64_t b = bidx[i];
    oracle_channel(L, N, K, disc, lo, hi, x + i * L, z + i * L, B + b * L * N,
                   C + b * L * N, dt_raw + b * L, conv_w + i * K, conv_b[i],
                   w_dt[i], dt_bias[i], A_log + i * N, D[i],
                   hist ? hist + i * (K - 1) : NULL, h0 ? h0 + i * N : NULL,
                   out + i * L, h_out + i * N, hist_out + i * (K - 1));
  }
}

/* [AX] "Algorithm": the x_proj input u = SiLU(conv1d(x)) of n channels (the
 * branch that feeds x_proj in the block diagram), channel i from x[i*L..] with
 * its own weights and history (hist may be NULL: zeros). */
void oracle_conv_silu_channels(int64_t n_ch, int64_t L, int K, const double *x,
                               const double *conv_w, const double *conv_b,
                               const double *hist, double *u, int n_threads) {
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(static)
#endif
  for (int64_t i = 0; i < n_ch; ++i) {
    oracle_causal_conv(L, K, hist ? hist + i * (K - 1) : NULL, x + i * L,
                       conv_w + i * K, conv_b[i], u + i * L);
    for (int64_t t = 0; t < L; ++t) u[i * L + t] = oracle_silu(u[i * L + t]);
  }
}

/* Threads the OpenMP runtime would use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
