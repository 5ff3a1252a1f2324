"""Parity oracle for the selective state-space block core (test infrastructure).

Thin ctypes wrapper around ``ssm_oracle.c``, the plain double-precision CPU
definition of the method. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import this package; the product path never
does, and nothing here is shared with the CUDA sources.

Arrays are widened exactly to float64 before the call (bf16/fp32 -> f64 is
exact), so the oracle sees the very values the kernels read.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssm_oracle.c")
LIB = os.path.join(HERE, "libssm_oracle.so")

EULER_B = 0
ZOH = 1
_DISC = {"euler": EULER_B, "euler_b": EULER_B, "zoh": ZOH}

_lib = None


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into libssm_oracle.so (gcc, OpenMP, IEEE math)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", SRC, "-o", LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        d, i64, i32 = ctypes.c_double, ctypes.c_int64, ctypes.c_int
        p = ctypes.c_void_p
        lib.oracle_scan.argtypes = [i64, i32, i32, p, p, p, p, p, d, p, p, p]
        lib.oracle_scan.restype = None
        lib.oracle_channels.argtypes = [i64, i64, i32, i32, i32, d, d] + [p] * 5 + [p] * 7 + [p, p] + [p, p, p] + [i32]
        lib.oracle_channels.restype = None
        lib.oracle_causal_conv.argtypes = [i64, i32, p, p, p, d, p]
        lib.oracle_causal_conv.restype = None
        lib.oracle_conv_silu_channels.argtypes = [i64, i64, i32, p, p, p, p, p, i32]
        lib.oracle_conv_silu_channels.restype = None
        for name in ("oracle_silu", "oracle_softplus", "oracle_A"):
            getattr(lib, name).argtypes = [d]
            getattr(lib, name).restype = d
        lib.oracle_dt.argtypes = [d, d, d, d, d]
        lib.oracle_dt.restype = d
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i32
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def silu(v: float) -> float:
    return _load().oracle_silu(float(v))


def softplus(v: float) -> float:
    return _load().oracle_softplus(float(v))


def dt_of(dt_raw: float, w_dt: float, dt_bias: float, lo: float, hi: float) -> float:
    return _load().oracle_dt(float(dt_raw), float(w_dt), float(dt_bias), float(lo), float(hi))


def A_of(A_log: float) -> float:
    return _load().oracle_A(float(A_log))


def causal_conv(x, w, bias=0.0, hist=None):
    """Causal depthwise conv of one channel: returns c[L]."""
    x, w, hist = _f64(x), _f64(w), _f64(hist)
    L, K = x.shape[0], w.shape[0]
    c = np.empty(max(L, 1))
    _load().oracle_causal_conv(L, K, _ptr(hist), _ptr(x), _ptr(w), float(bias), _ptr(c))
    return c[:L]


def scan(u, dt, A, B, C, D=0.0, h0=None, disc="euler"):
    """Selective scan of one channel. u, dt: [L]; A: [N]; B, C: [L, N].
    Returns (y_pre_gate[L], h_final[N])."""
    u, dt, A, B, C, h0 = map(_f64, (u, dt, A, B, C, h0))
    L, N = u.shape[0], A.shape[0]
    assert B.shape == (L, N) and C.shape == (L, N) and dt.shape == (L,)
    y = np.empty(max(L, 1))
    h = np.empty(N)
    _load().oracle_scan(L, N, _DISC[disc], _ptr(u), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), float(D), _ptr(h0), _ptr(y), _ptr(h))
    return y[:L], h


def channels(x, z, B, C, dt_raw, bidx, conv_w, conv_b, w_dt, dt_bias, A_log, D,
             hist=None, h0=None, lo=1e-4, hi=1.0, disc="euler", threads=0):
    """Run the block core on n independent channels.

    x, z: [n, L] (the channel's columns); B, C: [nseq, L, N]; dt_raw: [nseq, L];
    bidx: [n] sequence index of each channel; conv_w: [n, K]; conv_b, w_dt,
    dt_bias, D: [n]; A_log: [n, N]; hist: [n, K-1] or None; h0: [n, N] or None.
    Returns (out[n, L], h_out[n, N], hist_out[n, K-1]) in float64."""
    x, z, B, C, dt_raw = map(_f64, (x, z, B, C, dt_raw))
    conv_w, conv_b, w_dt, dt_bias, A_log, D, hist, h0 = map(_f64, (conv_w, conv_b, w_dt, dt_bias, A_log, D, hist, h0))
    bidx = np.ascontiguousarray(np.asarray(bidx, dtype=np.int64))
    n, L = x.shape
    N, K = A_log.shape[1], conv_w.shape[1]
    assert z.shape == (n, L) and B.shape[1:] == (L, N) and C.shape == B.shape and dt_raw.shape == B.shape[:2]
    assert bidx.shape == (n,) and (n == 0 or (bidx.min() >= 0 and bidx.max() < B.shape[0]))
    out = np.empty((n, max(L, 1)))
    h_out = np.empty((n, N))
    hist_out = np.empty((n, max(K - 1, 1)))
    _load().oracle_channels(n, L, N, K, _DISC[disc], float(lo), float(hi), _ptr(x), _ptr(z), _ptr(B), _ptr(C), _ptr(dt_raw),
                            _ptr(bidx), _ptr(conv_w), _ptr(conv_b), _ptr(w_dt), _ptr(dt_bias), _ptr(A_log), _ptr(D),
                            _ptr(hist), _ptr(h0), _ptr(out), _ptr(h_out), _ptr(hist_out), int(threads))
    return out[:, :L], h_out, hist_out[:, : K - 1]


def conv_silu(x, conv_w, conv_b, hist=None, threads=0):
    """u = SiLU(causal_conv(x)) of n channels. x: [n, L]; conv_w: [n, K];
    conv_b: [n]; hist: [n, K-1] or None (zeros). Returns u [n, L]."""
    x, conv_w, conv_b, hist = map(_f64, (x, conv_w, conv_b, hist))
    n, L = x.shape
    K = conv_w.shape[1]
    u = np.empty((n, max(L, 1)))
    _load().oracle_conv_silu_channels(n, L, K, _ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(hist), _ptr(u), int(threads))
    return u[:, :L]


def block(hidden, W_in, W_x, W_out, conv_w, conv_b, w_dt, dt_bias, A_log, D, hist=None, h0=None, lo=1e-4, hi=1.0,
          disc="euler", threads=0):
    """The AxonSSMBlock forward of "Axon-SSM: selective state space model",
    "Algorithm" diagram, in float64:

      x, z   = split(hidden @ W_in^T)           in_proj (D -> 2E), x first, no bias
      u      = SiLU(conv1d(x))                   depthwise causal conv, K = 4
      B, C, dt_raw = split(u @ W_x^T)            x_proj (E -> 2N + 1), in that order, no bias
      y      = scan core (channels(): dt_proj + softplus + clip, the scan, D skip, y * SiLU(z))
      out    = y @ W_out^T                       out_proj (E -> D), no bias

    hidden: [b, L, D]; W_in: [2E, D]; W_x: [2N + 1, E]; W_out: [D, E]
    (projection weights are [out_features, in_features]); the scan-core
    parameters as in channels() but per channel [E, ...]; hist: [b, K-1, E] or
    None; h0: [b, E, N] or None. The matrix products are library matmuls (a
    plain step each). Returns (out [b, L, D], h_out [b, E, N], hist_out [b, K-1, E])."""
    hidden, W_in, W_x, W_out = map(_f64, (hidden, W_in, W_x, W_out))
    conv_w, conv_b, w_dt, dt_bias, A_log, D = map(_f64, (conv_w, conv_b, w_dt, dt_bias, A_log, D))
    b, L, Dm = hidden.shape
    E = W_in.shape[0] // 2
    N = A_log.shape[1]
    K = conv_w.shape[1]
    assert W_in.shape == (2 * E, Dm) and W_x.shape == (2 * N + 1, E) and W_out.shape == (Dm, E)
    xz = hidden @ W_in.T
    x, z = xz[..., :E], xz[..., E:]
    # channel-major rows (sequence s, channel e) -> row s * E + e
    xs = np.ascontiguousarray(x.transpose(0, 2, 1).reshape(b * E, L))
    zs = np.ascontiguousarray(z.transpose(0, 2, 1).reshape(b * E, L))
    tile = lambda a: np.ascontiguousarray(np.tile(a, (b,) + (1,) * (a.ndim - 1)))  # noqa: E731
    hist_rows = None if hist is None else np.ascontiguousarray(_f64(hist).transpose(0, 2, 1).reshape(b * E, K - 1))
    h0_rows = None if h0 is None else np.ascontiguousarray(_f64(h0).reshape(b * E, N))
    u = conv_silu(xs, tile(conv_w), tile(conv_b), hist_rows, threads).reshape(b, E, L).transpose(0, 2, 1)
    bcd = u @ W_x.T
    B, C, dt_raw = bcd[..., :N], bcd[..., N:2 * N], bcd[..., 2 * N]
    out, h_out, hist_out = channels(xs, zs, np.ascontiguousarray(B), np.ascontiguousarray(C),
                                    np.ascontiguousarray(dt_raw), np.repeat(np.arange(b), E), tile(conv_w),
                                    tile(conv_b), tile(w_dt), tile(dt_bias), tile(A_log), tile(D), hist=hist_rows,
                                    h0=h0_rows, lo=lo, hi=hi, disc=disc, threads=threads)
    y = out.reshape(b, E, L).transpose(0, 2, 1)
    return y @ W_out.T, h_out.reshape(b, E, N), hist_out.reshape(b, E, K - 1).transpose(0, 2, 1)


def prefill_sampled(x, z, B, C, dt_raw, conv_w, conv_b, w_dt, dt_bias, A_log, D, chans,
                    conv_cache_in=None, ssm_state_in=None, lo=1e-4, hi=1.0, disc="euler", threads=0):
    """Oracle prefill on selected channels of dense inputs.

    x, z: [b, L, E] (any row stride); B, C: [b, L, N]; dt_raw: [b, L];
    parameters [E] / [E, K] / [E, N]; conv_cache_in: [b, K-1, E] or None;
    ssm_state_in: [b, E, N] or None; chans: list of (batch, channel) pairs.
    Returns (out[n, L], state[n, N], conv_cache[n, K-1]) for those channels."""
    bs = np.array([c[0] for c in chans], dtype=np.int64)
    es = np.array([c[1] for c in chans], dtype=np.int64)

    def cols(t):  # [b, L, E] -> [n, L]
        return np.stack([_f64(t[b, :, e]) for b, e in zip(bs, es)]) if len(bs) else np.empty((0, t.shape[1]))

    hist = None if conv_cache_in is None else np.stack([_f64(conv_cache_in[b, :, e]) for b, e in zip(bs, es)])
    h0 = None if ssm_state_in is None else np.stack([_f64(ssm_state_in[b, e, :]) for b, e in zip(bs, es)])
    conv_w, conv_b, w_dt, dt_bias, A_log, D = map(_f64, (conv_w, conv_b, w_dt, dt_bias, A_log, D))
    return channels(cols(x), cols(z), B, C, dt_raw, bs, conv_w[es], conv_b[es], w_dt[es], dt_bias[es], A_log[es], D[es],
                    hist=hist, h0=h0, lo=lo, hi=hi, disc=disc, threads=threads)


def segment_summary(x, B, dt_raw, conv_w, conv_b, w_dt, dt_bias, A_log, hist=None, lo=1e-4, hi=1.0, disc="euler",
                    threads=0):
    """What one segment of a sequence hands to the segments after it, for the
    sequence-parallel prefill: the intra-chunk step of "What is the Mamba
    model?" (velog, Texnee), "chunkscan", with the segment as the chunk.

    For every sequence s and channel e of a segment of T tokens:
      h_zero[s, :, e] = the state after the segment's last token when the scan
                        starts from h = 0 (the recurrence, token by token)
      dtsum[s, e]     = sum_t dt_t, so that the segment's decay product is
                        prod_t exp(dt_t A_n) = exp(A_n * dtsum)

    x: [b, T, E]; B: [b, T, N]; dt_raw: [b, T]; parameters per channel as in
    channels(); hist: [b, K-1, E] (the raw x rows before the segment) or None.
    Returns [b, N + 1, E] in float64: h_zero in rows 0..N-1, dtsum in row N."""
    x, B, dt_raw = map(_f64, (x, B, dt_raw))
    conv_w, conv_b, w_dt, dt_bias, A_log = map(_f64, (conv_w, conv_b, w_dt, dt_bias, A_log))
    b, T, E = x.shape
    N, K = A_log.shape[1], conv_w.shape[1]
    hist = None if hist is None else _f64(hist)
    out = np.zeros((b, N + 1, E))
    for s in range(b):
        u = conv_silu(np.ascontiguousarray(x[s].T), conv_w, conv_b,
                      None if hist is None else np.ascontiguousarray(hist[s].T), threads)
        for e in range(E):
            dt = np.array([dt_of(dt_raw[s, t], w_dt[e], dt_bias[e], lo, hi) for t in range(T)])
            A = np.array([A_of(a) for a in A_log[e]])
            _, h = scan(u[e], dt, A, B[s], np.zeros((T, N)), 0.0, None, disc)
            out[s, :N, e] = h
            out[s, N, e] = dt.sum()
    return out


def segment_carry(summaries, A_log, h_init=None):
    """The state entering segment r = len(summaries): the inter-chunk step of
    "What is the Mamba model?", "chunkscan", written as the closed form of
    "Mamba/SSM basics" (molayo insights), "Technical details",
    h_t = A_t ... A_1 h_0 + sum_j (A_t ... A_{j+1}) B_j x_j, at the granularity
    of segments: segment j contributes h_zero_j and multiplies what enters it
    by P_j = exp(A * dtsum_j), so

      h_in = (prod_{j<r} P_j) h_init + sum_{j<r} (prod_{j<k<r} P_k) h_zero_j

    summaries: [r, b, N + 1, E] (segment_summary's layout); A_log: [E, N];
    h_init: [b, E, N] (the state before segment 0) or None (zeros).
    Returns h_in [b, E, N] in float64."""
    S = _f64(summaries)
    A_log = _f64(A_log)
    r, b, N1, E = S.shape  # r may be 0 (segment 0: nothing enters but h_init)
    N = N1 - 1
    A = np.array([[A_of(a) for a in row] for row in A_log])                  # [E, N]
    P = [np.exp(A[None] * S[j, :, N, :][..., None]) for j in range(r)]       # [b, E, N] each
    hz = [S[j, :, :N, :].transpose(0, 2, 1) for j in range(r)]               # [b, E, N] each
    h = np.zeros((b, E, N)) if h_init is None else _f64(h_init).copy()
    for j in range(r):
        h = h * P[j]                                                         # prod_{j<r} P_j h_init
    for j in range(r):
        term = hz[j].copy()
        for k in range(j + 1, r):
            term = term * P[k]
        h = h + term
    return h


def ssd_chunk_scan(cb, x, dt, dA_cumsum, C, prev_states, D=None):
    """Output of the Mamba-2 chunk scan, "What is the Mamba model?" (velog,
    Texnee), "chunkscan" section, in float64, for every position l of chunk c
    and head h (group g = h // (nheads / ngroups)):

      out[l] = sum_{s <= l} cb[l, s] exp(dA[l] - dA[s]) dt[s] x[s]      (intra-chunk scan)
             + exp(dA[l]) C[l] . prev_states                           (state carried into the chunk)
             + D x[l]                                                  (skip)

    cb: [b, nchunks, ngroups, cs, cs]; x: [b, L, nheads, headdim];
    dt, dA_cumsum: [b, nheads, nchunks, cs]; C: [b, L, ngroups, dstate];
    prev_states: [b, nchunks, nheads, headdim, dstate]; D: [nheads] or None.
    The contractions are library einsums (a plain step each). Returns out
    [b, L, nheads, headdim]."""
    cb, x, dt, dA_cumsum, C, prev_states = map(_f64, (cb, x, dt, dA_cumsum, C, prev_states))
    b, L, H, P = x.shape
    _, nc, G, cs, _ = cb.shape
    assert L == nc * cs and H % G == 0
    rep = H // G
    g_of = np.arange(H) // rep
    cbh = cb[:, :, g_of]                                    # [b, c, h, l, s]
    Ch = C[:, :, g_of].reshape(b, nc, cs, H, -1)            # [b, c, l, h, n]
    xc = x.reshape(b, nc, cs, H, P)                         # [b, c, s, h, p]
    seg = dA_cumsum[..., :, None] - dA_cumsum[..., None, :]  # [b, h, c, l, s]
    causal = np.tril(np.ones((cs, cs), dtype=bool))
    w = np.where(causal, cbh * np.exp(seg).transpose(0, 2, 1, 3, 4), 0.0)  # [b, c, h, l, s]
    w = w * dt.transpose(0, 2, 1, 3)[:, :, :, None, :]      # times dt[s]
    out = np.einsum("bchls,bcshp->bclhp", w, xc)
    out += np.einsum("bclhn,bchpn->bclhp", Ch, prev_states) * np.exp(dA_cumsum).transpose(0, 2, 3, 1)[..., None]
    out = out.reshape(b, L, H, P)
    if D is not None:
        out = out + _f64(D)[None, None, :, None] * x
    return out
