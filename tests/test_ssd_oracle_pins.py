"""Pins of the chunk-scan oracle (oracle.ssd_chunk_scan): the output formula of
"What is the Mamba model?" (velog, Texnee), "chunkscan" section.

  S1  duality: with cb = C B^T (one group per head here or shared), dA_cumsum =
      the within-chunk cumulative sum of dt A_h (a scalar A per head) and
      prev_states = the recurrent state entering each chunk, the chunk-scan
      output equals the plain sequential scan h_t = exp(dt_t A_h) h_{t-1} +
      dt_t B_t x_t, y_t = C_t h_t + D_h x_t, run token by token in Python
      (a different algorithm: no chunks, no decay matrix);
  S2  causality: the output at position l does not change when x at later
      positions of the chunk, or cb[l, s > l], change;
  S3  special cases: prev_states = 0 and cb = 0 leave D x; dA = 0, dt = 1,
      cb = 1 (lower triangle) give the within-chunk prefix sum of x.
"""
import math

import numpy as np
import pytest

import oracle


def recurrent_reference(x, dt, A, B, C, D, h0):
    """y[b, t, h, p] by the sequential recurrence; h0 [b, h, p, n]."""
    b, L, H, P = x.shape
    N = B.shape[-1]
    y = np.zeros_like(x)
    for bb in range(b):
        for hh in range(H):
            h = h0[bb, hh].copy()  # [P, N]
            for t in range(L):
                g = B[bb, t, hh]  # per-head B/C here (ngroups = nheads) or broadcast by the caller
                h = math.exp(dt[bb, t, hh] * A[hh]) * h + dt[bb, t, hh] * np.outer(x[bb, t, hh], g)
                y[bb, t, hh] = h @ C[bb, t, hh] + D[hh] * x[bb, t, hh]
    return y


@pytest.mark.parametrize("G", [1, 2])
def test_S1_chunk_scan_equals_the_sequential_recurrence(G):
    rng = np.random.default_rng(10 + G)
    b, H, P, N, cs, nc = 2, 4, 3, 5, 6, 3
    L = cs * nc
    x = rng.normal(size=(b, L, H, P))
    dt = rng.uniform(0.01, 0.3, size=(b, L, H))
    A = -rng.uniform(0.5, 2.0, size=H)
    Bg = rng.normal(size=(b, L, G, N))
    Cg = rng.normal(size=(b, L, G, N))
    D = rng.uniform(0.5, 1.5, size=H)
    h_init = rng.normal(size=(b, H, P, N)) * 0.3
    g_of = np.arange(H) // (H // G)
    Bh, Ch = Bg[:, :, g_of], Cg[:, :, g_of]
    y_ref = recurrent_reference(x, dt, A, Bh, Ch, D, h_init)
    # chunk-scan inputs derived from the same model
    cb = np.einsum("bclgn,bcsgn->bcgls", Cg.reshape(b, nc, cs, G, N), Bg.reshape(b, nc, cs, G, N))
    dtc = dt.reshape(b, nc, cs, H).transpose(0, 3, 1, 2)                  # [b, h, c, cs]
    dA = np.cumsum(dtc * A[None, :, None, None], axis=-1)                 # within-chunk cumulative sum
    prev = np.zeros((b, nc, H, P, N))
    h = h_init.copy()
    for c in range(nc):                                                  # states entering each chunk
        prev[:, c] = h
        for t in range(c * cs, (c + 1) * cs):
            h = np.exp(dt[:, t, :, None, None] * A[None, :, None, None]) * h + \
                dt[:, t, :, None, None] * x[:, t, :, :, None] * Bh[:, t, :, None, :]
    y = oracle.ssd_chunk_scan(cb, x, dtc, dA, Cg, prev, D)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-12)


def test_S2_causality():
    rng = np.random.default_rng(3)
    b, H, P, N, cs, nc, G = 1, 2, 3, 4, 8, 2, 1
    L = cs * nc
    args = dict(cb=rng.normal(size=(b, nc, G, cs, cs)), x=rng.normal(size=(b, L, H, P)),
                dt=rng.uniform(0.01, 0.2, size=(b, H, nc, cs)), C=rng.normal(size=(b, L, G, N)),
                prev_states=rng.normal(size=(b, nc, H, P, N)), D=rng.normal(size=H))
    args["dA_cumsum"] = np.cumsum(-args["dt"], axis=-1)
    y = oracle.ssd_chunk_scan(**args)
    l = 4  # position inside chunk 0
    x2 = args["x"].copy()
    x2[:, l + 1:cs] += 5.0                 # later positions of the same chunk
    cb2 = args["cb"].copy()
    cb2[:, :, :, l, l + 1:] += 7.0         # the upper triangle of row l
    y2 = oracle.ssd_chunk_scan(**{**args, "x": x2, "cb": cb2})
    np.testing.assert_array_equal(y2[:, :l + 1], y[:, :l + 1])
    assert not np.allclose(y2[:, l + 1:cs], y[:, l + 1:cs])


def test_S3_special_cases():
    rng = np.random.default_rng(4)
    b, H, P, N, cs, nc, G = 2, 3, 4, 2, 5, 3, 1
    L = cs * nc
    x = rng.normal(size=(b, L, H, P))
    C = rng.normal(size=(b, L, G, N))
    D = rng.uniform(0.5, 1.5, size=H)
    zero_dt = np.zeros((b, H, nc, cs))
    y = oracle.ssd_chunk_scan(np.zeros((b, nc, G, cs, cs)), x, zero_dt + 0.1, zero_dt, C,
                              np.zeros((b, nc, H, P, N)), D)
    np.testing.assert_allclose(y, D[None, None, :, None] * x, rtol=1e-15, atol=0)
    y = oracle.ssd_chunk_scan(np.ones((b, nc, G, cs, cs)), x, zero_dt + 1.0, zero_dt, C,
                              np.zeros((b, nc, H, P, N)), None)
    want = np.cumsum(x.reshape(b, nc, cs, H, P), axis=2).reshape(b, L, H, P)
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-13)
