"""Pins of the sequence-parallel prefill oracle (oracle.segment_summary,
oracle.segment_carry): the three steps of "What is the Mamba model?" (velog,
Texnee), "chunkscan" -- intra-chunk scan, inter-chunk scan, combine -- with a
segment of the sequence as the chunk, and the closed form of "Mamba/SSM
basics" (molayo insights), "Technical details".

  Q1  invariance: summaries of segments 0..r-1, carried into segment r and
      followed by the ordinary prefill of segment r from that state (with the
      previous raw x rows as conv history), reproduce the unsplit prefill:
      outputs, final state and conv cache, for uneven segments (some shorter
      than the conv history), both discretisations, with and without initial
      caches;
  Q2  special cases of the summary: constant dt (w_dt = 0) makes dtsum = T dt;
      B = 0 leaves h_zero at 0; A -> -inf (every decay 0) leaves only the last
      token's injection; and brute force of the closed form on tiny segments;
  Q3  the carry: nothing enters segment 0 but h_init; explicit nested
      recurrences for one and three segments.

The last test restates in float64 the block decomposition the GPU summary
computes (backward walk over 256-token blocks, then an in-order fold) and
checks it against the oracle's recurrence.
"""
import math

import numpy as np
import pytest

import oracle

N = 16


def params(rng, E):
    return dict(conv_w=rng.normal(0, 0.5, (E, 4)), conv_b=rng.normal(0, 0.1, E), w_dt=rng.uniform(-1, 1, E),
                dt_bias=np.log(np.expm1(np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), E)))),
                A_log=np.tile(np.log(np.arange(1, N + 1)), (E, 1)) + rng.uniform(-0.5, 0.5, (E, N)),
                D=rng.uniform(0.5, 1.5, E))


def inputs(rng, b, L, E):
    return dict(x=rng.normal(size=(b, L, E)), z=rng.normal(size=(b, L, E)), B=rng.normal(size=(b, L, N)),
                C=rng.normal(size=(b, L, N)), dt_raw=rng.normal(size=(b, L)))


def prefill(inp, p, t0, t1, hist, h0, disc):
    """Oracle prefill of tokens [t0, t1) of every sequence and channel:
    (out [b, T, E], state [b, E, N], conv cache [b, 3, E])."""
    b, _, E = inp["x"].shape
    chans = [(s, e) for s in range(b) for e in range(E)]
    sl = {k: (v[:, t0:t1] if k != "dt_raw" else v[:, t0:t1]) for k, v in inp.items()}
    out, h, hc = oracle.prefill_sampled(sl["x"], sl["z"], sl["B"], sl["C"], sl["dt_raw"], p["conv_w"], p["conv_b"],
                                        p["w_dt"], p["dt_bias"], p["A_log"], p["D"], chans, conv_cache_in=hist,
                                        ssm_state_in=h0, disc=disc)
    T = t1 - t0
    return (out.reshape(b, E, T).transpose(0, 2, 1), h.reshape(b, E, N), hc.reshape(b, E, 3).transpose(0, 2, 1))


def history_before(x, t0, hist0):
    """The 3 raw x rows before token t0 ([b, 3, E]): rows of x, then of the
    initial cache hist0 (or zeros) where t0 < 3."""
    b, _, E = x.shape
    full = np.concatenate([np.zeros((b, 3, E)) if hist0 is None else hist0, x], axis=1)
    return full[:, t0:t0 + 3]


@pytest.mark.parametrize("disc", ["euler", "zoh"])
@pytest.mark.parametrize("with_init", [False, True])
def test_Q1_segments_carried_reproduce_the_unsplit_prefill(disc, with_init):
    rng = np.random.default_rng(11 + with_init)
    b, E = 2, 8
    lens = [13, 1, 2, 20, 14, 7]
    L = sum(lens)
    p = params(rng, E)
    inp = inputs(rng, b, L, E)
    hist0 = rng.normal(size=(b, 3, E)) if with_init else None
    h_init = rng.normal(size=(b, E, N)) if with_init else None
    want_out, want_h, want_hc = prefill(inp, p, 0, L, hist0, h_init, disc)
    starts = np.concatenate([[0], np.cumsum(lens)])
    summaries = []
    outs = []
    for r, (t0, t1) in enumerate(zip(starts[:-1], starts[1:])):
        hist = history_before(inp["x"], t0, hist0)
        h_in = oracle.segment_carry(np.array(summaries).reshape(r, b, N + 1, E), p["A_log"], h_init)
        out, h, hc = prefill(inp, p, t0, t1, hist, h_in, disc)
        outs.append(out)
        summaries.append(oracle.segment_summary(inp["x"][:, t0:t1], inp["B"][:, t0:t1], inp["dt_raw"][:, t0:t1],
                                                p["conv_w"], p["conv_b"], p["w_dt"], p["dt_bias"], p["A_log"],
                                                hist=hist, disc=disc))
    np.testing.assert_allclose(np.concatenate(outs, axis=1), want_out, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(h, want_h, rtol=1e-11, atol=1e-13)
    np.testing.assert_array_equal(hc, want_hc)
    # and the last segment's summary carried once more is the final state
    h_end = oracle.segment_carry(np.array(summaries), p["A_log"], h_init)
    np.testing.assert_allclose(h_end, want_h, rtol=1e-11, atol=1e-13)


def softplus(v):
    return max(v, 0.0) + math.log1p(math.exp(-abs(v)))


def test_Q2_constant_dt_sums_exactly():
    rng = np.random.default_rng(21)
    b, T, E = 2, 37, 5
    p = params(rng, E)
    p["w_dt"][:] = 0.0
    p["dt_bias"] = np.array([-12.0, -3.0, 0.0, 0.3, 5.0])  # below lo, inside, above hi
    inp = inputs(rng, b, T, E)
    S = oracle.segment_summary(inp["x"], inp["B"], inp["dt_raw"], p["conv_w"], p["conv_b"], p["w_dt"], p["dt_bias"],
                               p["A_log"])
    for e in range(E):
        dt = min(max(softplus(p["dt_bias"][e]), 1e-4), 1.0)
        np.testing.assert_allclose(S[:, N, e], T * dt, rtol=1e-13)


def test_Q2_zero_B_leaves_zero_state():
    rng = np.random.default_rng(22)
    b, T, E = 2, 29, 4
    p = params(rng, E)
    inp = inputs(rng, b, T, E)
    S = oracle.segment_summary(inp["x"], np.zeros_like(inp["B"]), inp["dt_raw"], p["conv_w"], p["conv_b"],
                               p["w_dt"], p["dt_bias"], p["A_log"], hist=rng.normal(size=(b, 3, E)))
    assert np.all(S[:, :N] == 0.0)


def silu(v):
    return v / (1.0 + math.exp(-v))


def u_at(x, hist, w, cb, t):
    """SiLU of the causal conv at token t of one channel, written out."""
    xh = list(hist) + list(x)
    return silu(cb + sum(w[k] * xh[t + k] for k in range(4)))


@pytest.mark.parametrize("disc", ["euler", "zoh"])
def test_Q2_no_memory_keeps_only_the_last_injection(disc):
    rng = np.random.default_rng(23)
    b, T, E = 1, 9, 3
    p = params(rng, E)
    p["A_log"][:] = 40.0  # A = -e^40: exp(dt A) = 0 for every dt >= 1e-4
    inp = inputs(rng, b, T, E)
    hist = rng.normal(size=(b, 3, E))
    S = oracle.segment_summary(inp["x"], inp["B"], inp["dt_raw"], p["conv_w"], p["conv_b"], p["w_dt"], p["dt_bias"],
                               p["A_log"], hist=hist, disc=disc)
    for e in range(E):
        u = u_at(inp["x"][0, :, e], hist[0, :, e], p["conv_w"][e], p["conv_b"][e], T - 1)
        dt = min(max(softplus(inp["dt_raw"][0, -1] * p["w_dt"][e] + p["dt_bias"][e]), 1e-4), 1.0)
        A = -math.exp(p["A_log"][e, 0])
        scale = dt if disc == "euler" else (math.exp(dt * A) - 1.0) / A
        np.testing.assert_allclose(S[0, :N, e], scale * inp["B"][0, -1] * u, rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("disc", ["euler", "zoh"])
def test_Q2_brute_force_closed_form(disc):
    rng = np.random.default_rng(24)
    b, T, E = 1, 6, 2
    p = params(rng, E)
    inp = inputs(rng, b, T, E)
    hist = rng.normal(size=(b, 3, E))
    S = oracle.segment_summary(inp["x"], inp["B"], inp["dt_raw"], p["conv_w"], p["conv_b"], p["w_dt"], p["dt_bias"],
                               p["A_log"], hist=hist, disc=disc)
    for e in range(E):
        dts = [min(max(softplus(inp["dt_raw"][0, t] * p["w_dt"][e] + p["dt_bias"][e]), 1e-4), 1.0) for t in range(T)]
        us = [u_at(inp["x"][0, :, e], hist[0, :, e], p["conv_w"][e], p["conv_b"][e], t) for t in range(T)]
        for n in range(N):
            A = -math.exp(p["A_log"][e, n])
            h = 0.0
            for j in range(T):  # h_T = sum_j exp(A * sum_{i>j} dt_i) * inj_j
                inj = (dts[j] if disc == "euler" else (math.exp(dts[j] * A) - 1.0) / A) * inp["B"][0, j, n] * us[j]
                h += math.exp(A * sum(dts[j + 1:])) * inj
            np.testing.assert_allclose(S[0, n, e], h, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(S[0, N, e], sum(dts), rtol=1e-14)


def test_Q3_nothing_enters_segment_zero_but_the_initial_state():
    rng = np.random.default_rng(31)
    b, E = 2, 3
    A_log = rng.uniform(-1, 2, (E, N))
    h0 = rng.normal(size=(b, E, N))
    empty = np.zeros((0, b, N + 1, E))
    np.testing.assert_array_equal(oracle.segment_carry(empty, A_log, h0), h0)
    np.testing.assert_array_equal(oracle.segment_carry(empty, A_log), np.zeros((b, E, N)))


def test_Q3_nested_recurrence_over_segments():
    rng = np.random.default_rng(32)
    b, E = 2, 3
    A_log = rng.uniform(-1, 2, (E, N))
    h0 = rng.normal(size=(b, E, N))
    summ = rng.normal(size=(3, b, N + 1, E))
    summ[:, :, N] = rng.uniform(0.0, 3.0, (3, b, E))  # dt sums are positive
    for r in (1, 3):
        got = oracle.segment_carry(summ[:r], A_log, h0)
        for s in range(b):
            for e in range(E):
                for n in range(N):
                    A = -math.exp(A_log[e, n])
                    h = h0[s, e, n]
                    for j in range(r):  # h <- exp(A dtsum_j) h + h_zero_j
                        h = math.exp(A * summ[j, s, N, e]) * h + summ[j, s, n, e]
                    assert got[s, e, n] == pytest.approx(h, rel=1e-13, abs=1e-15)


def test_block_decomposition_of_the_summary_matches_the_recurrence():
    """The segment summary as the kernels compute it, restated in float64:
    256-token blocks, each walked backwards with R = the dt mass after the
    token, h_blk = sum_t exp(A R_t) dt_t B_t u_t, then the blocks folded in
    order, h <- exp(A tot_k) h + h_blk_k. It must equal the oracle's token-by-
    token recurrence (a different algorithm), here for a segment of 3 blocks
    with a ragged last one."""
    rng = np.random.default_rng(41)
    b, T, E = 1, 600, 3
    p = params(rng, E)
    inp = inputs(rng, b, T, E)
    hist = rng.normal(size=(b, 3, E))
    want = oracle.segment_summary(inp["x"], inp["B"], inp["dt_raw"], p["conv_w"], p["conv_b"], p["w_dt"],
                                  p["dt_bias"], p["A_log"], hist=hist)
    xh = np.concatenate([hist, inp["x"]], axis=1)[0]  # raw rows, token t at t + 3
    blk = 256
    for e in range(E):
        u = [silu(p["conv_b"][e] + sum(p["conv_w"][e, k] * xh[t + k, e] for k in range(4))) for t in range(T)]
        dt = [min(max(softplus(inp["dt_raw"][0, t] * p["w_dt"][e] + p["dt_bias"][e]), 1e-4), 1.0) for t in range(T)]
        A = -np.exp(p["A_log"][e])
        h = np.zeros(N)
        dtsum = 0.0
        for t0 in range(0, T, blk):
            hb = np.zeros(N)
            R = 0.0
            for t in range(min(T, t0 + blk) - 1, t0 - 1, -1):  # backwards through the block
                hb += np.exp(A * R) * dt[t] * inp["B"][0, t] * u[t]
                R += dt[t]
            h = np.exp(A * R) * h + hb  # fold: R is now the block's dt total
            dtsum += R
        np.testing.assert_allclose(h, want[0, :N, e], rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(dtsum, want[0, N, e], rtol=1e-13)
