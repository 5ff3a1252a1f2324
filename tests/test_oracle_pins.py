"""Pins for the CPU oracle: each test checks it against something other than
itself -- a result a page prints, a closed form, an invariant the method states,
or a library routine for a special case -- so that a dropped term, a wrong sign
or index, or a transposed operand anywhere in the oracle fails at least one.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LO, HI = 1e-4, 1.0


def silu_lib(v):
    return v * expit(v)


def softplus_lib(v):
    return np.logaddexp(0.0, v)


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split("=", 1)
                out[k] = v
    return out


def conv_kernel(A, Bv, Cv, dt, L, disc):
    """K_k = C . (Abar^k * Bbar) for a fixed diagonal SSM."""
    Abar = np.exp(dt * A)
    Bbar = (Abar - 1.0) / A * Bv if disc == "zoh" else dt * Bv
    return np.array([np.dot(Cv, Abar ** k * Bbar) for k in range(L)])


def causal_apply(Kk, u):
    """y_t = sum_{k<=t} K_k u_{t-k} (a full convolution, truncated)."""
    return np.convolve(u, Kk)[: len(u)]


# ---------------------------------------------------------------- page 4 -----
def test_printed_example_recurrence_equals_convolution():
    """The page's own fixed-parameter example: recurrence == convolution."""
    g = read_golden("ultralytics_ssm_recurrence_conv_identity.txt")
    L, N, delta, atol = int(g["L"]), int(g["N"]), float(g["delta"]), float(g["atol"])
    torch.manual_seed(int(g["seed"]))
    x = torch.randn(L).double().numpy()
    A = (-(torch.rand(N) + 0.5)).double().numpy()
    Bv = torch.randn(N).double().numpy()
    Cv = torch.randn(N).double().numpy()
    y_rec, _ = oracle.scan(x, np.full(L, delta), A, np.tile(Bv, (L, 1)), np.tile(Cv, (L, 1)), D=0.0, disc="zoh")
    y_conv = causal_apply(conv_kernel(A, Bv, Cv, delta, L, "zoh"), x)
    same = bool(np.allclose(y_rec, y_conv, atol=atol))
    assert same == (g["same_outputs"] == "True")
    np.testing.assert_allclose(y_rec, y_conv, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("disc", ["euler", "zoh"])
def test_full_channel_fixed_params_is_a_convolution(disc):
    """With w_dt = 0 (dt constant per channel) and B_t, C_t constant in t, the
    whole channel (conv -> SiLU -> dt -> scan -> D skip -> gate) reduces to
    out_t = (sum_k K_k u_{t-k} + D u_t) * SiLU(z_t)."""
    rng = np.random.default_rng(1)
    L, N, K = 96, 16, 4
    x = rng.normal(size=L)
    z = rng.normal(size=L)
    Bv, Cv = rng.normal(size=N), rng.normal(size=N)
    dt_bias, D = -3.1, 0.7
    A_log = np.log(np.arange(1, N + 1.0)) + rng.uniform(-0.3, 0.3, size=N)
    conv_w = np.array([0.0, 0.0, 0.0, 1.0])  # identity tap on the current token
    out, _, _ = oracle.channels(x[None], z[None], np.tile(Bv, (1, L, 1)), np.tile(Cv, (1, L, 1)), rng.normal(size=(1, L)),
                                [0], conv_w[None], [0.0], [0.0], [dt_bias], A_log[None], [D], lo=LO, hi=HI, disc=disc)
    u = silu_lib(x)
    dt = float(np.clip(softplus_lib(dt_bias), LO, HI))
    A = -np.exp(A_log)
    want = (causal_apply(conv_kernel(A, Bv, Cv, dt, L, disc), u) + D * u) * silu_lib(z)
    np.testing.assert_allclose(out[0], want, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- page 5 -----
def brute_force_unrolled(u, dt, A, B, C, D, h0, disc):
    """h_t = (prod_{i<=t} A_i) h_0 + sum_{j<=t} (prod_{j<i<=t} A_i) B_j x_j, per state."""
    L, N = B.shape
    y = np.zeros(L)
    hs = np.zeros((L, N))
    for t in range(L):
        for n in range(N):
            dA = [math.exp(dt[i] * A[n]) for i in range(L)]
            if disc == "zoh":
                dB = [math.expm1(dt[j] * A[n]) / A[n] * B[j, n] for j in range(L)]
            else:
                dB = [dt[j] * B[j, n] for j in range(L)]
            acc = math.prod(dA[: t + 1]) * h0[n]
            for j in range(t + 1):
                acc += math.prod(dA[j + 1: t + 1]) * dB[j] * u[j]
            hs[t, n] = acc
        y[t] = sum(C[t, n] * hs[t, n] for n in range(N)) + D * u[t]
    return y, hs[-1] if L else h0


@pytest.mark.parametrize("disc", ["euler", "zoh"])
@pytest.mark.parametrize("L", list(range(1, 9)))
def test_scan_matches_unrolled_closed_form(L, disc):
    rng = np.random.default_rng(100 + L)
    N = 5
    u = rng.normal(size=L)
    dt = rng.uniform(1e-3, 0.8, size=L)
    A = -rng.uniform(0.2, 6.0, size=N)
    B = rng.normal(size=(L, N))
    C = rng.normal(size=(L, N))
    h0 = rng.normal(size=N)
    D = 0.3
    y, h = oracle.scan(u, dt, A, B, C, D=D, h0=h0, disc=disc)
    y_bf, h_bf = brute_force_unrolled(u, dt, A, B, C, D, h0, disc)
    np.testing.assert_allclose(y, y_bf, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(h, h_bf, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- page 1 -----
def test_A_init_gives_diagonal_minus_one_to_minus_N():
    """A_log[n] = ln(n+1) must give A_n = -(n+1): recovered from the impulse
    response of the full channel, state by state."""
    L, N, K = 6, 16, 4
    dt_bias = float(np.log(np.expm1(0.05)))  # dt = 0.05
    x = np.zeros(L)
    x[0] = 1.3
    z = np.full(L, 40.0)  # SiLU(40) == 40 in double
    A_log = np.log(np.arange(1, N + 1.0))
    for n in range(N):
        Bm = np.zeros((1, L, N))
        Cm = np.zeros((1, L, N))
        Bm[0, :, n] = 1.0
        Cm[0, :, n] = 1.0
        out, _, _ = oracle.channels(x[None], z[None], Bm, Cm, np.zeros((1, L)), [0], np.array([[0, 0, 0, 1.0]]), [0.0],
                                    [0.0], [dt_bias], A_log[None], [0.0], lo=LO, hi=HI)
        y = out[0] / 40.0
        ratio = y[2] / y[1]
        A_rec = math.log(ratio) / 0.05
        assert abs(A_rec - (-(n + 1))) < 1e-9, (n, A_rec)
        assert abs(y[0] - 0.05 * silu_lib(1.3)) < 1e-15  # first output: dt * B * u


def random_channel(rng, L, N=16, K=4, n=3):
    return dict(
        x=rng.normal(size=(n, L)), z=rng.normal(size=(n, L)), B=rng.normal(size=(1, L, N)), C=rng.normal(size=(1, L, N)),
        dt_raw=rng.normal(size=(1, L)), bidx=[0] * n, conv_w=rng.normal(size=(n, K)) * 0.5, conv_b=rng.normal(size=n) * 0.1,
        w_dt=rng.uniform(-1, 1, size=n), dt_bias=np.log(np.expm1(rng.uniform(1e-3, 1e-1, size=n))),
        A_log=np.tile(np.log(np.arange(1, N + 1.0)), (n, 1)), D=rng.normal(size=n))


def run(ch, t0, t1, hist=None, h0=None, disc="euler"):
    return oracle.channels(ch["x"][:, t0:t1], ch["z"][:, t0:t1], ch["B"][:, t0:t1], ch["C"][:, t0:t1],
                           ch["dt_raw"][:, t0:t1], ch["bidx"], ch["conv_w"], ch["conv_b"], ch["w_dt"], ch["dt_bias"],
                           ch["A_log"], ch["D"], hist=hist, h0=h0, lo=LO, hi=HI, disc=disc)


@pytest.mark.parametrize("L0", [0, 1, 2, 3, 7])
def test_decode_steps_continue_the_prefill(L0):
    """Prefill of L0 tokens, then one-token calls carrying [conv_cache,
    ssm_state], must equal one prefill of L0 + k tokens."""
    rng = np.random.default_rng(7 + L0)
    k = 6
    ch = random_channel(rng, L0 + k)
    out_full, h_full, c_full = run(ch, 0, L0 + k)
    out, h, c = run(ch, 0, L0)
    outs = [out]
    for s in range(k):
        o, h, c = run(ch, L0 + s, L0 + s + 1, hist=c, h0=h)
        outs.append(o)
    np.testing.assert_array_equal(np.concatenate(outs, axis=1), out_full)
    np.testing.assert_array_equal(h, h_full)
    np.testing.assert_array_equal(c, c_full)


def test_conv_cache_holds_last_raw_rows():
    rng = np.random.default_rng(3)
    ch = random_channel(rng, 10)
    _, _, c = run(ch, 0, 10)
    np.testing.assert_array_equal(c, ch["x"][:, 7:10])
    _, _, c2 = run(ch, 0, 2)  # L < K-1: the oldest row is the zero history
    np.testing.assert_array_equal(c2[:, 0], 0.0)
    np.testing.assert_array_equal(c2[:, 1:], ch["x"][:, 0:2])
    hist = rng.normal(size=(3, 3))
    _, _, c3 = run(ch, 0, 1, hist=hist)
    np.testing.assert_array_equal(c3, np.concatenate([hist[:, 1:], ch["x"][:, 0:1]], axis=1))


def test_zero_length_returns_the_incoming_cache():
    rng = np.random.default_rng(4)
    ch = random_channel(rng, 4)
    hist, h0 = rng.normal(size=(3, 3)), rng.normal(size=(3, 16))
    out, h, c = run(ch, 0, 0, hist=hist, h0=h0)
    assert out.shape == (3, 0)
    np.testing.assert_array_equal(h, h0)
    np.testing.assert_array_equal(c, hist)


@pytest.mark.parametrize("disc", ["euler", "zoh"])
def test_chunk_split_invariance(disc):
    """The chunked walk of the scan: any split point, with the carried state
    and conv history, gives the unsplit result."""
    rng = np.random.default_rng(5)
    L = 23
    ch = random_channel(rng, L)
    out_full, h_full, c_full = run(ch, 0, L, disc=disc)
    for s in range(L + 1):
        o1, h1, c1 = run(ch, 0, s, disc=disc)
        o2, h2, c2 = run(ch, s, L, hist=c1, h0=h1, disc=disc)
        np.testing.assert_array_equal(np.concatenate([o1, o2], axis=1), out_full)
        np.testing.assert_array_equal(h2, h_full)
        np.testing.assert_array_equal(c2, c_full)


# ------------------------------------------------------- special cases -------
def test_conv_orientation_bias_and_history_against_numpy():
    rng = np.random.default_rng(6)
    L, K = 17, 4
    x, w, hist = rng.normal(size=L), rng.normal(size=K), rng.normal(size=K - 1)
    c = oracle.causal_conv(x, w, 0.25, hist=hist)
    want = np.correlate(np.concatenate([hist, x]), w, mode="valid") + 0.25
    np.testing.assert_allclose(c, want, rtol=1e-13, atol=1e-14)
    c0 = oracle.causal_conv(x, w, 0.0)
    want0 = np.convolve(x, w[::-1])[:L]  # zero history == truncated full convolution
    np.testing.assert_allclose(c0, want0, rtol=1e-13, atol=1e-14)


def test_C_zero_leaves_the_gated_skip():
    """C == 0: out = D * SiLU(conv(x)) * SiLU(z), whatever the state does."""
    rng = np.random.default_rng(8)
    L, N = 33, 16
    ch = random_channel(rng, L, n=2)
    ch["C"] = np.zeros((1, L, N))
    out, _, _ = run(ch, 0, L)
    for i in range(2):
        c = np.convolve(ch["x"][i], ch["conv_w"][i][::-1])[:L] + ch["conv_b"][i]
        want = ch["D"][i] * silu_lib(c) * silu_lib(ch["z"][i])
        np.testing.assert_allclose(out[i], want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("disc", ["euler", "zoh"])
def test_memoryless_limit_reads_dt_through_softplus_and_clip(disc):
    """A -> -inf (dA = 0): y_t = (dB u)_t . C_t + D u_t. With one-hot B, C and
    D = 0, the output exposes dt_t = clip(softplus(dt_raw * w_dt + dt_bias))
    over a range of pre-activations that crosses both clip bounds."""
    L, N = 200, 16
    raw = np.linspace(-40.0, 40.0, L)
    w_dt, dt_bias = 0.5, -2.0
    x = np.full(L, 2.0)
    z = np.full(L, 40.0)
    Bm = np.zeros((1, L, N))
    Cm = np.zeros((1, L, N))
    Bm[0, :, 3] = 1.0
    Cm[0, :, 3] = 1.0
    A_log = np.full((1, N), 40.0)  # A = -exp(40): exp(dt*A) underflows to 0
    out, _, _ = oracle.channels(x[None], z[None], Bm, Cm, raw[None], [0], np.array([[0, 0, 0, 1.0]]), [0.0], [w_dt],
                                [dt_bias], A_log, [0.0], lo=LO, hi=HI, disc=disc)
    dt_seen = out[0] / (silu_lib(2.0) * 40.0)
    if disc == "zoh":  # ZOH injection (exp(dt A) - 1)/A -> -1/A = exp(-40), whatever dt is
        np.testing.assert_allclose(dt_seen, np.exp(-40.0), rtol=1e-12)
        return
    want = np.clip(softplus_lib(raw * w_dt + dt_bias), LO, HI)
    np.testing.assert_allclose(dt_seen, want, rtol=1e-12)
    assert abs(dt_seen.min() / LO - 1) < 1e-12 and abs(dt_seen.max() / HI - 1) < 1e-12  # both bounds reached


def test_zoh_and_euler_agree_to_first_order_in_dt():
    rng = np.random.default_rng(9)
    L, N = 40, 16
    u, B, C = rng.normal(size=L), rng.normal(size=(L, N)), rng.normal(size=(L, N))
    A = -np.arange(1, N + 1.0)
    errs = []
    for dt in (1e-2, 1e-3):
        ye, _ = oracle.scan(u, np.full(L, dt), A, B, C, disc="euler")
        yz, _ = oracle.scan(u, np.full(L, dt), A, B, C, disc="zoh")
        errs.append(np.abs(ye - yz).max() / np.abs(ye).max())
    assert errs[1] < errs[0] / 5  # the gap shrinks with dt


def test_long_memory_at_the_lower_clip_is_a_discounted_prefix_sum():
    """dt == lo, A = -1: h_t = sum_j (1 - lo)^(t-j)-ish discounting; compare
    with the geometric closed form of a constant-input recurrence."""
    L, N = 500, 1
    u = np.ones(L)
    dt = np.full(L, LO)
    A = np.array([-1.0])
    B = np.ones((L, N))
    C = np.ones((L, N))
    y, h = oracle.scan(u, dt, A, B, C, D=0.0)
    a = math.exp(-LO)
    t = np.arange(1, L + 1)
    want = LO * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(y, want, rtol=1e-10)
