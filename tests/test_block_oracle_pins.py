"""Pins of the block oracle (oracle.block): the AxonSSMBlock forward of
"Axon-SSM: selective state space model", "Algorithm" diagram (in_proj, conv1d,
SiLU, x_proj -> B, C, dt_raw, dt_proj + softplus + clip, scan, y * SiLU(z),
out_proj). The scan core under it is pinned in test_oracle_pins.py; these
tests pin the composition: which half of in_proj feeds the conv, the order of
x_proj's outputs, the orientation of every weight, and the cache carry.

  B1  special case: B = C = 0 (x_proj's first 2N rows zero) leaves the state at
      zero, so the core output is D * u * SiLU(z) and the block output is its
      out_proj image; written out with explicit loops;
  B2  index mappings: permutation matrices as in_proj / out_proj and one-hot
      x_proj rows turn the block into the pinned core on permuted inputs;
  B3  brute force on tiny sizes: the whole block with the scan in its unrolled
      closed form h_t = sum_j (prod_{i>j} dA_i) dt_j B_j u_j (a different
      algorithm from the oracle's recurrence), plain Python floats;
  B4  invariance: two calls chained through the caches equal one call.
"""
import math

import numpy as np
import pytest

import oracle

N = 16


def params(rng, E, N=N):
    return dict(conv_w=rng.normal(0, 0.5, (E, 4)), conv_b=rng.normal(0, 0.1, E), w_dt=rng.uniform(-1, 1, E),
                dt_bias=np.log(np.expm1(np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), E)))),
                A_log=np.tile(np.log(np.arange(1, N + 1)), (E, 1)), D=rng.uniform(0.5, 1.5, E))


def run_block(hidden, W_in, W_x, W_out, p, **kw):
    return oracle.block(hidden, W_in, W_x, W_out, p["conv_w"], p["conv_b"], p["w_dt"], p["dt_bias"], p["A_log"],
                        p["D"], **kw)


def silu(v):
    return v / (1.0 + math.exp(-v))


def test_B1_zero_B_and_C_rows_leave_D_u_gate():
    rng = np.random.default_rng(1)
    b, L, Dm, E = 2, 9, 5, 4
    p = params(rng, E)
    hidden = rng.normal(size=(b, L, Dm))
    W_in = rng.normal(0, 0.4, (2 * E, Dm))
    W_x = rng.normal(0, 0.4, (2 * N + 1, E))
    W_x[:2 * N] = 0.0  # B = C = 0; dt_raw row kept (dt no longer matters)
    W_out = rng.normal(0, 0.4, (Dm, E))
    out, h, hist = run_block(hidden, W_in, W_x, W_out, p)
    want = np.zeros((b, L, Dm))
    for s in range(b):
        for t in range(L):
            y = []
            for e in range(E):
                x = [sum(W_in[e, d] * hidden[s, tt, d] for d in range(Dm)) if tt >= 0 else 0.0
                     for tt in range(t - 3, t + 1)]
                z = sum(W_in[E + e, d] * hidden[s, t, d] for d in range(Dm))
                c = p["conv_b"][e] + sum(p["conv_w"][e, k] * x[k] for k in range(4))
                y.append(p["D"][e] * silu(c) * silu(z))
            for d in range(Dm):
                want[s, t, d] = sum(W_out[d, e] * y[e] for e in range(E))
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-14)
    assert np.all(h == 0.0)
    x_last = np.einsum("ld,ed->le", hidden[:, -3:].reshape(-1, Dm), W_in[:E]).reshape(b, 3, E)
    np.testing.assert_allclose(hist, x_last, rtol=1e-13, atol=1e-15)  # raw x rows of the last 3 tokens


def test_B2_permutations_and_one_hot_x_proj_reduce_to_the_core():
    rng = np.random.default_rng(2)
    b, L, E = 2, 11, 6
    Dm = E
    p = params(rng, E)
    hidden = rng.normal(size=(b, L, Dm))
    P, Q, R = (np.eye(E)[rng.permutation(E)] for _ in range(3))
    W_in = np.concatenate([P, 0.5 * Q])          # x = hidden[..., perm_P], z = 0.5 * hidden[..., perm_Q]
    a, c = rng.integers(0, E, N), rng.integers(0, E, N)
    d = int(rng.integers(0, E))
    W_x = np.zeros((2 * N + 1, E))
    W_x[np.arange(N), a] = 1.0                    # B_n = u[a_n]
    W_x[N + np.arange(N), c] = 1.0                # C_n = u[c_n]
    W_x[2 * N, d] = 1.0                           # dt_raw = u[d]
    out, h, hist = run_block(hidden, W_in, W_x, R, p)
    x = hidden @ P.T
    z = 0.5 * (hidden @ Q.T)
    u = np.stack([oracle.conv_silu(x[s].T, p["conv_w"], p["conv_b"]).T for s in range(b)])  # [b, L, E]
    B, C, dt_raw = u[..., a], u[..., c], u[..., d]
    rows = [(s, e) for s in range(b) for e in range(E)]
    y, h_c, hist_c = oracle.channels(np.stack([x[s, :, e] for s, e in rows]), np.stack([z[s, :, e] for s, e in rows]),
                                     B, C, dt_raw, [s for s, _ in rows], np.tile(p["conv_w"], (b, 1)),
                                     np.tile(p["conv_b"], b), np.tile(p["w_dt"], b), np.tile(p["dt_bias"], b),
                                     np.tile(p["A_log"], (b, 1)), np.tile(p["D"], b))
    y = y.reshape(b, E, L).transpose(0, 2, 1)
    np.testing.assert_allclose(out, y @ R.T, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(h, h_c.reshape(b, E, N), rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(hist, hist_c.reshape(b, E, 3).transpose(0, 2, 1))


def brute_block(hidden, W_in, W_x, W_out, p, n_state, lo=1e-4, hi=1.0):
    """The block on one sequence in plain Python, the scan in unrolled form."""
    L, Dm = len(hidden), len(hidden[0])
    E = len(W_in) // 2
    x = [[sum(W_in[e][d] * hidden[t][d] for d in range(Dm)) for e in range(E)] for t in range(L)]
    z = [[sum(W_in[E + e][d] * hidden[t][d] for d in range(Dm)) for e in range(E)] for t in range(L)]
    u = [[silu(p["conv_b"][e] + sum(p["conv_w"][e][k] * (x[t + k - 3][e] if t + k - 3 >= 0 else 0.0)
                                    for k in range(4))) for e in range(E)] for t in range(L)]
    bcd = [[sum(W_x[o][e] * u[t][e] for e in range(E)) for o in range(2 * n_state + 1)] for t in range(L)]
    out = []
    for t in range(L):
        y = []
        for e in range(E):
            def dt_of(j):
                v = bcd[j][2 * n_state] * p["w_dt"][e] + p["dt_bias"][e]
                return min(max(math.log1p(math.exp(v)), lo), hi)
            acc = 0.0
            for n in range(n_state):
                A = -math.exp(p["A_log"][e][n])
                h = 0.0
                for j in range(t + 1):  # h_t = sum_j exp(A * sum_{i=j+1..t} dt_i) * dt_j * B_j * u_j
                    decay = math.exp(A * sum(dt_of(i) for i in range(j + 1, t + 1)))
                    h += decay * dt_of(j) * bcd[j][n] * u[j][e]
                acc += bcd[t][n_state + n] * h
            y.append((acc + p["D"][e] * u[t][e]) * silu(z[t][e]))
        out.append([sum(W_out[d][e] * y[e] for e in range(E)) for d in range(Dm)])
    return out


@pytest.mark.parametrize("n_state", [1, 3])
def test_B3_brute_force_tiny_block(n_state):
    rng = np.random.default_rng(3 + n_state)
    L, Dm, E = 5, 3, 2
    p = params(rng, E, n_state)
    p["A_log"] = rng.uniform(-1, 1, (E, n_state))
    hidden = rng.normal(size=(1, L, Dm))
    W_in, W_x, W_out = rng.normal(0, 0.6, (2 * E, Dm)), rng.normal(0, 0.6, (2 * n_state + 1, E)), rng.normal(
        0, 0.6, (Dm, E))
    out, _, _ = run_block(hidden, W_in, W_x, W_out, p)
    want = brute_block(hidden[0].tolist(), W_in.tolist(), W_x.tolist(), W_out.tolist(),
                       {k: v.tolist() for k, v in p.items()}, n_state)
    np.testing.assert_allclose(out[0], np.array(want), rtol=1e-11, atol=1e-13)


def test_B4_chained_calls_equal_one_call():
    rng = np.random.default_rng(4)
    b, L, Dm, E = 2, 40, 7, 5
    p = params(rng, E)
    hidden = rng.normal(size=(b, L, Dm))
    W_in, W_x, W_out = rng.normal(0, 0.4, (2 * E, Dm)), rng.normal(0, 0.4, (2 * N + 1, E)), rng.normal(0, 0.4, (Dm, E))
    full, h_full, hist_full = run_block(hidden, W_in, W_x, W_out, p)
    cut = 17
    a, h1, hist1 = run_block(hidden[:, :cut], W_in, W_x, W_out, p)
    b2, h2, hist2 = run_block(hidden[:, cut:], W_in, W_x, W_out, p, hist=hist1, h0=h1)
    np.testing.assert_allclose(np.concatenate([a, b2], axis=1), full, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(h2, h_full, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(hist2, hist_full)
