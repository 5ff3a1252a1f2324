"""GPU parity of the whole block forward (ssm_block_forward: the library's
tcgen05 GEMM for in_proj, the fused tcgen05 x_proj kernel, the prefill core,
the same GEMM for out_proj) against the block oracle, on seeded synthetic
inputs.

Tolerance. The GPU path stores four intermediate quantities in bf16: x and z
(the in_proj output), u (the x_proj operand), the gated core output, and the
output itself. Each RNE rounding has relative error at most 2^-9, RMS 2^-9/sqrt(3)
~ 1.1e-3, and each reaches the output about linearly (the projections average
independent errors over thousands of terms; dt enters through exp(dt A) with a
bounded factor). Four of them give ~2.3e-3 RMS, so the test allows relative L2
1e-2 on the output, the final state and the conv cache (whose rows are the
bf16-rounded in_proj output against the oracle's unrounded float64 one).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_depthwise_b200 import api
from selective_state_space_depthwise_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_BLOCK = 1e-2
PARAMS = ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def rel_l2(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def inputs(b, L, Dm, E, seed):
    w = W.Workload("blk", batch=b, seqlen=L, d_inner=E, seed=seed)
    return W.make_block_inputs(w, Dm, device="cuda")


def run_gpu(inp, **kw):
    proj = {k: inp[k] for k in api.PROJ_NAMES}
    out = api.block_forward(inp["hidden"], inp, proj, **kw)
    torch.cuda.synchronize()
    return out


def run_oracle(inp, hist=None, h0=None, hidden=None):
    f = lambda t: t.detach().double().cpu().numpy()  # noqa: E731
    return oracle.block(f(inp["hidden"] if hidden is None else hidden), f(inp["W_in"]), f(inp["W_x"]),
                        f(inp["W_out"]), *(f(inp[k]) for k in PARAMS), hist=None if hist is None else f(hist),
                        h0=None if h0 is None else f(h0))


def check(got, want, label):
    out, cc, st = got
    e = [rel_l2(out.double().cpu().numpy(), want[0]), rel_l2(st.double().cpu().numpy(), want[1]),
         rel_l2(cc.double().cpu().numpy(), want[2])]
    assert torch.isfinite(out).all(), f"{label}: non-finite output"
    assert max(e) <= TOL_BLOCK, f"{label}: rel-L2 out {e[0]:.2e} state {e[1]:.2e} cache {e[2]:.2e}"
    return e


@pytest.mark.parametrize("b,L,Dm,E", [
    (2, 300, 64, 128),   # two K chunks, ragged last token tile
    (1, 100, 48, 40),    # one partial K chunk (E < 64), fewer tokens than a tile
    (3, 129, 32, 192),   # one token past a tile
])
def test_block_small_against_the_oracle(b, L, Dm, E):
    inp = inputs(b, L, Dm, E, seed=L + E)
    e = check(run_gpu(inp), run_oracle(inp), f"block b={b} L={L} D={Dm} E={E}")
    print(f"block b={b} L={L} D={Dm} E={E}: out {e[0]:.2e} state {e[1]:.2e} cache {e[2]:.2e}")


def test_block_both_projections_cut_along_k():
    """b=1, L=64, D=128, E=1088: in_proj (64 x 2176 x 128) and out_proj
    (64 x 128 x 1088) both cut tiles along K between CTA pairs. Their tile
    counters lead the shared GEMM scratch and are zeroed once per block call;
    in_proj's completing contributors set theirs back to zero, so out_proj
    starts from zero (else out_proj's tiles would never be stored). The output
    must match the oracle and be bit-equal over repeated calls on one
    workspace, also when that workspace holds garbage (every counter -1, every
    partial NaN) before the call."""
    b, L, Dm, E = 1, 64, 128, 1088
    M = b * L
    assert api.proj_gemm_workspace_bytes(M, 2 * E, Dm) > 0 and api.proj_gemm_workspace_bytes(M, Dm, E) > 0
    inp = inputs(b, L, Dm, E, seed=17)
    ws = torch.empty(api.block_workspace_bytes(b, L, Dm, E), dtype=torch.uint8, device="cuda")
    first = run_gpu(inp, workspace=ws)
    e = check(first, run_oracle(inp), "block, both projections cut")
    print(f"block b={b} L={L} D={Dm} E={E} (both projections cut): out {e[0]:.2e} state {e[1]:.2e} cache {e[2]:.2e}")
    for i in range(3):
        again = run_gpu(inp, workspace=ws)
        assert all(torch.equal(x, y) for x, y in zip(first, again)), f"call {i + 2} differs"
    ws.fill_(0xFF)  # garbage scratch: the call zeroes the counters it needs
    again = run_gpu(inp, workspace=ws)
    assert all(torch.equal(x, y) for x, y in zip(first, again)), "block on a garbage-filled workspace differs"


def test_block_chained_calls_with_caches():
    b, L, Dm, E = 2, 260, 64, 128
    inp = inputs(b, L, Dm, E, seed=77)
    cut = 133
    h1 = inp["hidden"][:, :cut].contiguous()
    h2 = inp["hidden"][:, cut:].contiguous()
    proj = {k: inp[k] for k in api.PROJ_NAMES}
    o1, c1, s1 = api.block_forward(h1, inp, proj)
    o2, c2, s2 = api.block_forward(h2, inp, proj, conv_cache_in=c1, ssm_state_in=s1)
    torch.cuda.synchronize()
    want = run_oracle(inp)
    check((torch.cat([o1, o2], dim=1), c2, s2), want, "chained block")


def test_block_zero_length_copies_the_caches():
    inp = inputs(2, 4, 32, 64, seed=3)
    cin = (torch.randn(2, 3, 64) * 0.5).to(torch.bfloat16).cuda()
    sin = torch.randn(2, 64, 16).cuda()
    proj = {k: inp[k] for k in api.PROJ_NAMES}
    out, cc, st = api.block_forward(inp["hidden"][:, :0].contiguous(), inp, proj, conv_cache_in=cin, ssm_state_in=sin)
    torch.cuda.synchronize()
    assert out.shape == (2, 0, 32) and torch.equal(cc, cin) and torch.equal(st, sin)


def test_block_full_size_axon_layer():
    """The pages' layer shape: b=1, L=2048, D=2560, E=7680, every output."""
    w, Dm = W.BLOCK_WORKLOADS["block_axon_layer"]
    inp = W.make_block_inputs(w, Dm, device="cuda", gen_device="cuda")
    e = check(run_gpu(inp), run_oracle(inp), "block_axon_layer")
    print(f"block_axon_layer: out {e[0]:.2e} state {e[1]:.2e} cache {e[2]:.2e}")
