"""GPU parity of the Mamba-2 chunk scan (ssm_ssd_chunk_scan, tcgen05) against
its oracle (oracle.ssd_chunk_scan) on seeded synthetic SSD inputs.

Tolerance. The kernel rounds one operand tile to bf16 for the tensor cores,
the masked, decayed scores cb exp(dA[l] - dA[s]) dt[s] (relative error at
most 2^-9, RMS ~1.1e-3; the 128-term sums average independent errors; C and
prev_states are bf16 inputs and enter exactly, exp(dA[l]) is applied in fp32),
and the output itself (RNE to bf16, ~1.1e-3). About 1.6e-3 RMS in all, so the
test allows relative L2 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_depthwise_b200 import api
from selective_state_space_depthwise_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_SSD = 1e-2
ARGS = ("cb", "x", "dt", "dA_cumsum", "C", "prev_states", "D")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def run(inp, **kw):
    out = api.ssd_chunk_scan(*(inp[k] for k in ARGS), **kw)
    torch.cuda.synchronize()
    return out


def rel_l2(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def oracle_on(inp, bs, cs_idx):
    """The oracle on sequence bs and chunk index cs_idx (all heads)."""
    cs = inp["cb"].shape[3]
    sl = slice(cs_idx * cs, (cs_idx + 1) * cs)
    f = lambda t: t.detach().double().cpu().numpy()  # noqa: E731
    return oracle.ssd_chunk_scan(f(inp["cb"][bs:bs + 1, cs_idx:cs_idx + 1]), f(inp["x"][bs:bs + 1, sl]),
                                 f(inp["dt"][bs:bs + 1, :, cs_idx:cs_idx + 1]),
                                 f(inp["dA_cumsum"][bs:bs + 1, :, cs_idx:cs_idx + 1]), f(inp["C"][bs:bs + 1, sl]),
                                 f(inp["prev_states"][bs:bs + 1, cs_idx:cs_idx + 1]), f(inp["D"]))[0]


def test_ssd_small_every_output():
    spec = W.SSD_WORKLOADS["ssd_small"]
    inp = W.make_ssd_inputs(spec, device="cuda")
    out = run(inp).double().cpu().numpy()
    f = lambda t: t.detach().double().cpu().numpy()  # noqa: E731
    want = oracle.ssd_chunk_scan(*(f(inp[k]) for k in ARGS))
    e = rel_l2(out, want)
    print(f"ssd_small: rel-L2 {e:.2e}")
    assert e <= TOL_SSD


def test_ssd_without_skip_and_zero_state():
    spec = dict(W.SSD_WORKLOADS["ssd_small"], seed=17)
    inp = W.make_ssd_inputs(spec, device="cuda")
    inp["prev_states"] = torch.zeros_like(inp["prev_states"])
    out = api.ssd_chunk_scan(*(inp[k] for k in ARGS[:-1]), None)
    torch.cuda.synchronize()
    f = lambda t: t.detach().double().cpu().numpy()  # noqa: E731
    want = oracle.ssd_chunk_scan(*(f(inp[k]) for k in ARGS[:-1]), None)
    assert rel_l2(out.double().cpu().numpy(), want) <= TOL_SSD


def test_ssd_two_groups_many_chunks():
    """b = 2, 32 chunks, 8 heads in 2 groups of 4 (each head takes its group's
    cb and C): 512 (sequence, chunk, head) units, every output against the
    oracle."""
    spec = dict(batch=2, seqlen=4096, nheads=8, headdim=64, ngroups=2, dstate=128, chunk_size=128, seed=23)
    inp = W.make_ssd_inputs(spec, device="cuda")
    out = run(inp).double().cpu().numpy()
    f = lambda t: t.detach().double().cpu().numpy()  # noqa: E731
    want = oracle.ssd_chunk_scan(*(f(inp[k]) for k in ARGS))
    e = rel_l2(out, want)
    print(f"ssd 2x4096, 8 heads, 2 groups: rel-L2 {e:.2e}")
    assert e <= TOL_SSD


def test_ssd_full_size_sampled_chunks():
    """b=8, L=4096, 80 heads: chunks of the first and last sequence and a seeded
    sample of (sequence, chunk) pairs, every head and position of each."""
    spec = W.SSD_WORKLOADS["ssd_chunk_scan"]
    inp = W.make_ssd_inputs(spec, device="cuda")
    out = run(inp)
    nc = spec["seqlen"] // spec["chunk_size"]
    rng = np.random.default_rng(0)
    picks = [(0, 0), (0, nc - 1), (spec["batch"] - 1, 0), (spec["batch"] - 1, nc - 1)]
    picks += [(int(rng.integers(spec["batch"])), int(rng.integers(nc))) for _ in range(4)]
    cs = spec["chunk_size"]
    num = den = 0.0
    for bs, c in picks:
        got = out[bs, c * cs:(c + 1) * cs].double().cpu().numpy()
        want = oracle_on(inp, bs, c)
        num += float(np.sum((got - want) ** 2))
        den += float(np.sum(want ** 2))
    e = (num / den) ** 0.5
    print(f"ssd_chunk_scan: rel-L2 {e:.2e} over {len(picks)} (sequence, chunk) pairs")
    assert e <= TOL_SSD
    assert torch.isfinite(out).all()
