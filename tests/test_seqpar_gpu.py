"""GPU parity of the sequence-parallel prefill: ssm_segment_summary and
ssm_segment_carry against oracle.segment_summary / oracle.segment_carry, and
the whole path (summaries, carries, per-segment prefill; seqpar.prefill_segments
on one device) against the unsplit oracle prefill, element by element, up to
the long-context workload cut into 8 segments.

Tolerances: the summary and the carry are fp32 arithmetic on exactly stored
inputs, so they are held to rel-L2 1e-5 at every io dtype; the path's outputs
to the prefill tolerances (1e-5 fp32 io, 2e-3 bf16 io) and the conv cache bit
for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import TOL, all_channels, compare, compare_full, format_report, gather, oracle_prefill, rel_l2
from selective_state_space_depthwise_b200 import api, seqpar
from selective_state_space_depthwise_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL_SUMMARY = 1e-5
N = 16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def small(io_dtype, b=2, L=300, E=72, seed=41):
    return W.Workload("seg", batch=b, seqlen=L, d_inner=E, io_dtype=io_dtype, seed=seed)


def np64(t):
    return None if t is None else t.detach().to("cpu").double().numpy()


def oracle_summary(inp, t0, t1, hist, disc="euler"):
    return oracle.segment_summary(np64(inp["x"][:, t0:t1]), np64(inp["B"][:, t0:t1]), np64(inp["dt_raw"][:, t0:t1]),
                                  np64(inp["conv_w"]), np64(inp["conv_b"]), np64(inp["w_dt"]), np64(inp["dt_bias"]),
                                  np64(inp["A_log"]), hist=np64(hist), disc=disc)


def check_summary(got, want, label):
    got = np64(got)
    e_h = rel_l2(got[:, :N], want[:, :N])
    e_s = rel_l2(got[:, N], want[:, N])
    assert np.isfinite(got).all(), f"{label}: non-finite summary"
    assert e_h <= TOL_SUMMARY and e_s <= TOL_SUMMARY, f"{label}: h_zero {e_h:.2e}, dtsum {e_s:.2e}"
    return e_h, e_s


@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("disc", ["euler", "zoh"])
@pytest.mark.parametrize("t0,t1", [(0, 300), (0, 128), (5, 6), (7, 9), (100, 233), (0, 0)])
def test_summary_matches_oracle(io_dtype, disc, t0, t1):
    """Segments of one, two, 128 (half of one 256-token block), 300 (a whole
    block and a ragged second) and other ragged lengths; E = 72 leaves a ragged
    128-channel group; history from the tokens before the segment (or zeros at
    the start)."""
    w = small(io_dtype)
    inp = W.make_inputs(w, device="cuda")
    full = torch.cat([torch.zeros((w.batch, 3, w.d_inner), dtype=io_dtype, device="cuda"), inp["x"]], dim=1)
    hist = None if t0 == 0 else full[:, t0:t0 + 3].contiguous()
    got = api.segment_summary(inp["x"][:, t0:t1], inp["B"][:, t0:t1], inp["dt_raw"][:, t0:t1], inp, conv_cache_in=hist,
                              discretization=disc)
    torch.cuda.synchronize()
    want = oracle_summary(inp, t0, t1, hist, disc)
    if t1 == t0:
        assert np.all(np64(got) == 0.0)
    else:
        check_summary(got, want, f"summary {disc} [{t0}, {t1})")


@pytest.mark.parametrize("count", [0, 1, 3])
@pytest.mark.parametrize("with_init", [False, True])
def test_carry_matches_oracle(count, with_init):
    g = torch.Generator().manual_seed(51 + count)
    b, E = 3, 40
    w = small(torch.float32, b=b, E=E)
    p = W.make_inputs(w, device="cuda")
    summ = torch.randn((count, b, N + 1, E), generator=g)
    summ[:, :, N] = torch.rand((count, b, E), generator=g) * 4.0
    h0 = torch.randn((b, E, N), generator=g) if with_init else None
    got = api.segment_carry(summ.cuda(), p, ssm_state_in=None if h0 is None else h0.cuda())
    torch.cuda.synchronize()
    want = oracle.segment_carry(summ.double().numpy(), np64(p["A_log"]), None if h0 is None else h0.double().numpy())
    if count == 0 and not with_init:
        assert np.all(np64(got) == 0.0)
    else:
        assert rel_l2(np64(got), want) <= TOL_SUMMARY


def test_carry_in_place():
    g = torch.Generator().manual_seed(57)
    b, E = 2, 24
    p = W.make_inputs(small(torch.float32, b=b, E=E), device="cuda")
    summ = torch.randn((2, b, N + 1, E), generator=g)
    summ[:, :, N] = torch.rand((2, b, E), generator=g)
    h = torch.randn((b, E, N), generator=g)
    want = oracle.segment_carry(summ.double().numpy(), np64(p["A_log"]), h.double().numpy())
    hd = h.cuda()
    api.segment_carry(summ.cuda(), p, ssm_state_in=hd, out=hd)
    torch.cuda.synchronize()
    assert rel_l2(np64(hd), want) <= TOL_SUMMARY


@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("disc", ["euler", "zoh"])
@pytest.mark.parametrize("with_init", [False, True])
def test_segments_path_matches_unsplit_oracle(io_dtype, disc, with_init):
    """seqpar.prefill_segments on the GPU (summary, carry and prefill kernels
    per segment, segments of 2, 0, 1 and ragged lengths) against one oracle
    prefill of the whole sequence."""
    w = small(io_dtype, L=700, E=72)
    inp = W.make_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(61)
    init = {}
    if with_init:
        init = dict(conv_cache_in=torch.randn((w.batch, 3, w.d_inner), generator=g, device="cuda").to(io_dtype),
                    ssm_state_in=torch.randn((w.batch, w.d_inner, N), generator=g, device="cuda"))
    bounds = [0, 2, 2, 3, 260, 517, 700]
    y, cc, st = seqpar.prefill_segments(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp, bounds,
                                        discretization=disc, **init)
    torch.cuda.synchronize()
    chans = all_channels(w.batch, w.d_inner)
    compare(io_dtype, gather(y, cc, st, chans), oracle_prefill(inp, chans, disc=disc, **init),
            label=f"segments {disc}")


def test_full_size_long_context_in_eight_segments():
    """The long-context workload (b = 1, L = 65536, E = 7680, bf16) cut into 8
    segments of 8192 tokens, as 8 GPUs would hold it, against the oracle on
    every channel; and segment 0's summary against the oracle's on sampled
    channels."""
    w = W.WORKLOADS["long_context"]
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    L = w.seqlen
    bounds = [L * r // 8 for r in range(9)]
    y, cc, st = seqpar.prefill_segments(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp, bounds)
    torch.cuda.synchronize()
    rep = compare_full(w.io_dtype, inp, (y, cc, st), label="long_context in 8 segments")
    print(f"long_context / 8 segments: {format_report(rep)}")

    T = bounds[1]
    summ = api.segment_summary(inp["x"][:, :T], inp["B"][:, :T], inp["dt_raw"][:, :T], inp)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    es = np.sort(rng.choice(w.d_inner, 48, replace=False))
    sub = {k: inp[k][es.tolist()] for k in ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log")}
    sub.update(x=inp["x"][:, :, es.tolist()], B=inp["B"], dt_raw=inp["dt_raw"])
    want = oracle_summary(sub, 0, T, None)
    check_summary(summ[:, :, es.tolist()], want, "long_context segment 0 summary")
