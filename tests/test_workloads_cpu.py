"""CPU checks of the input recipe (workloads.py): the documented parameter
distributions, the stated A initialisation, the long-context workload's
clip-stressed channels, and that the draws are deterministic and agree with
the helper that names the stressed channels."""
import math

import torch

from selective_state_space_depthwise_b200 import workloads as W


def softplus(v):
    return torch.nn.functional.softplus(v.double())


def test_long_context_parameters_follow_the_recipe():
    w = W.WORKLOADS["long_context"]
    p = W.make_params(w)
    E = w.d_inner
    # conv_w ~ N(0, variance 0.25): the sample std of 4 E draws within 4 standard errors
    std = float(p["conv_w"].std())
    assert abs(std - 0.5) < 4 * 0.5 / math.sqrt(2 * 4 * E)
    assert abs(float(p["conv_w"].mean())) < 4 * 0.5 / math.sqrt(4 * E)
    assert torch.all(p["conv_b"] == 0) and torch.all(p["D"] == 1)
    # w_dt ~ U(-1, 1)
    assert float(p["w_dt"].min()) >= -1.0 and float(p["w_dt"].max()) <= 1.0
    assert abs(float(p["w_dt"].mean())) < 4 / math.sqrt(3 * E)
    # A_log[e, n] = ln(n + 1): A = -1 .. -16 on every channel
    A = -torch.exp(p["A_log"].double())
    assert torch.allclose(A, -torch.arange(1, 17, dtype=torch.float64).expand(E, 16), rtol=1e-6, atol=0)


def test_long_context_clip_stress_channels():
    """5% of channels at softplus^-1(1e-4) = -9.21029 and 5% at
    softplus^-1(1.0) = 0.541325; every other channel's softplus(dt_bias) in
    [1e-3, 1e-1] (log-uniform)."""
    w = W.WORKLOADS["long_context"]
    p = W.make_params(w)
    lo, hi = W.clip_stress_channels(w)
    assert len(lo) == len(hi) == w.d_inner // 20 == 384
    assert not set(lo.tolist()) & set(hi.tolist())
    assert torch.allclose(p["dt_bias"][lo].double(), torch.full((384,), -9.210290, dtype=torch.float64), atol=1e-5)
    assert torch.allclose(p["dt_bias"][hi].double(), torch.full((384,), 0.541325, dtype=torch.float64), atol=1e-5)
    assert torch.allclose(softplus(p["dt_bias"][lo]), torch.full((384,), 1e-4, dtype=torch.float64), rtol=1e-4)
    assert torch.allclose(softplus(p["dt_bias"][hi]), torch.ones(384, dtype=torch.float64), rtol=1e-6)
    rest = torch.ones(w.d_inner, dtype=torch.bool)
    rest[lo] = False
    rest[hi] = False
    d = softplus(p["dt_bias"][rest])
    assert float(d.min()) >= 1e-3 * (1 - 1e-5) and float(d.max()) <= 1e-1 * (1 + 1e-5)
    # log-uniform: the median of log d sits near the middle of [ln 1e-3, ln 1e-1]
    assert abs(float(torch.log(d).median()) - math.log(1e-2)) < 0.15


def test_unstressed_workloads_have_no_stress_channels():
    for name in ("tiny", "axon_layer", "batched", "decode"):
        lo, hi = W.clip_stress_channels(W.WORKLOADS[name])
        assert len(lo) == 0 and len(hi) == 0


def test_draws_are_deterministic_and_typed():
    w = W.Workload("t", batch=2, seqlen=40, d_inner=24, seed=9, decode_steps=3)
    a, b = W.make_inputs(w), W.make_inputs(w)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert a["x"].dtype == a["z"].dtype == torch.bfloat16 and a["x"].shape == (2, 43, 24)
    assert a["B"].dtype == a["C"].dtype == a["dt_raw"].dtype == torch.float32
    assert a["B"].shape == (2, 43, 16) and a["dt_raw"].shape == (2, 43)
    # another seed gives other draws
    c = W.make_inputs(w.scaled(seed=10))
    assert not torch.equal(a["x"], c["x"]) and not torch.equal(a["conv_w"], c["conv_w"])
    # a fused in_proj row stride keeps the channel block and adds filler columns
    f = W.make_inputs(w.scaled(x_row_stride=48))
    assert f["x"].shape == (2, 43, 48)
