"""CPU checks of bench.py's host logic: the ALU roofline bounds against their
closed forms, the algorithmic bytes of one long-context prefill, and the
reference arm's JSON line (the oracle on the host cores), which must carry the
GPU arm's metric string and the keys the benchmark contract asks for."""
import importlib.util
import json
import os
import subprocess
import sys

from selective_state_space_depthwise_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_alu_bounds_match_their_closed_forms():
    """With S SFU-class and F FP32 operations per channel-token, k of the
    SFU evaluations may move to an 8-operation FMA polynomial; the bound is
    148 SMs x clock / min_k max((S - k) / 16, (F + 8 k) / 128). Where the two
    pipes balance, 128 (S - k) = 16 (F + 8 k): k = (8 S - F) / 16."""
    b = load_bench()
    clk = 148 * 1965e6
    # per-state (22, 84): k = 5.75, 1.015625 clocks a channel-token per SM
    assert abs(b.alu_peak_ct_per_s(1965.0, "per_state") / (clk / ((22 - 5.75) / 16)) - 1) < 1e-9
    # powers (6, 83): the FMA pipe binds with no SFU work moved (k = 0)
    assert abs(b.alu_peak_ct_per_s(1965.0, "power") / (clk / (83 / 128)) - 1) < 1e-9
    # zero-order hold (22, 132): k = 2.75
    assert abs(b.alu_peak_ct_per_s(1965.0, "zoh") / (clk / ((22 - 2.75) / 16)) - 1) < 1e-9


def test_algorithmic_bytes_of_the_long_context_prefill():
    """x and z read and y written once (bf16), B and C (fp32, 16 each) and
    dt_raw read once, the per-channel parameters and both caches: 3.03 GB."""
    b = load_bench()
    w = W.WORKLOADS["long_context"]
    assert b.min_bytes_prefill(w) == 3029824512
    per_ct = b.min_bytes_prefill(w) / (w.batch * w.seqlen * w.d_inner)
    assert 6.0 < per_ct < 6.1  # 3 x 2 bytes plus the shared and per-channel terms


def test_reference_arm_prints_the_contract_line():
    b = load_bench()
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == b.METRIC  # the GPU arm prints the same string, so the two can be compared
    assert line["unit"] == "channel-tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "channel-tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["seq_len"] == 65536 and line["config"]["d_inner"] == 7680
