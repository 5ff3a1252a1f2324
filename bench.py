"""Benchmark of the selective-scan block core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one prefill (conv, SiLU, dt, discretisation, scan, D skip, gate,
final state and conv cache) over one batch of the workload, inputs resident in
HBM. Default workload: long-context prefill, b=1, L=65536, E=7680, N=16, K=4,
bf16 x/z/y, fp32 B/C/dt_raw/state (3 GB of inputs: larger than L2, so no
flush is needed between steps). The JSON line also carries the decode
workload (prompt 512, then 1024 one-token steps at b=256, E=7680), the
roofline of the dominant kernel, the oracle timed on the host cores, and an
end-to-end figure through the API with host buffers.

The default launch takes the power decay path (the workloads use the pages'
A initialisation, A_n = (n+1) A_0); the line also reports the per-state path
on the same inputs (decay_paths) and the layer-shape and batched workloads
(configs).

With N > 1 (torchrun, one process per GPU) every rank runs its own independent
sequence of the workload (batch sharding: weak scaling, no collective on the
data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_depthwise_b200 import workloads as W  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
PROFILES = os.path.join(ROOT, "profiles")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# The headline metric, printed identically by both arms (the benchmark's stated metric).
METRIC = "selective-scan channel-tokens/s; achieved HBM GB/s vs B200 peak"

# SM resources used to derive the ALU roofline (B200, sm_100a): 148 SMs,
# 16 SFU lanes and 128 FP32 lanes per SM per clock (the SFU and FFMA rates
# were confirmed by a throughput probe on this GPU model).
SMS, SFU_PER_CLK, FMA_PER_CLK = 148, 16, 128
# Algorithmic work per channel-token, by decay path:
#  per-state exponentials: 16 exp (dA) + 2 sigmoid (exp + reciprocal) + 1
#    softplus (exp + log1p) = 22 SFU-class evaluations; 4 FP32 ops per state
#    (dt*A, dt*u*B, h FMA, readout FMA) + ~20 scalar ops = 84 FP32-pipe ops;
#  powers (A_n = (n+1) A_0): 1 exp (q) + 2 sigmoid + 1 softplus = 6 SFU-class
#    evaluations; 15 multiplies for q^2..q^16, then 3 FP32 ops per state
#    (dt*u*B, h FMA, readout FMA) + ~20 scalar ops = 83 FP32-pipe ops;
#  zero-order hold: the per-state SFU work (22); 7 FP32 ops per state (dt*A,
#    e^{dt A} - 1, times 1/A, times u, times B, h FMA, readout FMA) + ~20
#    scalar ops = 132 FP32-pipe ops.
ALU_MODEL = {"per_state": (22, 84), "power": (6, 83), "zoh": (22, 132)}
POLY_EXP_FMA_OPS = 8


def alu_peak_ct_per_s(sm_mhz: float, path: str = "per_state") -> float:
    """Best channel-tokens/s the SM pipes allow for the path's algorithmic
    work, when k of its SFU evaluations may move to an FMA-pipe polynomial
    (~8 FP32 ops each): minimise max((S-k)/16, (F+8k)/128) clocks per
    channel-token per SM."""
    sfu, fma = ALU_MODEL[path]
    best = math.inf
    for i in range(0, 100 * sfu + 1):
        k = i / 100.0
        best = min(best, max((sfu - k) / SFU_PER_CLK, (fma + POLY_EXP_FMA_OPS * k) / FMA_PER_CLK))
    return SMS * sm_mhz * 1e6 / best


def min_bytes_prefill(w: W.Workload) -> float:
    """Algorithmic bytes of one prefill: read x, z, B, C, dt_raw and the
    parameters once, write y, the final state and conv cache once."""
    io = 2 if w.io_dtype == torch.bfloat16 else 4
    b, L, E, N = w.batch, w.seqlen, w.d_inner, w.d_state
    act = b * L * E * io * 3 + b * L * (2 * N + 1) * 4
    params = E * (4 + 1 + 1 + 1 + N + 1) * 4
    caches = b * E * N * 4 + b * 3 * E * io
    return float(act + params + caches)


def min_bytes_decode_step(w: W.Workload) -> float:
    """One decode step: state read + write, cache read + write, x, z, y, B, C,
    dt_raw, parameters."""
    io = 2 if w.io_dtype == torch.bfloat16 else 4
    b, E, N = w.batch, w.d_inner, w.d_state
    return float(2 * b * E * N * 4 + 2 * b * 3 * E * io + 3 * b * E * io + b * (2 * N + 1) * 4
                 + E * (4 + 1 + 1 + 1 + N + 1) * 4)


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_bf16_peak() -> float:
    """Measured dense bf16 GEMM throughput (burst), else the fallback figure."""
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return FALLBACK_BF16_TFLOPS


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # The raw samples go to SSM_CLOCKS_DIR (default: the system temp directory); the
        # bench line carries their summary.
        out_dir = os.environ.get("SSM_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_gpu{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# Device sources of each kernel (its own file and the device headers it includes).
KERNEL_SOURCES = {
    "prefill": ("prefill.cu", "ssm_math.cuh", "sm100_ptx.cuh"),
    "decode": ("decode.cu", "ssm_math.cuh", "sm100_ptx.cuh"),
    "ssd": ("ssd.cu", "ssm_math.cuh", "sm100_ptx.cuh", "tma_map.cuh"),
    "gemm": ("gemm.cu", "sm100_ptx.cuh", "tma_map.cuh"),
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_depthwise_b200", "csrc")
    for n in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, n), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(PROFILES, "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t[f"{kernel}:{workload}"]
        if e.get("source_hash") != kernel_source_hash(kernel):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def step_config(w: W.Workload, world: int) -> dict:
    """The `config` of the step workload, the same in both arms' lines."""
    return {"workload": f"{w.name}: {w.note}; b={w.batch} L={w.seqlen} E={w.d_inner} N=16 K=4",
            "batch": w.batch, "seq_len": w.seqlen, "d_inner": w.d_inner, "d_state": 16, "d_conv": 4,
            "parallelism": (f"dp{world}: one independent sequence of the workload per GPU (batch sharding, "
                            f"no collective)") if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (no flush)" if min_bytes_prefill(w) > 126e6 else "inputs fit in L2"}


# ----------------------------------------------------------------- oracle ---
def cpu_baseline(w: W.Workload, target_s: float = 10.0):
    """The oracle, as it stands, on the host cores: n channels of sequence 0
    over the workload's full length, n sized for about `target_s` of wall time."""
    import oracle

    oracle.build()
    params = W.make_params(w)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    L, N = w.seqlen, w.d_state
    threads = oracle.max_threads()

    def run(n):
        x = torch.randn((n, L), generator=g).to(w.io_dtype).double().numpy()
        z = torch.randn((n, L), generator=g).to(w.io_dtype).double().numpy()
        B = torch.randn((1, L, N), generator=g).double().numpy()
        C = torch.randn((1, L, N), generator=g).double().numpy()
        dt = torch.randn((1, L), generator=g).double().numpy()
        e = slice(0, n)
        p = {k: v[e].double().numpy() for k, v in params.items()}
        t0 = time.perf_counter()
        oracle.channels(x, z, B, C, dt, [0] * n, p["conv_w"], p["conv_b"], p["w_dt"], p["dt_bias"], p["A_log"],
                        p["D"], lo=w.dt_min, hi=w.dt_max, threads=threads)
        return time.perf_counter() - t0

    cal_n = max(threads, 1)
    cal = run(cal_n)
    n = int(min(w.d_inner, max(cal_n, cal_n * target_s / max(cal, 1e-3))))
    n = max(threads, (n // threads) * threads)
    dt_s = run(n)
    return {"value": n * L / dt_s, "unit": "channel-tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} channels x L={L} of the {w.name} workload, float64, OpenMP over channels",
            "seconds": round(dt_s, 3)}


def cpu_single_core(w: W.Workload, target_s: float = 4.0):
    """The oracle on ONE host core over n channels of the workload (its full
    length), n sized for about `target_s`."""
    import oracle

    oracle.build()
    params = W.make_params(w)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    L, N = w.seqlen, w.d_state

    def run(n):
        x = torch.randn((n, L), generator=g).to(w.io_dtype).double().numpy()
        z = torch.randn((n, L), generator=g).to(w.io_dtype).double().numpy()
        B = torch.randn((1, L, N), generator=g).double().numpy()
        C = torch.randn((1, L, N), generator=g).double().numpy()
        dt = torch.randn((1, L), generator=g).double().numpy()
        p = {k: v[:n].double().numpy() for k, v in params.items()}
        t0 = time.perf_counter()
        oracle.channels(x, z, B, C, dt, [0] * n, p["conv_w"], p["conv_b"], p["w_dt"], p["dt_bias"], p["A_log"],
                        p["D"], lo=w.dt_min, hi=w.dt_max, threads=1)
        return time.perf_counter() - t0

    cal = run(4)
    n = int(min(w.d_inner, max(4, 4 * target_s / max(cal, 1e-3))))
    dt_s = run(n)
    return {"value": n * L / dt_s, "unit": "channel-tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} channels x L={L} of the {w.name} workload, float64, one core",
            "seconds": round(dt_s, 3)}


# ------------------------------------------------------------------- GPU ---
def make_device_inputs(w: W.Workload, rank: int):
    wr = w.scaled(seed=w.seed + 1000 * rank) if rank else w
    return W.make_inputs(wr, device="cuda", gen_device="cuda")


def timed_prefill(inp, steps, warmup, dist, tuning=None, clocks=True, disc="euler"):
    from selective_state_space_depthwise_b200 import api

    args = (inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp)
    y, cc, st = api.prefill(*args, tuning=tuning, discretization=disc)
    for _ in range(warmup):
        api.prefill(*args, y=y, conv_cache_out=cc, ssm_state_out=st, tuning=tuning, discretization=disc)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) if clocks else _NoClock() as clk:
        ev0.record(stream)
        for _ in range(steps):
            api.prefill(*args, y=y, conv_cache_out=cc, ssm_state_out=st, tuning=tuning, discretization=disc)
        ev1.record(stream)
        torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    ms = ev0.elapsed_time(ev1)
    return ms, clk.summary()


class _NoClock:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False

    def summary(self):
        return None


def prefill_figures(w: W.Workload, ms_step: float, hbm_peak: float, peak_kind: str, path: str) -> dict:
    """ct/s, the HBM fraction and the ALU fraction (against the path's own
    algorithmic bound at 1965 MHz) of one prefill of `w` taking ms_step."""
    ct = w.batch * w.seqlen * w.d_inner
    gbs = min_bytes_prefill(w) / (ms_step * 1e-3) / 1e9
    peak_ct = alu_peak_ct_per_s(1965.0, path)
    return {"ms_per_step": round(ms_step, 4), "value": ct / (ms_step * 1e-3), "unit": "channel-tokens/s",
            "alu": {"achieved": ct / (ms_step * 1e-3), "peak": peak_ct, "frac": round(ct / (ms_step * 1e-3) / peak_ct, 4),
                    "path": path},
            "hbm": {"achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
                    "peak_kind": peak_kind, "algorithmic_bytes_per_launch": min_bytes_prefill(w)}}


def decay_path_bench(w: W.Workload, inp, hbm_peak: float, peak_kind: str, steps: int = 10, warmup: int = 3,
                     zoh: bool = False):
    """The same workload on each decay path (and, with zoh, the zero-order-hold
    discretisation), CUDA events, inputs resident."""
    out = {}
    runs = [("power", "power", None, "euler"), ("per_state", "per_state", {"decay_path": 1}, "euler")]
    if zoh:
        runs.append(("zoh", "zoh", None, "zoh"))
    for name, path, tun, disc in runs:
        ms, _ = timed_prefill(inp, steps, warmup, False, tuning=tun, clocks=False, disc=disc)
        out[name] = prefill_figures(w, ms / steps, hbm_peak, peak_kind, path)
    out["note"] = ("power: decays as powers of q = exp(dt A_0), taken automatically by every CTA whose channels "
                   "have A_n = (n+1) A_0 (the workloads' A initialisation); per_state: one exponential per state "
                   "(forced with decay_path = 1; the path for any other A)" +
                   ("; zoh: zero-order-hold discretisation (per-state exponentials)" if zoh else ""))
    return out


def config_bench(name: str, hbm_peak: float, peak_kind: str, steps: int = 20, warmup: int = 3):
    """Another prefill workload of the pages' shapes (parity config), both decay paths."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    res = {"workload": f"{w.name}: {w.note}; b={w.batch} L={w.seqlen} E={w.d_inner} N=16 K=4"}
    res.update(decay_path_bench(w, inp, hbm_peak, peak_kind, steps, warmup))
    res.pop("note")
    del inp
    torch.cuda.empty_cache()
    return res


def e2e_prefill(w: W.Workload, inp, steps):
    """Same metric through the public API with host buffers: every step hands
    the step's inputs in pinned host memory to ssm_prefill_host, which copies
    them in chunk by chunk, runs the kernels and copies y back with the copies
    overlapped; the final caches are then read back to the host as well."""
    from selective_state_space_depthwise_b200 import api

    names = ("x", "z", "B", "C", "dt_raw")
    host = {k: inp[k].to("cpu").pin_memory() for k in names}
    params = {k: inp[k] for k in ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")}
    b, L, E = w.batch, w.seqlen, w.d_inner
    y_h = torch.empty((b, L, E), dtype=w.io_dtype).pin_memory()
    cc = torch.empty((b, 3, E), dtype=w.io_dtype, device="cuda")
    st = torch.empty((b, E, 16), dtype=torch.float32, device="cuda")
    cc_h = torch.empty(cc.shape, dtype=cc.dtype).pin_memory()
    st_h = torch.empty(st.shape, dtype=st.dtype).pin_memory()
    ws = torch.empty(api.host_workspace_bytes(b, L, E, w.io_dtype), dtype=torch.uint8, device="cuda")
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = y_h.numel() * y_h.element_size() + cc.numel() * cc.element_size() + st.numel() * st.element_size()

    def step():
        api.prefill_host(host["x"], host["z"], host["B"], host["C"], host["dt_raw"], params, y=y_h,
                         conv_cache_out=cc, ssm_state_out=st, workspace=ws)
        cc_h.copy_(cc, non_blocking=True)
        st_h.copy_(st, non_blocking=True)

    step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / steps
    return {"value": b * L * E / (ms * 1e-3), "unit": "channel-tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "path": ("ssm_prefill_host: 4096-token chunks (the last 4096 tokens as quarters), H2D / kernel / D2H "
                     "overlapped on three streams")}


def decode_bench(w: W.Workload, rank: int, hbm_peak: float, peak_kind: str):
    """Prompt prefill (untimed), then the workload's one-token steps, each a
    separate C call; per-step device time from CUDA events. The same loop
    replayed from a CUDA graph is reported beside it (graph_us_per_step)."""
    from selective_state_space_depthwise_b200 import api

    inp = make_device_inputs(w, rank)
    L0, steps = w.seqlen, w.decode_steps
    pre = {**inp, **{k: inp[k][:, :L0] for k in ("x", "z", "B", "C", "dt_raw")}}
    _, cc, st = api.prefill(pre["x"], pre["z"], pre["B"], pre["C"], pre["dt_raw"], pre)
    y = torch.empty((w.batch, w.d_inner), dtype=w.io_dtype, device="cuda")
    cc0, st0 = cc.clone(), st.clone()

    def step(t):
        api.decode_step(inp["x"][:, t], inp["z"][:, t], inp["B"][:, t], inp["C"][:, t], inp["dt_raw"][:, t], inp,
                        cc, st, y=y)

    for t in range(L0, L0 + 8):  # warm-up on the first tokens, then restore the caches
        step(t)
    cc.copy_(cc0)
    st.copy_(st0)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for t in range(L0, L0 + steps):
        step(t)
    ev1.record(stream)
    torch.cuda.synchronize()
    us = ev0.elapsed_time(ev1) * 1e3 / steps
    # The same steps captured once in a CUDA graph and replayed: no host work between launches.
    graph = torch.cuda.CUDAGraph()
    cc.copy_(cc0)
    st.copy_(st0)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        for t in range(L0, L0 + steps):
            step(t)
    cc.copy_(cc0)
    st.copy_(st0)
    graph.replay()  # warm
    cc.copy_(cc0)
    st.copy_(st0)
    torch.cuda.synchronize()
    ev0.record(stream)
    graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    graph_us = ev0.elapsed_time(ev1) * 1e3 / steps
    del graph
    ct = w.batch * w.d_inner
    gbs = min_bytes_decode_step(w) / (us * 1e-6) / 1e9
    return {"workload": f"decode b={w.batch} E={w.d_inner} N=16 K=4 bf16 x/z/y, fp32 state; prompt {L0}, "
                        f"{steps} one-token steps",
            "us_per_step": round(us, 2), "graph_us_per_step": round(graph_us, 2),
            "value": ct / (us * 1e-6), "unit": "channel-tokens/s",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4), "peak_kind": peak_kind,
                         "traffic": ncu_traffic("decode", "decode"),
                         "algorithmic_bytes_per_launch": min_bytes_decode_step(w)},
            "gpu_launches": steps}


def block_bench(name: str, bf16_peak: float, steps: int = 10, warmup: int = 3):
    """The whole block forward (ssm_block_forward) on device-resident inputs:
    ms per call by CUDA events, tokens/s, and the projections' tensor FLOPs
    (in_proj 2E*D, x_proj 33*E, out_proj D*E per token, x2) per second against
    the measured bf16 GEMM peak."""
    from selective_state_space_depthwise_b200 import api

    w, d_model = W.BLOCK_WORKLOADS[name]
    inp = W.make_block_inputs(w, d_model, device="cuda", gen_device="cuda")
    proj = {k: inp[k] for k in api.PROJ_NAMES}
    b, L, E = w.batch, w.seqlen, w.d_inner
    out = torch.empty((b, L, d_model), dtype=torch.bfloat16, device="cuda")
    cc = torch.empty((b, 3, E), dtype=torch.bfloat16, device="cuda")
    st = torch.empty((b, E, 16), dtype=torch.float32, device="cuda")
    ws = torch.empty(api.block_workspace_bytes(b, L, d_model, E), dtype=torch.uint8, device="cuda")

    def call():
        api.block_forward(inp["hidden"], inp, proj, out=out, conv_cache_out=cc, ssm_state_out=st, workspace=ws)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        call()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / steps
    tokens = b * L
    flops = 2.0 * tokens * (2 * E * d_model + 33 * E + d_model * E)
    tflops = flops / (ms * 1e-3) / 1e12
    return {"workload": f"{name}: {w.note}; b={b} L={L} D={d_model} E={E}", "ms_per_step": round(ms, 4),
            "value": tokens / (ms * 1e-3), "unit": "tokens/s", "steps": steps,
            "projections": {"tflops": round(tflops, 1), "peak": bf16_peak, "unit": "TFLOP/s",
                            "frac": round(tflops / bf16_peak, 4), "flops_per_step": flops,
                            "note": "GEMM FLOPs of in_proj, x_proj and out_proj over the whole block time "
                                    "(the scan core's SFU-bound time is included in the denominator)"},
            "gpu_launches_per_step": 4,
            "note": "in_proj and out_proj are this library's tcgen05 GEMM; no library GEMM runs"}


def gemm_bench(bf16_peak: float, steps: int = 20, warmup: int = 3):
    """The block's two projection GEMMs (ssm_proj_gemm, tcgen05) timed alone
    at the layer shape (2048 tokens, D = 2560, E = 7680) and at the
    long-context block's 65536 tokens: us per call by CUDA events, TFLOP/s
    against the measured dense bf16 peak (burst: each is timed alone)."""
    from selective_state_space_depthwise_b200 import api

    D, E = 2560, 7680
    out = []
    for M in (2048, 65536):
        for name, N, K in (("in_proj", 2 * E, D), ("out_proj", D, E)):
            g = torch.Generator(device="cuda").manual_seed(M + N)
            A = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
            Wt = (torch.randn((N, K), device="cuda", generator=g) * K ** -0.5).to(torch.bfloat16)
            C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            for _ in range(warmup):
                api.proj_gemm(A, Wt, out=C)
            torch.cuda.synchronize()
            stream = torch.cuda.current_stream()
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for _ in range(steps):
                api.proj_gemm(A, Wt, out=C)
            ev1.record(stream)
            torch.cuda.synchronize()
            us = ev0.elapsed_time(ev1) * 1e3 / steps
            tflops = 2.0 * M * N * K / (us * 1e-6) / 1e12
            out.append({"gemm": name, "M": M, "N": N, "K": K, "us": round(us, 2), "tflops": round(tflops, 1),
                        "peak": bf16_peak, "frac": round(tflops / bf16_peak, 4)})
            del A, Wt, C
    torch.cuda.empty_cache()
    return out


def ssd_bench(name: str, hbm_peak: float, bf16_peak: float, steps: int = 20, warmup: int = 3, spec_over=None):
    """The Mamba-2 chunk scan on device-resident inputs: us per call by CUDA
    events; HBM roofline on the algorithmic bytes (read cb, x, dt, dA_cumsum, C,
    prev_states, D once, write out once) and the tensor FLOPs of the two
    contractions (2 cs cs P + 2 cs N P per chunk and head). spec_over replaces
    fields of the named workload (another built chunk length or state dim)."""
    from selective_state_space_depthwise_b200 import api

    spec = dict(W.SSD_WORKLOADS[name], **(spec_over or {}))
    inp = W.make_ssd_inputs(spec, device="cuda")
    args = [inp[k] for k in ("cb", "x", "dt", "dA_cumsum", "C", "prev_states", "D")]
    out = torch.empty_like(inp["x"])
    for _ in range(warmup):
        api.ssd_chunk_scan(*args, out=out)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        api.ssd_chunk_scan(*args, out=out)
    ev1.record(stream)
    torch.cuda.synchronize()
    us = ev0.elapsed_time(ev1) * 1e3 / steps
    b, L, H, P, G, N, cs = (spec[k] for k in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate",
                                             "chunk_size"))
    nc = L // cs
    nbytes = sum(t.numel() * t.element_size() for t in args) + out.numel() * out.element_size()
    flops = 2.0 * b * nc * H * (cs * cs * P + cs * N * P)
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"workload": f"{name}: b={b} L={L} heads={H} headdim={P} groups={G} dstate={N} chunk={cs}",
            "us_per_step": round(us, 2), "value": b * L * H / (us * 1e-6), "unit": "token-heads/s",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4), "algorithmic_bytes_per_launch": nbytes,
                         "tensor_tflops": round(flops / (us * 1e-6) / 1e12, 1), "tensor_peak": bf16_peak,
                         "traffic": ncu_traffic("ssd", name)},
            "gpu_launches_per_step": 1}


def seqpar_bench(w: W.Workload, R: int = 8, reps: int = 10):
    """The sequence-parallel prefill on one GPU: the workload cut into R
    segments as R GPUs would hold it. Times, by CUDA events, the segment
    summary (segment 1), the carry of R-1 summaries, one segment's prefill from
    its carried state, and the whole path run segment after segment on this
    GPU. The per-rank kernel time of a middle rank (summary + carry + prefill)
    gives the R-GPU figure without the exchange, which this box cannot time;
    the exchanged bytes are reported."""
    from selective_state_space_depthwise_b200 import api, seqpar

    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    b, L, E = w.batch, w.seqlen, w.d_inner
    T = L // R
    bounds = [T * r for r in range(R)] + [L]
    x1, B1, d1 = inp["x"][:, T:2 * T], inp["B"][:, T:2 * T], inp["dt_raw"][:, T:2 * T]
    halo = inp["x"][:, T - 3:T].contiguous()
    ws = torch.empty(api.segment_summary_workspace_bytes(b, T, E, w.io_dtype), dtype=torch.uint8, device="cuda")
    summ = torch.empty((b, 17, E), dtype=torch.float32, device="cuda")
    summaries = torch.stack([api.segment_summary(inp["x"][:, bounds[r]:bounds[r + 1]], inp["B"][:, bounds[r]:bounds[r + 1]],
                                                 inp["dt_raw"][:, bounds[r]:bounds[r + 1]], inp,
                                                 conv_cache_in=None if r == 0 else
                                                 inp["x"][:, bounds[r] - 3:bounds[r]].contiguous())
                             for r in range(R - 1)]).contiguous()
    h_in = torch.empty((b, E, 16), dtype=torch.float32, device="cuda")
    r_last = R - 1
    xs, zs = inp["x"][:, bounds[r_last]:], inp["z"][:, bounds[r_last]:]
    Bs, Cs, ds = inp["B"][:, bounds[r_last]:], inp["C"][:, bounds[r_last]:], inp["dt_raw"][:, bounds[r_last]:]
    halo_last = inp["x"][:, bounds[r_last] - 3:bounds[r_last]].contiguous()
    y = torch.empty((b, L - bounds[r_last], E), dtype=w.io_dtype, device="cuda")
    cc = torch.empty((b, 3, E), dtype=w.io_dtype, device="cuda")
    st = torch.empty((b, E, 16), dtype=torch.float32, device="cuda")

    def t_us(fn, n=reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / n

    us_sum = t_us(lambda: api.segment_summary(x1, B1, d1, inp, conv_cache_in=halo, summary=summ, workspace=ws))
    us_carry = t_us(lambda: api.segment_carry(summaries, inp, out=h_in))
    us_pre = t_us(lambda: api.prefill(xs, zs, Bs, Cs, ds, inp, conv_cache_in=halo_last, ssm_state_in=h_in, y=y,
                                      conv_cache_out=cc, ssm_state_out=st))
    us_path = t_us(lambda: seqpar.prefill_segments(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp, bounds),
                   n=3)
    ct_seg = b * T * E
    sfu_peak = 148 * 16 * 1965e6 / 19  # 16 decays + softplus + SiLU (exp2, rcp) per channel-token on the SFU
    per_rank = us_sum + us_carry + us_pre
    return {"workload": f"{w.name} cut into {R} segments of {T} tokens (b={b} E={E})",
            "summary_us": round(us_sum, 1), "carry_us": round(us_carry, 1), "segment_prefill_us": round(us_pre, 1),
            "one_gpu_path_ms": round(us_path / 1e3, 3),
            "summary_roofline": {"bound": "alu", "achieved": ct_seg / (us_sum * 1e-6), "peak": sfu_peak,
                                 "unit": "channel-tokens/s", "frac": round(ct_seg / (us_sum * 1e-6) / sfu_peak, 4),
                                 "peak_basis": "SFU 16 lanes/clk/SM x 148 SMs at 1965 MHz, 19 SFU ops per "
                                               "channel-token"},
            "per_rank_kernel_us": round(per_rank, 1),
            "projected_value": b * L * E / (per_rank * 1e-6), "projected_unit": "channel-tokens/s",
            "projected_note": f"{R} GPUs, each running summary + carry + its segment's prefill; the all-gathers are "
                              f"not included (one GPU here)",
            "exchange_bytes_per_rank": b * 17 * E * 4 + 3 * b * E * (2 if w.io_dtype == torch.bfloat16 else 4),
            "gpu_launches_per_rank": 2 + 1 + 1}


def seq_parallel_main(args, w: W.Workload):
    """--seq-parallel: one sequence split along L across the ranks (strong
    scaling; seqpar.prefill_sequence_parallel). Rank r holds tokens
    [L r / N, L (r + 1) / N) of the workload. A step is the whole path on every
    rank: the all-gather of the conv tails, the segment summary (ranks
    0..N-2), the all-gather of the summaries, the carry and the segment's
    prefill. Timed by CUDA events between barriers, max over ranks."""
    import datetime

    from selective_state_space_depthwise_b200 import _lib, seqpar

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29531")
    os.environ.setdefault("RANK", "0")
    os.environ.setdefault("WORLD_SIZE", "1")
    torch.cuda.set_device(local_rank)
    torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                         device_id=torch.device("cuda", local_rank))
    _lib.load()
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")  # the same seeded problem on every rank
    b, L, E = w.batch, w.seqlen, w.d_inner
    t0, t1 = L * rank // world, L * (rank + 1) // world
    seg = {k: inp[k][:, t0:t1] for k in ("x", "z", "B", "C", "dt_raw")}
    params = {k: inp[k] for k in ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")}

    lengths = [L * (r + 1) // world - L * r // world for r in range(world)]

    def step():
        return seqpar.prefill_sequence_parallel(seg["x"], seg["z"], seg["B"], seg["C"], seg["dt_raw"], params,
                                                lengths=lengths)

    for _ in range(args.warmup):
        step()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    torch.distributed.barrier()
    t = torch.tensor([ev0.elapsed_time(ev1)], device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms_step = float(t.item()) / args.steps
    clocks = clk.summary()
    torch.distributed.destroy_process_group()
    if rank != 0:
        return
    value = b * L * E / (ms_step * 1e-3)
    peak_ct = alu_peak_ct_per_s(1965.0, "power")
    per_gpu = value / world
    print(json.dumps({
        "metric": METRIC,
        "value": value, "unit": "channel-tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "f32", "io_dtype": "bf16" if w.io_dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.note}; b={b} L={L} E={E} N=16 K=4", "batch": b, "seq_len": L,
                   "d_inner": E, "parallelism": f"sp{world} (sequence segments; all-gather of conv tails and "
                                               f"segment summaries over NCCL)",
                   "l2": "inputs larger than L2 (no flush)"},
        "roofline": {"bound": "alu", "achieved": per_gpu, "peak": peak_ct, "unit": "channel-tokens/s",
                     "frac": round(per_gpu / peak_ct, 4), "traffic": None,
                     "note": "per GPU; ranks 0..N-2 also run the segment summary"},
        "gpu_launches": args.steps * (3 if world > 1 else 1),  # rank 0: summary (2) + prefill; alone: prefill
        "clocks": clocks,
        "e2e": None,
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_context", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-decode", action="store_true", help="skip the decode sub-benchmark")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the layer-shape and batched prefill sub-benchmarks")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end measurement")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-block", action="store_true",
                    help="skip the block-forward and chunk-scan sub-benchmarks")
    ap.add_argument("--no-seqpar", action="store_true", help="skip the sequence-parallel sub-benchmark")
    ap.add_argument("--seq-parallel", action="store_true",
                    help="split the workload's sequence across the ranks (strong scaling) instead of running "
                         "the same workload on every rank")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = W.WORKLOADS[args.workload]
    if w.decode_steps:
        ap.error("the step workload must be a prefill shape; the decode workload is reported alongside")

    if args.seq_parallel and args.impl == "native":
        return seq_parallel_main(args, w)

    if args.impl == "reference":
        # The oracle is the reference arm: rank 0 alone runs it on the host cores.
        if rank != 0:
            return
        per_step = []
        cb = None
        for i in range(args.warmup + args.steps):
            cb = cpu_baseline(w, target_s=2.0)
            if i >= args.warmup:
                per_step.append(cb["value"])
        value = statistics.median(per_step)
        cb["value"] = value
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": value,
                          "unit": "channel-tokens/s", "n_gpus": args.gpus, "steps": args.steps,
                          "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "f64", "data": "synthetic", "config": step_config(w, args.gpus),
                          "cpu_baseline": cb,
                          "e2e": {"value": value, "unit": "channel-tokens/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return

    dist = world > 1
    if dist:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    from selective_state_space_depthwise_b200 import _lib

    _lib.load()
    hbm_peak, peak_kind = load_peaks()

    inp = make_device_inputs(w, rank)
    ms, clocks = timed_prefill(inp, args.steps, args.warmup, dist)
    if dist:
        t = torch.tensor([ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    ms_step = ms / args.steps
    ct_step = w.batch * w.seqlen * w.d_inner
    value = ct_step * world / (ms_step * 1e-3)
    per_gpu = ct_step / (ms_step * 1e-3)
    gbs = min_bytes_prefill(w) / (ms_step * 1e-3) / 1e9
    # Every workload uses the pages' A initialisation, so the default launch
    # takes the power path in every CTA; its ALU bound is the roofline.
    peak_ct = alu_peak_ct_per_s(1965.0, "power")

    extra = {}
    # The sub-benchmarks (decay paths, configs, decode, block, GEMMs, chunk
    # scan, sequence-parallel pieces, CPU baseline) run only in a 1-GPU run:
    # with N ranks they would hold every GPU while rank 0 alone works.
    subs = world == 1
    if subs:
        extra["decay_paths"] = decay_path_bench(w, inp, hbm_peak, peak_kind, zoh=True)
    if not args.no_e2e:
        # Every rank moves its own inputs through the host path at the same time;
        # the job's time is the slowest rank's (CUDA events, max over ranks).
        if dist:
            torch.distributed.barrier()
        e2e = e2e_prefill(w, inp, steps=3)
        if dist:
            t = torch.tensor([e2e["ms_per_step"]], device="cuda")
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            e2e["ms_per_step"] = round(float(t.item()), 3)
            e2e["value"] = ct_step * world / (e2e["ms_per_step"] * 1e-3)
            e2e["h2d_bytes_per_step"] *= world
            e2e["d2h_bytes_per_step"] *= world
        extra["e2e"] = e2e
    if subs:
        del inp
        torch.cuda.empty_cache()
        if not args.no_configs:
            extra["configs"] = [config_bench(n, hbm_peak, peak_kind) for n in ("axon_layer", "batched")]
        if not args.no_decode:
            extra["decode"] = decode_bench(W.WORKLOADS["decode"], rank, hbm_peak, peak_kind)
        if not args.no_block:
            torch.cuda.empty_cache()
            bf16_peak = load_bf16_peak()
            extra["block"] = [block_bench(n, bf16_peak) for n in W.BLOCK_WORKLOADS]
            torch.cuda.empty_cache()
            extra["projection_gemms"] = gemm_bench(bf16_peak)
            torch.cuda.empty_cache()
            extra["ssd_chunk_scan"] = ssd_bench("ssd_chunk_scan", hbm_peak, bf16_peak)
            extra["ssd_chunk_scan_shapes"] = [
                ssd_bench("ssd_chunk_scan", hbm_peak, bf16_peak, spec_over={"chunk_size": cs, "dstate": ds})
                for cs, ds in ((64, 128), (256, 128), (128, 64))]
        if not args.no_seqpar:
            torch.cuda.empty_cache()
            extra["sequence_parallel"] = seqpar_bench(w)
        if not args.no_cpu:
            extra["cpu_baseline"] = cpu_baseline(w)
            extra["cpu_baseline"]["single_core_layer_shape"] = cpu_single_core(W.WORKLOADS["axon_layer"])
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    line = {
        "metric": METRIC,
        "value": value, "unit": "channel-tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "io_dtype": "bf16" if w.io_dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": step_config(w, world),
        "roofline": {"bound": "alu", "achieved": per_gpu, "peak": peak_ct, "unit": "channel-tokens/s",
                     "frac": round(per_gpu / peak_ct, 4),
                     "peak_basis": "SFU 16 + FP32 128 lanes/clk/SM x 148 SMs at 1965 MHz; the power decay path's "
                                   "algorithmic work, 6 SFU-class + 83 FP32 ops per channel-token, best SFU/FMA "
                                   "split (the per-state path's bound, 22 + 84, is in decay_paths)",
                     "traffic": ncu_traffic("prefill", w.name),
                     "hbm": {"achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(gbs / hbm_peak, 4), "peak_kind": peak_kind,
                             "algorithmic_bytes_per_launch": min_bytes_prefill(w)}},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    line.update(extra)
    print(json.dumps(line))


if __name__ == "__main__":
    main()
