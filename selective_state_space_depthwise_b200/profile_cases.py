"""Small, fixed launches of the kernels for profiler captures.

    python -m selective_state_space_depthwise_b200.profile_cases prefill WORKLOAD [L] [KERNEL DECAY_PATH] [E] [DISC]
    python -m selective_state_space_depthwise_b200.profile_cases decode [BATCH]
    python -m selective_state_space_depthwise_b200.profile_cases block NAME [L]
    python -m selective_state_space_depthwise_b200.profile_cases ssd NAME
    python -m selective_state_space_depthwise_b200.profile_cases segment WORKLOAD [T]
    python -m selective_state_space_depthwise_b200.profile_cases gemm M N K

prefill: three launches of the named workload's prefill (optionally shortened
to L tokens, optionally with an explicit kernel (3, 4 or 5) and decay path (0 auto,
1 per-state exponentials), E channels and the discretisation, euler or zoh); decode: a 4-token
prompt, then three decode steps at the decode workload's shape (batch 256,
E=7680, 252 MB of state); block: three block forwards of the named block
workload (optionally L tokens); segment: three segment summaries of the first
T tokens (default L / 8) of the named workload, then three carries of 7 such
summaries; gemm: three projection GEMMs C[M][N] = A[M][K] . W[N][K]^T (bf16). Inputs are drawn on the GPU; a capture skips the
first two launches of the kernel it selects (ncu -s 2 -c 1 -k regex:...).
"""
from __future__ import annotations

import sys

import torch

from . import api
from . import workloads as W


def prefill_case(name: str, L: int = 0, shape=None, E: int = 0, disc: str = "euler"):
    w = W.WORKLOADS[name]
    if L > 0:
        w = w.scaled(seqlen=L)
    if E > 0:
        w = w.scaled(d_inner=E)
    tun = None
    if shape:
        k, dp = shape
        tun = {"kernel": k, "decay_path": dp}
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    args = (inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp)
    for _ in range(3):
        y, _, _ = api.prefill(*args, tuning=tun, discretization=disc)
    torch.cuda.synchronize()
    print("prefill ok", name, w.seqlen, w.d_inner, float(y.float().abs().mean()))


def decode_case(batch: int = 256):
    w = W.WORKLOADS["decode"].scaled(batch=batch, seqlen=4, decode_steps=3)
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    pre = {**inp, **{k: inp[k][:, :4] for k in ("x", "z", "B", "C", "dt_raw")}}
    _, cc, st = api.prefill(pre["x"], pre["z"], pre["B"], pre["C"], pre["dt_raw"], pre)
    y = torch.empty((w.batch, w.d_inner), dtype=w.io_dtype, device="cuda")
    for t in range(4, 7):
        api.decode_step(inp["x"][:, t], inp["z"][:, t], inp["B"][:, t], inp["C"][:, t], inp["dt_raw"][:, t], inp, cc,
                        st, y=y)
    torch.cuda.synchronize()
    print("decode ok", float(y.float().abs().mean()))


def block_case(name: str, L: int = 0):
    w, d_model = W.BLOCK_WORKLOADS[name]
    if L > 0:
        w = w.scaled(seqlen=L)
    inp = W.make_block_inputs(w, d_model, device="cuda", gen_device="cuda")
    proj = {k: inp[k] for k in api.PROJ_NAMES}
    for _ in range(3):
        out, _, _ = api.block_forward(inp["hidden"], inp, proj)
    torch.cuda.synchronize()
    print("block ok", name, w.seqlen, float(out.float().abs().mean()))


def ssd_case(name: str):
    inp = W.make_ssd_inputs(W.SSD_WORKLOADS[name], device="cuda")
    for _ in range(3):
        out = api.ssd_chunk_scan(*(inp[k] for k in ("cb", "x", "dt", "dA_cumsum", "C", "prev_states", "D")))
    torch.cuda.synchronize()
    print("ssd ok", name, float(out.float().abs().mean()))


def segment_case(name: str, T: int = 0):
    w = W.WORKLOADS[name]
    T = T or w.seqlen // 8
    w = W.Workload(w.name, batch=w.batch, seqlen=T, d_inner=w.d_inner, io_dtype=w.io_dtype, seed=w.seed,
                   clip_stress=w.clip_stress)
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    for _ in range(3):
        summ = api.segment_summary(inp["x"], inp["B"], inp["dt_raw"], inp)
    stacked = summ.unsqueeze(0).repeat(7, 1, 1, 1).contiguous()
    for _ in range(3):
        h = api.segment_carry(stacked, inp)
    torch.cuda.synchronize()
    print("segment ok", name, T, float(summ.abs().mean()), float(h.abs().mean()))


def gemm_case(M: int, N: int, K: int):
    g = torch.Generator(device="cuda").manual_seed(0)
    A = torch.randn((M, K), device="cuda", generator=g).to(torch.bfloat16)
    Wt = (torch.randn((N, K), device="cuda", generator=g) * K ** -0.5).to(torch.bfloat16)
    for _ in range(3):
        C = api.proj_gemm(A, Wt)
    torch.cuda.synchronize()
    print("gemm ok", M, N, K, float(C.float().abs().mean()))


if __name__ == "__main__":
    if sys.argv[1] == "prefill":
        L = int(sys.argv[3]) if len(sys.argv) > 3 else 0
        shape = tuple(int(v) for v in sys.argv[4:6]) if len(sys.argv) > 5 else None
        E = int(sys.argv[6]) if len(sys.argv) > 6 else 0
        prefill_case(sys.argv[2], L, shape, E, sys.argv[7] if len(sys.argv) > 7 else "euler")
    elif sys.argv[1] == "ssd":
        ssd_case(sys.argv[2])
    elif sys.argv[1] == "block":
        block_case(sys.argv[2], int(sys.argv[3]) if len(sys.argv) > 3 else 0)
    elif sys.argv[1] == "segment":
        segment_case(sys.argv[2], int(sys.argv[3]) if len(sys.argv) > 3 else 0)
    elif sys.argv[1] == "gemm":
        gemm_case(int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4]))
    elif sys.argv[1] == "decode":
        decode_case(int(sys.argv[2]) if len(sys.argv) > 2 else 256)
    else:
        raise SystemExit(__doc__)
