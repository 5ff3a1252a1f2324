"""Seeded synthetic workloads for the selective-scan block core.

This module only draws inputs: shapes, seeds and value distributions. It holds
none of the method's arithmetic and is shared by the CUDA path's tests, the
benchmark and the oracle-side tests, so both sides read identical bytes.

Distributions (every workload): x, z ~ N(0, 1); conv_w ~ N(0, var 0.25);
conv_b = 0; B, C, dt_raw ~ N(0, 1); w_dt ~ U(-1, 1); dt_bias = softplus^-1(d)
with log d ~ U(ln 1e-3, ln 1e-1); A_log[e, n] = ln(n + 1) (the stated A
initialisation, giving A = -1 .. -N); D = 1; dt clip [1e-4, 1]; zero initial
state. The long-context workload also pins 5% of channels to dt_bias =
softplus^-1(1e-4) and another 5% to softplus^-1(1.0), so that dt sits at the
clip bounds there.

Draw order: one torch.Generator per workload seeded with its seed. Parameters
are drawn on the CPU in the order conv_w, conv_b, w_dt, dt_bias, A_log, D
(then the stress permutation, if any); activations x, z, B, C, dt_raw are then
drawn in that order on ``gen_device`` from a second generator on that device
seeded with the same seed (torch's CPU and CUDA generators differ, so the
device that drew the activations is part of a workload's identity).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    d_inner: int  # E, channels
    d_state: int = 16  # N
    d_conv: int = 4  # K
    io_dtype: torch.dtype = torch.bfloat16
    seed: int = 0
    dt_min: float = 1e-4
    dt_max: float = 1.0
    clip_stress: bool = False  # long-context: 10% of channels at the dt clip bounds
    decode_steps: int = 0  # >0: prompt of `seqlen`, then this many 1-token steps
    x_row_stride: int = 0  # 0 = d_inner (dense); 2*d_inner = fused in_proj buffer
    note: str = ""

    @property
    def total_len(self) -> int:
        return self.seqlen + self.decode_steps

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", batch=1, seqlen=64, d_inner=32, io_dtype=torch.float32, seed=0,
                     note="tiny prefill, fp32 throughout"),
    "axon_layer": Workload("axon_layer", batch=1, seqlen=2048, d_inner=7680, seed=1,
                           note="Axon-SSM layer shape prefill"),
    "batched": Workload("batched", batch=8, seqlen=4096, d_inner=5120, seed=2, note="batched prefill"),
    "long_context": Workload("long_context", batch=1, seqlen=65536, d_inner=7680, seed=3, clip_stress=True,
                             note="long-context prefill with dt clip stress"),
    "decode": Workload("decode", batch=256, seqlen=512, d_inner=7680, seed=4, decode_steps=1024,
                       note="prompt 512 then 1024 single-token decode steps"),
}


def clip_stress_channels(w: Workload):
    """(low, high): the channel indices whose dt_bias make_params pins to
    softplus^-1(dt_min) and softplus^-1(dt_max) (empty unless clip_stress).
    Replays the same draws, so it always agrees with make_params."""
    if not w.clip_stress:
        return torch.empty(0, dtype=torch.long), torch.empty(0, dtype=torch.long)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    E, K = w.d_inner, w.d_conv
    torch.randn(E, K, generator=g, dtype=torch.float32)
    torch.rand(E, generator=g, dtype=torch.float32)
    torch.rand(E, generator=g, dtype=torch.float64)
    perm = torch.randperm(E, generator=g)
    n5 = E // 20
    return perm[:n5].sort().values, perm[n5:2 * n5].sort().values


def softplus_inv(d: torch.Tensor) -> torch.Tensor:
    """Inverse of softplus, used only to place dt_bias (an initialisation recipe)."""
    return torch.log(torch.expm1(d))


def make_params(w: Workload) -> dict:
    """Per-channel parameters, fp32, drawn on the CPU in the documented order."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    E, N, K = w.d_inner, w.d_state, w.d_conv
    conv_w = torch.randn(E, K, generator=g, dtype=torch.float32) * 0.5  # var 0.25
    conv_b = torch.zeros(E, dtype=torch.float32)
    w_dt = torch.rand(E, generator=g, dtype=torch.float32) * 2.0 - 1.0
    log_d = torch.rand(E, generator=g, dtype=torch.float64) * (math.log(1e-1) - math.log(1e-3)) + math.log(1e-3)
    dt_bias = softplus_inv(torch.exp(log_d))
    if w.clip_stress:
        perm = torch.randperm(E, generator=g)
        n5 = E // 20
        dt_bias[perm[:n5]] = float(softplus_inv(torch.tensor(w.dt_min, dtype=torch.float64)))
        dt_bias[perm[n5:2 * n5]] = float(softplus_inv(torch.tensor(w.dt_max, dtype=torch.float64)))
    dt_bias = dt_bias.to(torch.float32)
    A_log = torch.log(torch.arange(1, N + 1, dtype=torch.float32)).repeat(E, 1).contiguous()
    D = torch.ones(E, dtype=torch.float32)
    return dict(conv_w=conv_w, conv_b=conv_b, w_dt=w_dt, dt_bias=dt_bias, A_log=A_log, D=D)


def _randn_chunked(shape, g, device, dtype, chunk_elems=1 << 28):
    """N(0,1) drawn in fp32 and rounded (RNE) to `dtype`, in bounded chunks
    along the leading dimension to cap the fp32 temporary."""
    out = torch.empty(shape, dtype=dtype, device=device)
    if out.numel() == 0:
        return out
    flat = out.view(shape[0], -1)
    per_row = flat.shape[1]
    rows = max(1, chunk_elems // max(per_row, 1))
    for r0 in range(0, shape[0], rows):
        r1 = min(shape[0], r0 + rows)
        flat[r0:r1] = torch.randn((r1 - r0, per_row), generator=g, device=device, dtype=torch.float32).to(dtype)
    return out


def make_activations(w: Workload, gen_device="cpu") -> dict:
    """x, z: [b, T, S] in io dtype, S = row stride (>= E; extra columns are
    filler a fused in_proj buffer would hold); B, C: [b, T, N] fp32;
    dt_raw: [b, T] fp32; T = prompt + decode steps."""
    g = torch.Generator(device=gen_device).manual_seed(w.seed)
    b, T, E, N = w.batch, w.total_len, w.d_inner, w.d_state
    S = w.x_row_stride or E
    x = _randn_chunked((b, T, S), g, gen_device, w.io_dtype)
    z = _randn_chunked((b, T, S), g, gen_device, w.io_dtype)
    B = torch.randn((b, T, N), generator=g, device=gen_device, dtype=torch.float32)
    C = torch.randn((b, T, N), generator=g, device=gen_device, dtype=torch.float32)
    dt_raw = torch.randn((b, T), generator=g, device=gen_device, dtype=torch.float32)
    return dict(x=x, z=z, B=B, C=C, dt_raw=dt_raw)


def make_inputs(w: Workload, device="cpu", gen_device=None) -> dict:
    """Parameters + activations, moved to `device`. Activations are drawn on
    `gen_device` (default: `device`)."""
    gen_device = gen_device or device
    p = {k: v.to(device) for k, v in make_params(w).items()}
    a = {k: v.to(device) for k, v in make_activations(w, gen_device).items()}
    p.update(a)
    return p



# ------------------------------------------------------------- the block ---
# The whole AxonSSMBlock forward at the pages' layer shape: hidden_dim D = 2560,
# E = 7680 ("Axon-SSM: selective state space model", "Algorithm").
BLOCK_WORKLOADS = {
    "block_axon_layer": (Workload("block_axon_layer", batch=1, seqlen=2048, d_inner=7680, seed=5,
                                  note="AxonSSMBlock forward at the Axon layer shape, D = 2560"), 2560),
    "block_long_context": (Workload("block_long_context", batch=1, seqlen=65536, d_inner=7680, seed=6,
                                    note="AxonSSMBlock forward over a 64K-token context, D = 2560"), 2560),
}


def make_block_inputs(w: Workload, d_model: int, device="cpu", gen_device=None) -> dict:
    """Synthetic inputs of the block forward: the core's parameters (make_params),
    hidden [b, L, D] ~ N(0, 1) and the projection weights W_in [2E, D] ~ N(0, 1/D),
    W_x [2N+1, E] ~ N(0, 1/E), W_out [D, E] ~ N(0, 1/E) (so x, z, B, C and dt_raw
    come out near unit variance, like the core workloads' draws), all bf16 (RNE
    from fp32), drawn in that order after the parameters from one seeded generator."""
    gen_device = gen_device or device
    p = {k: v.to(device) for k, v in make_params(w).items()}
    g = torch.Generator(device=gen_device).manual_seed(w.seed + 1000)
    b, L, E, N = w.batch, w.seqlen, w.d_inner, w.d_state
    hidden = _randn_chunked((b, L, d_model), g, gen_device, torch.bfloat16)
    scale = lambda t, s: (t.float() * s).to(torch.bfloat16)  # noqa: E731
    W_in = scale(_randn_chunked((2 * E, d_model), g, gen_device, torch.bfloat16), d_model ** -0.5)
    W_x = scale(_randn_chunked((2 * N + 1, E), g, gen_device, torch.bfloat16), E ** -0.5)
    W_out = scale(_randn_chunked((d_model, E), g, gen_device, torch.bfloat16), E ** -0.5)
    p.update(hidden=hidden.to(device), W_in=W_in.to(device), W_x=W_x.to(device), W_out=W_out.to(device))
    return p


# ---------------------------------------------------------- chunk scan ---
# The Mamba-2 chunk scan of "What is the Mamba model?" ("chunkscan"): the pages
# give the operation and a chunk length of 128 as their example, no sizes; these
# are a synthetic multi-head layout with one B/C group.
SSD_WORKLOADS = {
    "ssd_small": dict(batch=2, seqlen=384, nheads=4, headdim=64, ngroups=2, dstate=128, chunk_size=128, seed=7),
    "ssd_chunk_scan": dict(batch=8, seqlen=4096, nheads=80, headdim=64, ngroups=1, dstate=128, chunk_size=128,
                           seed=8),
}


def make_ssd_inputs(spec: dict, device="cpu") -> dict:
    """Seeded chunk-scan inputs drawn from one SSD model so that the values are
    those of a real layer: x ~ N(0,1); B, C ~ N(0,1)/sqrt(dstate) per group;
    dt = softplus(N(-2, 1)) per (token, head); A_h = -exp(U(ln 1/16, ln 1/2))
    (a few units of decay over a chunk, so the carried state matters);
    dA_cumsum = the within-chunk cumulative sum of dt A_h; cb = C B^T per chunk
    (fp32, then bf16); prev_states ~ N(0, 1/4); D ~ U(0.5, 1.5). bf16 for cb, x,
    C, prev_states (RNE from fp32), fp32 for dt, dA_cumsum, D. Drawn on `device`."""
    g = torch.Generator(device=device).manual_seed(spec["seed"])
    b, L, H, P = spec["batch"], spec["seqlen"], spec["nheads"], spec["headdim"]
    G, N, cs = spec["ngroups"], spec["dstate"], spec["chunk_size"]
    nc = L // cs
    f32 = dict(device=device, dtype=torch.float32, generator=g)
    x = torch.randn((b, L, H, P), **f32).to(torch.bfloat16)
    B = (torch.randn((b, L, G, N), **f32) * N ** -0.5).to(torch.bfloat16)
    C = (torch.randn((b, L, G, N), **f32) * N ** -0.5).to(torch.bfloat16)
    dt = torch.nn.functional.softplus(torch.randn((b, H, nc, cs), **f32) - 2.0)
    A = -torch.exp(torch.rand(H, **f32) * (math.log(0.5) - math.log(1 / 16)) + math.log(1 / 16))
    dA_cumsum = torch.cumsum(dt * A[None, :, None, None], dim=-1)
    Bc = B.float().reshape(b, nc, cs, G, N)
    Cc = C.float().reshape(b, nc, cs, G, N)
    cb = torch.einsum("bclgn,bcsgn->bcgls", Cc, Bc).to(torch.bfloat16).contiguous()
    prev = (torch.randn((b, nc, H, P, N), **f32) * 0.5).to(torch.bfloat16)
    D = torch.rand(H, **f32) + 0.5
    return dict(cb=cb, x=x, dt=dt.contiguous(), dA_cumsum=dA_cumsum.contiguous(), C=C, prev_states=prev, D=D)
