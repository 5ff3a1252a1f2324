"""Channel sharding across GPUs (one process per GPU).

Channels of the block core are independent: the depthwise conv and every
per-channel parameter (conv_w, conv_b, w_dt, dt_bias, A_log, D) touch one
channel only, and B, C, dt_raw are per token, shared by all channels. A
problem with E channels therefore splits into contiguous channel slices with
no exchange on the data path; each rank runs the ordinary kernels on its
slice (B, C, dt_raw replicated). Slices are multiples of 8 channels, the
kernels' channel granularity.
"""
from __future__ import annotations


def shard_range(E: int, world: int, rank: int, align: int = 8) -> tuple:
    """[lo, hi) of the channels rank `rank` owns, in units of `align`
    channels, balanced to within one unit."""
    if E % align:
        raise ValueError(f"E={E} must be a multiple of {align}")
    if not (0 <= rank < world):
        raise ValueError("rank out of range")
    units = E // align
    base, extra = divmod(units, world)
    lo_u = rank * base + min(rank, extra)
    hi_u = lo_u + base + (1 if rank < extra else 0)
    return lo_u * align, hi_u * align


PER_CHANNEL = ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")
PER_CHANNEL_ACTIVATIONS = ("x", "z")
SHARED = ("B", "C", "dt_raw")


def slice_inputs(inp: dict, lo: int, hi: int) -> dict:
    """The rank-local view of a full input dict: channel columns [lo, hi) of
    x, z and the parameters; B, C, dt_raw whole."""
    out = {}
    for k, v in inp.items():
        if k in PER_CHANNEL:
            out[k] = v[lo:hi].contiguous()
        elif k in PER_CHANNEL_ACTIVATIONS:
            out[k] = v[..., lo:hi]
        else:
            out[k] = v
    return out
