"""Sequence-parallel prefill: one sequence split along L across ranks (one
process per GPU), for contexts longer than one GPU should walk alone.

Rank r holds segment r of every sequence (tokens [start_r, start_r + T_r)),
and the steps are those of "What is the Mamba model?" (velog, Texnee),
"chunkscan", with the segment as the chunk:

  0. conv history: every rank's last 3 raw x rows are all-gathered, so rank r
     knows the 3 rows before its segment (segments shorter than 3 tokens take
     rows from further back, then from the initial conv cache);
  1. summary: ranks 0..R-2 reduce their segment to (zero-start final state,
     dt sum) -- ssm_segment_summary, independent across ranks;
  2. exchange: the summaries are all-gathered (b * 17 * E floats per rank);
  3. carry: rank r folds summaries 0..r-1 into the state entering its segment
     (ssm_segment_carry, the closed form of "Mamba/SSM basics", "Technical
     details", a segment at a time);
  4. combine: rank r runs the ordinary prefill of its segment from that state
     and history (ssm_prefill); its outputs are rounded once.

The last rank's conv cache and state are those of the whole sequence. Every
rank takes the same collective steps in the same order. The exchanged bytes
are small and independent of L: 3 x rows and one summary per rank.

The per-segment compute is passed in as `ops` (default: the CUDA library
through api.py); the exchange is torch.distributed all_gather, NCCL between
GPUs. There is no CPU path: the default ops reject tensors off the GPU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist

HIST = 3   # raw x rows of conv history (d_conv - 1)
N_STATE = 16


@dataclass
class SegmentOps:
    """The three per-segment computations of the path."""
    summary: Callable      # (x, B, dt_raw, params, conv_cache_in, **opt) -> [b, 17, E] fp32
    carry: Callable        # (summaries [r, b, 17, E], params, ssm_state_in) -> [b, E, 16] fp32
    prefill: Callable      # (x, z, B, C, dt_raw, params, conv_cache_in, ssm_state_in, **opt) -> (y, cc, st)
    summary_dtype: torch.dtype = torch.float32


def cuda_ops() -> SegmentOps:
    from . import api

    return SegmentOps(
        summary=lambda x, B, dt_raw, params, conv_cache_in, **o: api.segment_summary(
            x, B, dt_raw, params, conv_cache_in=conv_cache_in, **o),
        carry=lambda summaries, params, ssm_state_in: api.segment_carry(summaries, params, ssm_state_in=ssm_state_in),
        prefill=lambda x, z, B, C, dt_raw, params, conv_cache_in, ssm_state_in, **o: api.prefill(
            x, z, B, C, dt_raw, params, conv_cache_in=conv_cache_in, ssm_state_in=ssm_state_in, **o),
    )


def _as_bits(t: torch.Tensor) -> torch.Tensor:
    """Byte view for the exchange: every backend moves uint8 bit-exactly (NCCL
    has no 16-bit integer type, and gloo's bf16 support varies)."""
    return t.view(torch.uint8)


def history_before(tails: list, lengths: list, r: int, hist0: torch.Tensor) -> torch.Tensor:
    """The HIST raw x rows before segment r: the last rows of segments r-1,
    r-2, ... (each tail holds its segment's last min(HIST, T_j) rows,
    right-aligned in HIST rows), then of the initial history hist0.
    tails[j], hist0: [b, HIST, E]. Returns [b, HIST, E]."""
    rows = [hist0]
    for j in range(r):
        k = min(HIST, lengths[j])
        if k:
            rows.append(tails[j][:, HIST - k:])
    return torch.cat(rows, dim=1)[:, -HIST:].contiguous()


def prefill_sequence_parallel(x, z, B, C, dt_raw, params, *, group=None, conv_cache_in=None, ssm_state_in=None,
                              lengths: Optional[list] = None, final_caches_to_all: bool = False,
                              ops: Optional[SegmentOps] = None, **opt):
    """This rank's part of a sequence-parallel prefill.

    x, z: [b, T_r, E]; B, C: [b, T_r, 16]; dt_raw: [b, T_r] -- segment r of
    each sequence, r = this rank in `group`, segments in rank order.
    conv_cache_in [b, 3, E] and ssm_state_in [b, E, 16] describe the state
    before segment 0 and are passed identically on every rank (or None).
    `lengths` (every rank's T, in rank order) saves the exchange of the
    segment lengths, whose read-back synchronises the host; every rank must
    pass it or none. `opt` holds dt_min, dt_max, discretization. Returns
    (y [b, T_r, E], conv_cache_out, ssm_state_out); the last rank's caches are
    the sequence's, and with final_caches_to_all=True (on every rank) they are
    broadcast so that every rank returns the sequence's caches."""
    ops = ops or cuda_ops()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    b, T, E = x.shape
    dev, io = x.device, x.dtype

    # 0. conv history: segment lengths and last HIST raw x rows of every rank.
    if lengths is None:
        lens = torch.tensor([T], dtype=torch.int64, device=dev)
        all_lens = [torch.empty_like(lens) for _ in range(world)]
        dist.all_gather(all_lens, lens, group=group)
        lengths = [int(v.item()) for v in all_lens]
    elif len(lengths) != world or lengths[rank] != T:
        raise ValueError("lengths must list every rank's segment length, this rank's equal to x.shape[1]")
    tail = torch.zeros((b, HIST, E), dtype=io, device=dev)
    k = min(HIST, T)
    if k:
        tail[:, HIST - k:] = x[:, T - k:]
    tails_bits = [torch.empty_like(_as_bits(tail)) for _ in range(world)]
    dist.all_gather(tails_bits, _as_bits(tail), group=group)
    tails = [t.view(io) for t in tails_bits]
    hist0 = conv_cache_in if conv_cache_in is not None else torch.zeros((b, HIST, E), dtype=io, device=dev)
    halo = history_before(tails, lengths, rank, hist0)
    if rank == 0 and conv_cache_in is None:
        halo = None  # the kernels' zero history

    # 1. summary of this segment (the last one is needed by nobody).
    if rank < world - 1:
        summ = ops.summary(x, B, dt_raw, params, halo, **opt)
    else:
        summ = torch.zeros((b, N_STATE + 1, E), dtype=ops.summary_dtype, device=dev)

    # 2. exchange.
    gathered = [torch.empty_like(summ) for _ in range(world)]
    dist.all_gather(gathered, summ.contiguous(), group=group)

    # 3. carry into this segment.
    if rank == 0:
        h_in = ssm_state_in
    else:
        h_in = ops.carry(torch.stack(gathered[:rank]).contiguous(), params, ssm_state_in)

    # 4. combine: the ordinary prefill of the segment from the carried state.
    y, cc, st = ops.prefill(x, z, B, C, dt_raw, params, halo, h_in, **opt)
    if final_caches_to_all and world > 1:
        last = dist.get_global_rank(group, world - 1) if group is not None else world - 1
        cc_bits = _as_bits(cc.contiguous())
        dist.broadcast(cc_bits, src=last, group=group)
        st = st.contiguous()
        dist.broadcast(st, src=last, group=group)
        cc = cc_bits.view(cc.dtype).view(cc.shape)
    return y, cc, st


def prefill_segments(x, z, B, C, dt_raw, params, bounds, *, conv_cache_in=None, ssm_state_in=None,
                     ops: Optional[SegmentOps] = None, **opt):
    """The same path on one device: the sequence [b, L, ...] is cut at
    `bounds` (0 = s_0 < s_1 < ... < s_R = L), every segment but the last is
    summarised, and each segment is computed from its carried state. The
    segments' kernels do not wait on one another; this is how the
    sequence-parallel path is checked and timed with a single GPU.
    Returns (y [b, L, E], conv_cache_out, ssm_state_out)."""
    ops = ops or cuda_ops()
    b, L, E = x.shape
    if bounds[0] != 0 or bounds[-1] != L or any(b1 < b0 for b0, b1 in zip(bounds, bounds[1:])):
        raise ValueError("bounds must rise from 0 to L")
    R = len(bounds) - 1
    dev, io = x.device, x.dtype
    hist0 = conv_cache_in if conv_cache_in is not None else torch.zeros((b, HIST, E), dtype=io, device=dev)
    full = torch.cat([hist0, x], dim=1)  # raw rows; token t at full[:, t + HIST]
    halos = [None if (r == 0 and conv_cache_in is None) else full[:, bounds[r]:bounds[r] + HIST].contiguous()
             for r in range(R)]
    seg = lambda t, r: t[:, bounds[r]:bounds[r + 1]]  # noqa: E731
    summaries = [ops.summary(seg(x, r), seg(B, r), seg(dt_raw, r), params, halos[r], **opt) for r in range(R - 1)]
    ys, cc, st = [], None, None
    for r in range(R):
        h_in = ssm_state_in if r == 0 else ops.carry(torch.stack(summaries[:r]).contiguous(), params, ssm_state_in)
        y, cc, st = ops.prefill(seg(x, r), seg(z, r), seg(B, r), seg(C, r), seg(dt_raw, r), params, halos[r], h_in,
                                **opt)
        ys.append(y)
    return torch.cat(ys, dim=1), cc, st
