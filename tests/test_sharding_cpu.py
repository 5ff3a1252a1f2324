"""Multi-process host logic of channel sharding (gloo, world size 2, CPU).

Each rank owns a contiguous channel slice; B, C, dt_raw are replicated; no
data-path collective is needed. The test runs two gloo ranks that each compute
their slice (with the CPU oracle standing in for the kernels, which need a
GPU), gathers the slices once for checking, and compares with one unsharded
computation. It also checks the partition itself.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_depthwise_b200 import workloads as W
from selective_state_space_depthwise_b200.sharding import shard_range, slice_inputs


def test_shard_ranges_cover_and_balance():
    for E in (8, 64, 7680, 5120, 40):
        for world in (1, 2, 3, 4, 8):
            spans = [shard_range(E, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == E
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in spans]
            assert all(s % 8 == 0 for s in sizes)
            assert max(sizes) - min(sizes) <= 8
    with pytest.raises(ValueError):
        shard_range(12, 2, 0)


def _oracle_slice(inp, w, lo, hi):
    import oracle

    loc = slice_inputs(inp, lo, hi)
    n = hi - lo
    xs = np.stack([loc["x"][0, :, c].double().numpy() for c in range(n)])
    zs = np.stack([loc["z"][0, :, c].double().numpy() for c in range(n)])
    p = {k: loc[k].double().numpy() for k in ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")}
    out, h, cc = oracle.channels(xs, zs, loc["B"].double().numpy(), loc["C"].double().numpy(),
                                 loc["dt_raw"].double().numpy(), [0] * n, p["conv_w"], p["conv_b"], p["w_dt"],
                                 p["dt_bias"], p["A_log"], p["D"], lo=w.dt_min, hi=w.dt_max)
    return out, h, cc


def _worker(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.Workload("shard", batch=1, seqlen=40, d_inner=48, io_dtype=torch.float32, seed=21)
        inp = W.make_inputs(w)  # every rank draws the same global problem (seeded)
        lo, hi = shard_range(w.d_inner, world, rank)
        out, h, cc = _oracle_slice(inp, w, lo, hi)
        # gather the slices (check only; the data path itself needs no collective)
        n_max = max(b - a for a, b in (shard_range(w.d_inner, world, r) for r in range(world)))
        pad = np.zeros((n_max, out.shape[1] + 16 + 3))
        pad[: hi - lo] = np.concatenate([out, h, cc], axis=1)
        buf = [torch.zeros_like(torch.from_numpy(pad)) for _ in range(world)]
        dist.all_gather(buf, torch.from_numpy(pad))
        if rank == 0:
            parts = []
            for r in range(world):
                a, b = shard_range(w.d_inner, world, r)
                parts.append(buf[r][: b - a].numpy())
            np.save(result_path, np.concatenate(parts, axis=0))
    finally:
        dist.destroy_process_group()


def test_two_rank_channel_shards_equal_one_unsharded_run(tmp_path):
    world = 2
    port = 29500 + (os.getpid() % 1000)
    result = str(tmp_path / "gathered.npy")
    mp.start_processes(_worker, args=(world, port, result), nprocs=world, join=True, start_method="spawn")
    got = np.load(result)
    w = W.Workload("shard", batch=1, seqlen=40, d_inner=48, io_dtype=torch.float32, seed=21)
    inp = W.make_inputs(w)
    out, h, cc = _oracle_slice(inp, w, 0, w.d_inner)
    want = np.concatenate([out, h, cc], axis=1)
    np.testing.assert_array_equal(got, want)
