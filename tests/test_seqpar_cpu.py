"""Host logic of the sequence-parallel prefill (seqpar.py) on CPU.

The rank-local compute (segment summary, carry, prefill) is the oracle here,
standing in for the CUDA kernels, which need a GPU; the exchange is the real
torch.distributed path over gloo with 2 and 3 ranks. The gathered segment
outputs and the last rank's caches must equal one unsplit oracle prefill of
the whole sequence. Also checks the conv-history bookkeeping for segments
shorter than the history and the one-device driver prefill_segments.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_depthwise_b200 import seqpar

N = 16


def oracle_ops(disc="euler"):
    import oracle

    def to_np(t):
        return None if t is None else t.double().numpy()

    def summary(x, B, dt_raw, p, hist, **o):
        s = oracle.segment_summary(to_np(x), to_np(B), to_np(dt_raw), to_np(p["conv_w"]), to_np(p["conv_b"]),
                                   to_np(p["w_dt"]), to_np(p["dt_bias"]), to_np(p["A_log"]), hist=to_np(hist), disc=disc)
        return torch.from_numpy(s)

    def carry(summaries, p, h0):
        return torch.from_numpy(oracle.segment_carry(to_np(summaries), to_np(p["A_log"]), to_np(h0)))

    def prefill(x, z, B, C, dt_raw, p, hist, h0, **o):
        b, T, E = x.shape
        chans = [(s, e) for s in range(b) for e in range(E)]
        out, h, cc = oracle.prefill_sampled(x, z, B, C, dt_raw, *(to_np(p[k]) for k in
                                            ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")), chans,
                                            conv_cache_in=hist, ssm_state_in=h0, disc=disc)
        return (torch.from_numpy(out.reshape(b, E, T).transpose(0, 2, 1).copy()),
                torch.from_numpy(hc_rows(cc, b, E)), torch.from_numpy(h.reshape(b, E, N)))

    return seqpar.SegmentOps(summary=summary, carry=carry, prefill=prefill, summary_dtype=torch.float64)


def hc_rows(cc, b, E):
    return cc.reshape(b, E, 3).transpose(0, 2, 1).copy()


def problem(seed, b, L, E, with_init):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)  # noqa: E731
    p = dict(conv_w=0.5 * r(E, 4), conv_b=0.1 * r(E), w_dt=torch.rand(E, generator=g, dtype=torch.float64) * 2 - 1,
             dt_bias=torch.log(torch.expm1(torch.exp(torch.empty(E, dtype=torch.float64).uniform_(
                 np.log(1e-3), np.log(1e-1), generator=g)))),
             A_log=torch.log(torch.arange(1, N + 1, dtype=torch.float64)).repeat(E, 1), D=torch.ones(E, dtype=torch.float64))
    inp = dict(x=r(b, L, E), z=r(b, L, E), B=r(b, L, N), C=r(b, L, N), dt_raw=r(b, L))
    init = dict(conv_cache_in=r(b, 3, E), ssm_state_in=r(b, E, N)) if with_init else {}
    return p, inp, init


def unsplit(p, inp, init, disc="euler"):
    ops = oracle_ops(disc)
    return ops.prefill(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], p, init.get("conv_cache_in"),
                       init.get("ssm_state_in"))


def test_history_before_reaches_back_over_short_segments():
    b, E = 1, 2
    hist0 = torch.tensor([[[-3.0, -30], [-2, -20], [-1, -10]]])
    xs = [torch.tensor([[[1.0, 10], [2, 20], [3, 30], [4, 40]]]), torch.tensor([[[5.0, 50]]]),
          torch.zeros((1, 0, 2)), torch.tensor([[[6.0, 60], [7, 70]]])]
    tails = []
    for x in xs:
        t = torch.zeros((b, 3, E))
        k = min(3, x.shape[1])
        if k:
            t[:, 3 - k:] = x[:, x.shape[1] - k:]
        tails.append(t)
    lens = [x.shape[1] for x in xs]
    full = torch.cat([hist0] + xs, dim=1)
    starts = np.concatenate([[0], np.cumsum(lens)])
    for r in range(len(xs)):
        got = seqpar.history_before(tails, lens, r, hist0)
        torch.testing.assert_close(got, full[:, starts[r]:starts[r] + 3], rtol=0, atol=0)


@pytest.mark.parametrize("disc", ["euler", "zoh"])
def test_prefill_segments_one_device_equals_unsplit(disc):
    p, inp, init = problem(5, 2, 41, 8, True)
    want = unsplit(p, inp, init, disc)
    got = seqpar.prefill_segments(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], p, [0, 2, 17, 17, 30, 41],
                                  ops=oracle_ops(disc), **init)
    for g, w in zip(got, want):
        torch.testing.assert_close(g, w, rtol=1e-11, atol=1e-13)


def _worker(rank, world, port, lens, with_init, rank_knows_lengths, result_path, to_all=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p, inp, init = problem(7, 2, sum(lens), 8, with_init)  # every rank draws the same global problem
        s0 = sum(lens[:rank])
        seg = {k: v[:, s0:s0 + lens[rank]] for k, v in inp.items()}
        known = lens if rank_knows_lengths else None  # both ways of learning the lengths
        y, cc, st = seqpar.prefill_sequence_parallel(seg["x"], seg["z"], seg["B"], seg["C"], seg["dt_raw"], p,
                                                     lengths=known, final_caches_to_all=to_all, ops=oracle_ops(),
                                                     **init)
        m = max(lens)  # gloo gathers equal sizes: pad each segment to the longest (check only)
        pad = torch.zeros((2, m, 8), dtype=torch.float64)
        pad[:, :lens[rank]] = y
        ys = [torch.empty_like(pad) for _ in lens]
        dist.all_gather(ys, pad)
        if rank == (0 if to_all else world - 1):  # with to_all, rank 0 holds the sequence's caches too
            torch.save({"y": torch.cat([t[:, :n] for t, n in zip(ys, lens)], dim=1), "cc": cc, "st": st}, result_path)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens,with_init,known", [([23, 18], False, False), ([11, 2, 27], True, False),
                                                  ([11, 2, 27], False, True)])
def test_ranks_exchange_summaries_and_match_unsplit(tmp_path, lens, with_init, known):
    world = len(lens)
    port = 29700 + (os.getpid() % 200) + 7 * world + 3 * known
    result = str(tmp_path / "sp.pt")
    mp.start_processes(_worker, args=(world, port, lens, with_init, known, result), nprocs=world, join=True,
                       start_method="spawn")
    got = torch.load(result)
    p, inp, init = problem(7, 2, sum(lens), 8, with_init)
    y, cc, st = unsplit(p, inp, init)
    torch.testing.assert_close(got["y"], y, rtol=1e-11, atol=1e-13)
    torch.testing.assert_close(got["st"], st, rtol=1e-11, atol=1e-13)
    torch.testing.assert_close(got["cc"], cc, rtol=0, atol=0)


def test_final_caches_reach_every_rank(tmp_path):
    lens = [9, 14, 5]
    world = len(lens)
    port = 29900 + (os.getpid() % 50)
    result = str(tmp_path / "sp_all.pt")
    mp.start_processes(_worker, args=(world, port, lens, True, True, result, True), nprocs=world, join=True,
                       start_method="spawn")
    got = torch.load(result)
    p, inp, init = problem(7, 2, sum(lens), 8, True)
    y, cc, st = unsplit(p, inp, init)
    torch.testing.assert_close(got["y"], y, rtol=1e-11, atol=1e-13)
    torch.testing.assert_close(got["st"], st, rtol=1e-11, atol=1e-13)
    torch.testing.assert_close(got["cc"], cc, rtol=0, atol=0)
