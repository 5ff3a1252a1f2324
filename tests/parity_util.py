"""Helpers shared by the GPU parity tests: oracle runs over chosen channels and
the comparison metrics (relative L2 per tensor, bit-exact caches)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-3}  # relative L2 of outputs and final states, per io dtype


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    num = np.linalg.norm(got - want)
    return float(num / den) if den > 0 else float(num)


def round_io(a, dtype) -> np.ndarray:
    """Round oracle values once to the io dtype (RNE), back to float64."""
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).to(dtype).double().numpy()


def all_channels(b, E):
    return [(s, e) for s in range(b) for e in range(E)]


def oracle_prefill(inp, chans, *, L=None, conv_cache_in=None, ssm_state_in=None, dt_min=1e-4, dt_max=1.0,
                   disc="euler", threads=0):
    """Oracle over `chans` of inputs shaped like the kernel's (CPU or GPU
    tensors; the stored values are read back exactly). L limits the tokens."""
    x, z, B, C, dt = inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"]
    if L is not None:
        x, z, B, C, dt = x[:, :L], z[:, :L], B[:, :L], C[:, :L], dt[:, :L]
    seqs = sorted({s for s, _ in chans})
    remap = {s: i for i, s in enumerate(seqs)}
    Bn = B[seqs].detach().to("cpu").double().numpy()
    Cn = C[seqs].detach().to("cpu").double().numpy()
    dtn = dt[seqs].detach().to("cpu").double().numpy()
    xs = np.stack([x[s, :, e].detach().to("cpu").double().numpy() for s, e in chans])
    zs = np.stack([z[s, :, e].detach().to("cpu").double().numpy() for s, e in chans])
    es = [e for _, e in chans]
    p = {k: inp[k].detach().to("cpu").double().numpy() for k in ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")}
    hist = None if conv_cache_in is None else np.stack(
        [conv_cache_in[s, :, e].detach().to("cpu").double().numpy() for s, e in chans])
    h0 = None if ssm_state_in is None else np.stack(
        [ssm_state_in[s, e, :].detach().to("cpu").double().numpy() for s, e in chans])
    return oracle.channels(xs, zs, Bn, Cn, dtn, [remap[s] for s, _ in chans], p["conv_w"][es], p["conv_b"][es],
                           p["w_dt"][es], p["dt_bias"][es], p["A_log"][es], p["D"][es], hist=hist, h0=h0,
                           lo=dt_min, hi=dt_max, disc=disc, threads=threads)


def gather(y, cache, state, chans):
    """Kernel outputs of the chosen channels as float64 arrays."""
    ys = np.stack([y[s, :, e].detach().to("cpu").double().numpy() for s, e in chans])
    cs = np.stack([cache[s, :, e].detach().to("cpu").double().numpy() for s, e in chans])
    hs = np.stack([state[s, e, :].detach().to("cpu").double().numpy() for s, e in chans])
    return ys, cs, hs


def compare(io_dtype, got, want, label=""):
    """Assert the parity tolerances: y and state by relative L2, the conv
    cache bit-exact. Returns the measured errors."""
    ys, cs, hs = got
    out_o, h_o, c_o = want
    e_y = rel_l2(ys, round_io(out_o, io_dtype))
    e_h = rel_l2(hs, h_o)
    assert np.array_equal(cs, c_o), f"{label}: conv_cache differs"
    assert e_y <= TOL[io_dtype], f"{label}: y rel-L2 {e_y:.3e} > {TOL[io_dtype]:.0e}"
    assert e_h <= TOL[io_dtype], f"{label}: state rel-L2 {e_h:.3e} > {TOL[io_dtype]:.0e}"
    assert np.isfinite(ys).all() and np.isfinite(hs).all(), f"{label}: non-finite output"
    return e_y, e_h


def compare_full(io_dtype, inp, got, *, label="", disc="euler", dt_min=1e-4, dt_max=1.0, max_elems=1 << 25,
                 subsets=None):
    """Every (sequence, channel) of a run against the oracle. `got` is one
    (y, cache, state) triple or a dict {name: triple} of runs on the same
    inputs (the oracle then runs once for all of them). The channels go in
    blocks (whole sequences, or channel ranges of one long sequence) of at most
    about `max_elems` tokens x channels, so full-size workloads fit in host
    memory. Per (sequence, channel) the squared errors are kept, so besides the
    relative L2 over the whole run this reports, and bounds by the same
    tolerance, the worst single channel and each named channel subset
    (`subsets`: {name: channel indices}, applied in every sequence). The conv
    cache must match bit for bit. Returns {name: report} (or the report of the
    single run), a report being {"y", "state", "worst_y", "worst_state",
    "worst_channel", "subsets": {name: (y, state)}}.

    The run-wide and subset figures compare with the oracle rounded once to the
    io dtype, as the other parity checks do. The worst channel's y is measured
    against the unrounded oracle and bounded by the io dtype's unit roundoff
    (2^-8 for bf16, 2^-24 floor plus the fp32 bar for fp32): one output that
    sits on a rounding tie can land on either neighbour, and on a channel whose
    largest value dominates its norm that single step alone can exceed the
    run-wide bar even when both sides round correctly."""
    runs = got if isinstance(got, dict) else {"": got}
    x, z = inp["x"], inp["z"]
    b, L, E = x.shape
    p = {k: inp[k].detach().to("cpu").double().numpy() for k in ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")}
    per_seq = L * E
    seqs_per_block = max(1, max_elems // max(per_seq, 1))
    ch_per_block = E if seqs_per_block > 1 or per_seq <= max_elems else max(1, max_elems // max(L, 1))
    # per (sequence, channel): |dy|^2, |y|^2, |dh|^2, |h|^2
    acc = {n: np.zeros((b, E, 5)) for n in runs}  # + |y - unrounded oracle|^2
    for s0 in range(0, b, seqs_per_block):
        s1 = min(b, s0 + seqs_per_block)
        Bn = inp["B"][s0:s1].detach().to("cpu").double().numpy()
        Cn = inp["C"][s0:s1].detach().to("cpu").double().numpy()
        dtn = inp["dt_raw"][s0:s1].detach().to("cpu").double().numpy()
        for e0 in range(0, E, ch_per_block):
            e1 = min(E, e0 + ch_per_block)
            n_e = e1 - e0
            # (seq, channel) rows, channel fastest
            xs = x[s0:s1, :, e0:e1].permute(0, 2, 1).reshape(-1, L).double().cpu().numpy()
            zs = z[s0:s1, :, e0:e1].permute(0, 2, 1).reshape(-1, L).double().cpu().numpy()
            bidx = np.repeat(np.arange(s1 - s0), n_e).tolist()
            tile = lambda a: np.tile(a[e0:e1], (s1 - s0,) + (1,) * (a.ndim - 1))  # noqa: E731
            out_o, h_o, c_o = oracle.channels(xs, zs, Bn, Cn, dtn, bidx, tile(p["conv_w"]), tile(p["conv_b"]),
                                              tile(p["w_dt"]), tile(p["dt_bias"]), tile(p["A_log"]), tile(p["D"]),
                                              lo=dt_min, hi=dt_max, disc=disc)
            want_y = round_io(out_o, io_dtype)
            for name, (y, cache, state) in runs.items():
                ys = y[s0:s1, :, e0:e1].permute(0, 2, 1).reshape(-1, L).double().cpu().numpy()
                hs = state[s0:s1, e0:e1, :].reshape(-1, 16).double().cpu().numpy()
                cs = cache[s0:s1, :, e0:e1].permute(0, 2, 1).reshape(-1, 3).double().cpu().numpy()
                assert np.array_equal(cs, c_o), f"{label}{name}: conv_cache differs in sequences {s0}..{s1 - 1}"
                assert np.isfinite(ys).all() and np.isfinite(hs).all(), f"{label}{name}: non-finite output"
                blk = np.stack([np.sum((ys - want_y) ** 2, axis=1), np.sum(want_y ** 2, axis=1),
                                np.sum((hs - h_o) ** 2, axis=1), np.sum(h_o ** 2, axis=1),
                                np.sum((ys - out_o) ** 2, axis=1)], axis=1)
                acc[name][s0:s1, e0:e1] = blk.reshape(s1 - s0, n_e, 5)

    def rl2(a):
        return (float(np.sqrt(a[..., 0].sum() / a[..., 1].sum())) if a[..., 1].sum() > 0 else float(np.sqrt(a[..., 0].sum())),
                float(np.sqrt(a[..., 2].sum() / a[..., 3].sum())) if a[..., 3].sum() > 0 else float(np.sqrt(a[..., 2].sum())))

    tol = TOL[io_dtype]
    tol_channel = 2.0 ** -8 if io_dtype == torch.bfloat16 else tol
    reports = {}
    for name, a in acc.items():
        e_y, e_h = rl2(a)
        with np.errstate(divide="ignore", invalid="ignore"):
            cy = np.sqrt(np.where(a[..., 1] > 0, a[..., 4] / a[..., 1], a[..., 4]))
            ch = np.sqrt(np.where(a[..., 3] > 0, a[..., 2] / a[..., 3], a[..., 2]))
        wy = np.unravel_index(int(np.argmax(cy)), cy.shape)
        rep = {"y": e_y, "state": e_h, "worst_y": float(cy.max()), "worst_state": float(ch.max()),
               "worst_channel": (int(wy[0]), int(wy[1])), "subsets": {}}
        for sname, idx in (subsets or {}).items():
            idx = np.asarray(idx, dtype=np.int64)
            if idx.size:
                rep["subsets"][sname] = rl2(a[:, idx])
        tag = f"{label}{' ' + name if name else ''}"
        assert e_y <= tol, f"{tag}: y rel-L2 {e_y:.3e} > {tol:.0e}"
        assert e_h <= tol, f"{tag}: state rel-L2 {e_h:.3e} > {tol:.0e}"
        assert rep["worst_y"] <= tol_channel, \
            f"{tag}: worst channel {rep['worst_channel']} y rel-L2 {rep['worst_y']:.3e} against the unrounded oracle"
        assert rep["worst_state"] <= tol, f"{tag}: worst channel state rel-L2 {rep['worst_state']:.3e}"
        for sname, (sy, sh) in rep["subsets"].items():
            assert sy <= tol and sh <= tol, f"{tag}: subset {sname} rel-L2 y {sy:.3e}, state {sh:.3e}"
        reports[name] = rep
    return reports if isinstance(got, dict) else reports[""]


def format_report(rep) -> str:
    sub = ", ".join(f"{k} y {v[0]:.2e} / state {v[1]:.2e}" for k, v in rep["subsets"].items())
    return (f"y {rep['y']:.2e}, state {rep['state']:.2e}; worst channel {rep['worst_channel']}: "
            f"y {rep['worst_y']:.2e} (against the unrounded oracle), state worst {rep['worst_state']:.2e}"
            + (f"; {sub}" if sub else ""))
