"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle,
element by element on the same seeded inputs.

Small cases cover every channel and span several pipeline stages with a ragged
tail; the four GPU workload shapes run at full size in the launch configuration
the benchmark uses and are compared on every (sequence, channel), in blocks
that fit host memory.
"""
import numpy as np
import pytest
import torch

from parity_util import TOL, all_channels, compare, compare_full, gather, oracle_prefill, rel_l2, round_io
from selective_state_space_depthwise_b200 import api
from selective_state_space_depthwise_b200 import workloads as W

pytestmark = pytest.mark.gpu

# (kernel, G, channels per CTA): kernel 1 = channel tiles, kernel 2 = state slices (32 channels per CTA)
SHAPES = [(1, 1, 32), (1, 1, 64), (1, 1, 128), (1, 2, 16), (1, 2, 32), (1, 2, 64), (1, 4, 8), (1, 4, 16), (1, 4, 32),
          (1, 8, 8), (1, 8, 16), (1, 8, 32), (2, 2, 0), (2, 4, 0), (2, 8, 0), (3, 4, 0), (3, 8, 0), (4, 4, 0)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def small_workload(io_dtype, b=2, L=200, E=48, seed=11, **kw):
    return W.Workload("small", batch=b, seqlen=L, d_inner=E, io_dtype=io_dtype, seed=seed, **kw)


def run_prefill(inp, **kw):
    y, cc, st = api.prefill(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp, **kw)
    torch.cuda.synchronize()
    return y, cc, st


def device_inputs(w, gen_device="cpu"):
    return W.make_inputs(w, device="cuda", gen_device=gen_device)


@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"k{k}_G{g}_N{n}" for k, g, n in SHAPES])
def test_prefill_every_launch_shape(io_dtype, shape):
    # E = 48 leaves a ragged channel tile for N >= 32; L = 200 leaves a ragged stage.
    w = small_workload(io_dtype)
    inp = device_inputs(w)
    k, g, n = shape
    y, cc, st = run_prefill(inp, tuning={"kernel": k, "threads_per_channel": g, "channels_per_cta": n})
    chans = all_channels(w.batch, w.d_inner)
    compare(io_dtype, gather(y, cc, st, chans), oracle_prefill(inp, chans), label=f"kernel {k} G{g} N{n}")


POLY = [(1, 1, 32, 1), (1, 1, 32, 3), (1, 1, 64, 2), (1, 1, 128, 1), (2, 2, 0, 1), (2, 2, 0, 2), (2, 4, 0, 1)]


@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", POLY, ids=[f"k{k}_G{g}_N{n}_p{p}" for k, g, n, p in POLY])
def test_prefill_fma_pipe_exp2_variants(io_dtype, shape):
    """Launch shapes where some decays use the FMA-pipe exp2 polynomial."""
    w = small_workload(io_dtype, b=2, L=150, E=64, seed=13)
    inp = device_inputs(w)
    k, g, n, p = shape
    y, cc, st = run_prefill(inp, tuning={"kernel": k, "threads_per_channel": g, "channels_per_cta": n, "poly_pairs": p})
    chans = all_channels(w.batch, w.d_inner)
    compare(io_dtype, gather(y, cc, st, chans), oracle_prefill(inp, chans), label=f"poly {shape}")


@pytest.mark.parametrize("kg", [(2, 2), (2, 4), (2, 8), (3, 4), (3, 8), (4, 4)])
def test_slice_kernel_lengths_history_and_zoh(kg):
    """The state-slice kernels on short sequences, with incoming caches, and ZOH."""
    kern, g = kg
    for L, E, disc in ((1, 32, "euler"), (3, 40, "euler"), (33, 64, "zoh"), (97, 32, "euler")):
        w = small_workload(torch.bfloat16, b=2, L=L, E=E, seed=90 + L)
        inp = device_inputs(w)
        gen = torch.Generator(device="cpu").manual_seed(5)
        cc_in = torch.randn((2, 3, E), generator=gen).to(torch.bfloat16).cuda()
        st_in = torch.randn((2, E, 16), generator=gen).cuda()
        y, cc, st = run_prefill(inp, conv_cache_in=cc_in, ssm_state_in=st_in, discretization=disc,
                                tuning={"kernel": kern, "threads_per_channel": g})
        chans = all_channels(2, E)
        want = oracle_prefill(inp, chans, conv_cache_in=cc_in, ssm_state_in=st_in, disc=disc)
        compare(torch.bfloat16, gather(y, cc, st, chans), want, label=f"kernel {kern} G{g} L{L} {disc}")


def test_tiny_workload_fp32_full():
    w = W.WORKLOADS["tiny"]
    inp = device_inputs(w)
    y, cc, st = run_prefill(inp)
    chans = all_channels(w.batch, w.d_inner)
    e_y, e_h = compare(torch.float32, gather(y, cc, st, chans), oracle_prefill(inp, chans), label="tiny")
    print(f"tiny fp32: y rel-L2 {e_y:.2e}, state rel-L2 {e_h:.2e}")


@pytest.mark.parametrize("L", [0, 1, 2, 3, 4, 63, 64, 65, 130])
@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
def test_prefill_lengths_and_history(L, io_dtype):
    """Short sequences (L < K-1 included), stage boundaries, and a non-zero
    incoming cache and state."""
    w = small_workload(io_dtype, b=2, L=L, E=16, seed=20 + L)
    inp = device_inputs(w)
    g = torch.Generator(device="cpu").manual_seed(99)
    cc_in = torch.randn((2, 3, 16), generator=g).to(io_dtype).cuda()
    st_in = torch.randn((2, 16, 16), generator=g).cuda()
    chans = all_channels(2, 16)
    for kw in ({}, {"conv_cache_in": cc_in, "ssm_state_in": st_in}):
        y, cc, st = run_prefill(inp, **kw)
        want = oracle_prefill(inp, chans, conv_cache_in=kw.get("conv_cache_in"), ssm_state_in=kw.get("ssm_state_in"))
        if L == 0:
            assert y.numel() == 0
            np.testing.assert_array_equal(gather(y, cc, st, chans)[1], want[2])
            np.testing.assert_array_equal(gather(y, cc, st, chans)[2], want[1])
        else:
            compare(io_dtype, gather(y, cc, st, chans), want, label=f"L={L} {sorted(kw)}")


@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
def test_chained_prefill_equals_one_prefill(io_dtype):
    """A sequence processed in three pieces through the *_in caches gives the
    one-call result (the chunk carry across calls)."""
    w = small_workload(io_dtype, b=2, L=300, E=32, seed=31)
    inp = device_inputs(w)
    y_full, cc_full, st_full = run_prefill(inp)
    cuts = [0, 70, 71, 300]
    cc, st, ys = None, None, []
    for a, b in zip(cuts[:-1], cuts[1:]):
        piece = {k: (v[:, a:b] if k in ("x", "z", "B", "C", "dt_raw") else v) for k, v in inp.items()}
        y, cc, st = run_prefill(piece, conv_cache_in=cc, ssm_state_in=st)
        ys.append(y)
    y_cat = torch.cat(ys, dim=1)
    assert torch.equal(cc, cc_full)
    assert rel_l2(y_cat.double().cpu().numpy(), y_full.double().cpu().numpy()) <= TOL[io_dtype] / 4
    assert rel_l2(st.double().cpu().numpy(), st_full.double().cpu().numpy()) <= 1e-6


def test_fused_in_proj_buffer_strides():
    """x and z as the two halves of one [b, L, 2E] buffer; y written into a
    strided view of a wider output."""
    b, L, E = 2, 150, 64
    w = small_workload(torch.bfloat16, b=b, L=L, E=E, seed=41)
    inp = device_inputs(w)
    buf = torch.cat([inp["x"], inp["z"]], dim=2).contiguous()
    x, z = buf[:, :, :E], buf[:, :, E:]
    out_buf = torch.zeros((b, L, E + 16), dtype=torch.bfloat16, device="cuda")
    y = out_buf[:, :, 8:8 + E]
    y2, cc, st = api.prefill(x, z, inp["B"], inp["C"], inp["dt_raw"], inp, y=y)
    torch.cuda.synchronize()
    assert y2.data_ptr() == y.data_ptr()
    assert torch.count_nonzero(out_buf[:, :, :8]) == 0 and torch.count_nonzero(out_buf[:, :, 8 + E:]) == 0
    chans = all_channels(b, E)
    compare(torch.bfloat16, gather(y, cc, st, chans), oracle_prefill(inp, chans), label="fused")


@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
def test_zoh_discretisation(io_dtype):
    w = small_workload(io_dtype, b=1, L=160, E=32, seed=51)
    inp = device_inputs(w)
    y, cc, st = run_prefill(inp, discretization="zoh")
    chans = all_channels(1, 32)
    compare(io_dtype, gather(y, cc, st, chans), oracle_prefill(inp, chans, disc="zoh"), label="zoh")


def decode_run(inp, w, L0, steps, disc="euler", stride_view=True):
    """Prefill L0 tokens, then `steps` decode calls reading token L0+i of the
    same [b, T, *] tensors (strided views). Returns stacked y [b, L0+steps, E]."""
    y0, cc, st = run_prefill({**inp, **{k: inp[k][:, :L0] for k in ("x", "z", "B", "C", "dt_raw")}},
                             discretization=disc)
    b, E = w.batch, w.d_inner
    y = torch.empty((b, L0 + steps, E), dtype=w.io_dtype, device="cuda")
    y[:, :L0] = y0
    for i in range(steps):
        t = L0 + i
        api.decode_step(inp["x"][:, t], inp["z"][:, t], inp["B"][:, t], inp["C"][:, t], inp["dt_raw"][:, t], inp,
                        cc, st, y=y[:, t], discretization=disc)
    torch.cuda.synchronize()
    return y, cc, st


@pytest.mark.parametrize("L0", [0, 2, 5, 64])
@pytest.mark.parametrize("io_dtype", [torch.float32, torch.bfloat16])
def test_decode_continues_prefill(L0, io_dtype):
    steps = 9
    w = small_workload(io_dtype, b=3, L=L0 + steps, E=24 if io_dtype == torch.float32 else 40, seed=60 + L0)
    inp = device_inputs(w)
    y, cc, st = decode_run(inp, w, L0, steps)
    chans = all_channels(w.batch, w.d_inner)
    compare(io_dtype, gather(y, cc, st, chans), oracle_prefill(inp, chans), label=f"decode L0={L0}")


def test_decode_zoh():
    w = small_workload(torch.bfloat16, b=2, L=20, E=16, seed=71)
    inp = device_inputs(w)
    y, cc, st = decode_run(inp, w, 12, 8, disc="zoh")
    chans = all_channels(2, 16)
    compare(torch.bfloat16, gather(y, cc, st, chans), oracle_prefill(inp, chans, disc="zoh"), label="decode zoh")


# ------------------------------------------------------------ full sizes ---
@pytest.mark.parametrize("name", ["axon_layer", "batched", "long_context"])
def test_full_size_prefill_all_channels(name):
    """The workload at full size, in the default launch shape the benchmark
    times, against the oracle on every (sequence, channel)."""
    w = W.WORKLOADS[name]
    inp = device_inputs(w, gen_device="cuda")
    y, cc, st = run_prefill(inp)
    e_y, e_h = compare_full(w.io_dtype, inp, (y, cc, st), label=name)
    print(f"{name}: y rel-L2 {e_y:.2e}, state rel-L2 {e_h:.2e} over all {w.batch * w.d_inner} channels")


def test_full_size_decode_all_channels():
    """Prompt 512, then 1024 decode steps, against one oracle prefill of 1536,
    on every (sequence, channel)."""
    w = W.WORKLOADS["decode"]
    inp = device_inputs(w, gen_device="cuda")
    y, cc, st = decode_run(inp, w, w.seqlen, w.decode_steps)
    e_y, e_h = compare_full(w.io_dtype, inp, (y, cc, st), label="decode")
    print(f"decode: y rel-L2 {e_y:.2e}, state rel-L2 {e_h:.2e} over all {w.batch * w.d_inner} channels")
