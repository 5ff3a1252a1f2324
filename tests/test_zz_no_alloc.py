"""ssm_prefill_host_static: the host-memory prefill with its chunk buffers in the
library's static device scratch, so a call takes no workspace and allocates
nothing.

GPU: it equals the device prefill bit for bit (ragged chunks, the automatic
chunk, incoming caches, ZOH, fp32); calls issued back to back on two streams
share the scratch correctly; after the first call on a device, further calls
change neither the device's free memory nor PyTorch's allocation. CPU: argument
errors, including chunks that do not fit the scratch, return before any CUDA
call.
"""
import ctypes

import pytest
import torch

from selective_state_space_depthwise_b200 import _lib, api, build
from selective_state_space_depthwise_b200 import workloads as W

TOKEN_KEYS = ("x", "z", "B", "C", "dt_raw")
FAKE = 0x10000  # 16-byte-aligned, never dereferenced on the host


def inputs(io_dtype, b, L, E, seed):
    w = W.Workload("static", batch=b, seqlen=L, d_inner=E, io_dtype=io_dtype, seed=seed)
    return W.make_inputs(w, device="cuda")


def host_copy(inp):
    return {k: inp[k].to("cpu").pin_memory() for k in TOKEN_KEYS}


def run_static(inp, host, chunk=0, stream=None, **kw):
    return api.prefill_host(host["x"], host["z"], host["B"], host["C"], host["dt_raw"], inp, chunk_tokens=chunk,
                            static_scratch=True, stream=stream, **kw)


def run_device(inp, **kw):
    y, cc, st = api.prefill(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp, **kw)
    torch.cuda.synchronize()
    return y, cc, st


@pytest.mark.gpu
@pytest.mark.parametrize("io_dtype,b,L,E,chunk,with_caches,disc", [
    (torch.bfloat16, 2, 300, 64, 0, False, "euler"),   # automatic chunk (here: the whole sequence)
    (torch.bfloat16, 3, 333, 48, 100, True, "euler"),  # ragged last chunk, incoming caches
    (torch.float32, 1, 90, 32, 7, True, "zoh"),
])
def test_static_host_prefill_equals_device_prefill(io_dtype, b, L, E, chunk, with_caches, disc):
    inp = inputs(io_dtype, b, L, E, seed=L)
    cin = sin = None
    if with_caches:
        g = torch.Generator(device="cpu").manual_seed(L)
        cin = (torch.randn((b, 3, E), generator=g) * 0.5).to(io_dtype).cuda()
        sin = (torch.randn((b, E, 16), generator=g) * 0.1).cuda()
    want = run_device(inp, conv_cache_in=cin, ssm_state_in=sin, discretization=disc)
    y, cc, st = run_static(inp, host_copy(inp), chunk, conv_cache_in=cin, ssm_state_in=sin, discretization=disc)
    torch.cuda.synchronize()
    assert torch.equal(y, want[0].cpu()) and torch.equal(cc, want[1]) and torch.equal(st, want[2])


@pytest.mark.gpu
def test_static_host_prefill_full_size_layer_shape():
    """The Axon layer shape (b=1, L=2048, E=7680): the automatic chunk is cut to
    what fits the scratch (about 1450 tokens), so the sequence runs in two chunks."""
    w = W.WORKLOADS["axon_layer"]
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    want = run_device(inp)
    y, cc, st = run_static(inp, host_copy(inp))
    torch.cuda.synchronize()
    assert torch.equal(y, want[0].cpu()) and torch.equal(cc, want[1]) and torch.equal(st, want[2])


@pytest.mark.gpu
def test_calls_on_two_streams_share_the_scratch_in_order():
    a = inputs(torch.bfloat16, 2, 400, 64, seed=1)
    b = inputs(torch.bfloat16, 2, 400, 64, seed=2)
    want_a, want_b = run_device(a), run_device(b)
    ha, hb = host_copy(a), host_copy(b)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    ya, cca, sta = run_static(a, ha, 64, stream=s1)
    yb, ccb, stb = run_static(b, hb, 64, stream=s2)  # no synchronisation in between
    torch.cuda.synchronize()
    assert torch.equal(ya, want_a[0].cpu()) and torch.equal(sta, want_a[2]) and torch.equal(cca, want_a[1])
    assert torch.equal(yb, want_b[0].cpu()) and torch.equal(stb, want_b[2]) and torch.equal(ccb, want_b[1])


@pytest.mark.gpu
def test_steady_state_calls_allocate_nothing():
    b, L, E = 2, 512, 64
    inp = inputs(torch.bfloat16, b, L, E, seed=5)
    host = host_copy(inp)
    y = torch.empty((b, L, E), dtype=torch.bfloat16).pin_memory()
    cc = torch.empty((b, 3, E), dtype=torch.bfloat16, device="cuda")
    st = torch.empty((b, E, 16), dtype=torch.float32, device="cuda")
    run_static(inp, host, 128, y=y, conv_cache_out=cc, ssm_state_out=st)  # first call: loads, creates streams/events
    torch.cuda.synchronize()
    free0, torch0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(5):
        run_static(inp, host, 128, y=y, conv_cache_out=cc, ssm_state_out=st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == torch0


@pytest.mark.gpu
def test_chunk_that_does_not_fit_is_refused():
    inp = inputs(torch.bfloat16, 1, 4200, 7680, seed=9)  # longer than the chunk, so it is not clipped to L
    host = host_copy(inp)
    with pytest.raises(_lib.SsmError) as e:
        run_static(inp, host, 4096)  # 2 slots x 4096 tokens x 7680 x 6 B > 128 MiB
    assert e.value.status == _lib.SSM_ERR_INVALID_ARG


# ------------------------------------------------------------------ CPU ----
def _weights():
    w = _lib.SsmWeights()
    for n in api.PARAM_NAMES:
        setattr(w, n, FAKE)
    return w


def _call(lib, dims, ptrs=None, chunk=16):
    p = dict(x=FAKE, z=FAKE, B=FAKE, C=FAKE, dt=FAKE, y=FAKE + 4096, cout=FAKE, sout=FAKE)
    p.update(ptrs or {})
    w = _weights()
    return lib.ssm_prefill_host_static(ctypes.byref(dims), ctypes.byref(w), p["x"], p["z"], p["B"], p["C"], p["dt"],
                                       None, None, p["y"], p["cout"], p["sout"], chunk, None)


def test_static_entry_point_rejects_bad_arguments_on_the_host():
    build.build()
    lib = _lib.load()
    d = api.make_dims(2, 64, 32, torch.bfloat16)
    for k in ("x", "z", "B", "C", "dt", "y", "cout", "sout"):
        assert _call(lib, d, {k: None}) == _lib.SSM_ERR_INVALID_ARG, k
    assert _call(lib, d, {"y": FAKE}) == _lib.SSM_ERR_INVALID_ARG  # y aliases x
    assert _call(lib, d, chunk=-1) == _lib.SSM_ERR_INVALID_ARG
    big = api.make_dims(1, 100000, 8192, torch.bfloat16)
    assert _call(lib, big, chunk=8192) == _lib.SSM_ERR_INVALID_ARG  # 2 x 8192 x 8192 x 6 B > 128 MiB
    assert b"static scratch" in lib.ssm_last_error()
    huge = api.make_dims(4096, 100, 8192, torch.bfloat16)  # one token of every sequence already exceeds it
    assert _call(lib, huge, chunk=0) == _lib.SSM_ERR_UNSUPPORTED
