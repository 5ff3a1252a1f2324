"""GPU tests of ssm_prefill_host: prefill with the token tensors in host memory,
chunked, with the copies overlapped on the library's own streams.

Chunking with carried caches runs the same per-token arithmetic as one launch,
so the host path must equal the device path (api.prefill) bit for bit, for every
chunk size, ragged last chunk, strided host layout, discretisation and io
dtype. One case is also compared with the oracle directly, and the bench's
long-context workload runs at full size.
"""
import pytest
import torch

from parity_util import all_channels, compare, gather, oracle_prefill
from selective_state_space_depthwise_b200 import _lib, api
from selective_state_space_depthwise_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOKEN_KEYS = ("x", "z", "B", "C", "dt_raw")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def inputs(io_dtype, b, L, E, seed):
    w = W.Workload("host", batch=b, seqlen=L, d_inner=E, io_dtype=io_dtype, seed=seed)
    return W.make_inputs(w, device="cuda")


def host_copy(inp, pin=True):
    out = {}
    for k in TOKEN_KEYS:
        t = inp[k].to("cpu")
        out[k] = t.pin_memory() if pin else t
    return out


def run_host(inp, host, chunk, **kw):
    y, cc, st = api.prefill_host(host["x"], host["z"], host["B"], host["C"], host["dt_raw"], inp, chunk_tokens=chunk,
                                 **kw)
    torch.cuda.synchronize()
    return y, cc, st


def run_device(inp, **kw):
    y, cc, st = api.prefill(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp, **kw)
    torch.cuda.synchronize()
    return y, cc, st


def caches_in(inp, b, E, io_dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    cc = (torch.randn((b, 3, E), generator=g) * 0.5).to(io_dtype).cuda()
    st = (torch.randn((b, E, 16), generator=g) * 0.1).cuda()
    return cc, st


@pytest.mark.parametrize("io_dtype,b,L,E,chunk,with_caches,disc", [
    (torch.float32, 1, 64, 32, 7, False, "euler"),     # ragged chunks, several stages each
    (torch.bfloat16, 3, 300, 64, 128, True, "euler"),  # ragged last chunk, incoming caches
    (torch.bfloat16, 2, 100, 32, 1, False, "euler"),   # one token per chunk: 100 chunks, events reused
    (torch.bfloat16, 2, 257, 48, 0, True, "zoh"),      # default chunk longer than L: one chunk
    (torch.float32, 2, 200, 40, 64, True, "zoh"),
])
def test_host_prefill_equals_device_prefill(io_dtype, b, L, E, chunk, with_caches, disc):
    inp = inputs(io_dtype, b, L, E, seed=100 + L)
    cin, sin = caches_in(inp, b, E, io_dtype, seed=L) if with_caches else (None, None)
    want = run_device(inp, conv_cache_in=cin, ssm_state_in=sin, discretization=disc)
    got = run_host(inp, host_copy(inp), chunk, conv_cache_in=cin, ssm_state_in=sin, discretization=disc)
    assert not got[0].is_cuda
    assert torch.equal(got[0], want[0].cpu()), "y differs from the one-launch result"
    assert torch.equal(got[1], want[1]), "conv_cache_out differs"
    assert torch.equal(got[2], want[2]), "ssm_state_out differs"


def test_host_prefill_strided_host_layouts():
    """x and z as halves of one [b, L, 2E] pinned host buffer, B and C inside
    one [b, L, 40] buffer, dt_raw with a padded sequence stride, y written into
    a strided view of a wider host buffer."""
    b, L, E = 2, 150, 64
    inp = inputs(torch.bfloat16, b, L, E, seed=7)
    want = run_device(inp)
    xz = torch.cat([inp["x"], inp["z"]], dim=2).cpu().pin_memory()
    bc = torch.zeros((b, L, 40), dtype=torch.float32).pin_memory()
    bc[:, :, 0:16] = inp["B"].cpu()
    bc[:, :, 16:32] = inp["C"].cpu()
    dtb = torch.zeros((b, L + 5), dtype=torch.float32).pin_memory()
    dtb[:, :L] = inp["dt_raw"].cpu()
    out = torch.zeros((b, L, E + 16), dtype=torch.bfloat16).pin_memory()
    y = out[:, :, 8:8 + E]
    got = api.prefill_host(xz[:, :, :E], xz[:, :, E:], bc[:, :, 0:16], bc[:, :, 16:32], dtb[:, :L], inp, y=y,
                           chunk_tokens=48)
    torch.cuda.synchronize()
    assert got[0].data_ptr() == y.data_ptr()
    assert torch.count_nonzero(out[:, :, :8]) == 0 and torch.count_nonzero(out[:, :, 8 + E:]) == 0
    assert torch.equal(y, want[0].cpu())
    assert torch.equal(got[1], want[1]) and torch.equal(got[2], want[2])


@pytest.mark.parametrize("static", [False, True])
@pytest.mark.parametrize("which", ["y", "x", "dt_raw"])
def test_host_prefill_rejects_pageable_buffers(which, static):
    """A pageable host buffer (here y, x or dt_raw) is refused with
    SSM_ERR_INVALID_ARG before anything is enqueued, on both host entry points."""
    b, L, E = 1, 40, 32
    inp = inputs(torch.bfloat16, b, L, E, seed=9)
    host = host_copy(inp)
    y = torch.empty((b, L, E), dtype=torch.bfloat16).pin_memory()
    if which == "y":
        y = torch.empty((b, L, E), dtype=torch.bfloat16)
    else:
        host[which] = host[which].clone()  # clone of a pinned tensor is pageable
    assert not (y if which == "y" else host[which]).is_pinned()
    with pytest.raises(_lib.SsmError) as err:
        api.prefill_host(host["x"], host["z"], host["B"], host["C"], host["dt_raw"], inp, y=y, chunk_tokens=16,
                         static_scratch=static)
    assert err.value.status == _lib.SSM_ERR_INVALID_ARG
    assert "page-locked" in str(err.value)


def test_host_prefill_against_the_oracle():
    b, L, E = 2, 230, 32
    inp = inputs(torch.bfloat16, b, L, E, seed=17)
    y, cc, st = run_host(inp, host_copy(inp), 50)
    chans = all_channels(b, E)
    compare(torch.bfloat16, gather(y, cc, st, chans), oracle_prefill(inp, chans), label="host")


def test_host_prefill_zero_length_copies_the_caches():
    b, E = 2, 32
    cin, sin = caches_in(None, b, E, torch.bfloat16, seed=3)
    empty = {k: torch.empty((b, 0, 16) if k in ("B", "C") else (b, 0) if k == "dt_raw" else (b, 0, E),
                            dtype=torch.float32 if k in ("B", "C", "dt_raw") else torch.bfloat16)
             for k in TOKEN_KEYS}
    params = inputs(torch.bfloat16, b, 4, E, seed=3)
    y, cc, st = api.prefill_host(empty["x"], empty["z"], empty["B"], empty["C"], empty["dt_raw"], params,
                                 conv_cache_in=cin, ssm_state_in=sin)
    torch.cuda.synchronize()
    assert y.shape == (b, 0, E)
    assert torch.equal(cc, cin) and torch.equal(st, sin)


def test_host_prefill_long_context_full_size():
    """The bench's long-context workload (b=1, L=65536, E=7680), default chunk,
    against the device path, bit for bit."""
    w = W.WORKLOADS["long_context"]
    inp = W.make_inputs(w, device="cuda", gen_device="cuda")
    y_dev, cc_dev, st_dev = run_device(inp)
    host = host_copy(inp)
    y, cc, st = run_host(inp, host, 0)
    assert torch.equal(y, y_dev.cpu())
    assert torch.equal(cc, cc_dev) and torch.equal(st, st_dev)
