"""CPU checks of the C ABI: the library builds and loads, exports every
function include/ssm.h declares, and rejects bad arguments on the host before
any CUDA call (no kernel runs here)."""
import ctypes
import os
import re

import pytest
import torch

from selective_state_space_depthwise_b200 import _lib, api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(ssm_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_surface():
    assert declared_functions() == sorted(_lib.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version(lib):
    assert lib.ssm_status_string(0) == b"ok"
    assert b"invalid" in lib.ssm_status_string(1)
    assert b"unsupported" in lib.ssm_status_string(2)
    assert lib.ssm_status_string(99) == b"unknown status"
    assert re.fullmatch(rb"\d+\.\d+\.\d+", lib.ssm_version())


def valid_dims(**kw):
    d = api.make_dims(2, 64, 32, torch.bfloat16)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


FAKE = 0x10000  # a 16-byte-aligned non-null address; never dereferenced on the host


def fake_weights():
    w = _lib.SsmWeights()
    for n in api.PARAM_NAMES:
        setattr(w, n, FAKE)
    return w


def call_prefill(lib, dims, weights, ptrs=None):
    p = dict(x=FAKE, z=FAKE, B=FAKE, C=FAKE, dt=FAKE, cin=None, sin=None, y=FAKE + 4096, cout=FAKE, sout=FAKE)
    p.update(ptrs or {})
    return lib.ssm_prefill(ctypes.byref(dims) if dims is not None else None,
                           ctypes.byref(weights) if weights is not None else None, p["x"], p["z"], p["B"], p["C"],
                           p["dt"], p["cin"], p["sin"], p["y"], p["cout"], p["sout"], None, 0, None)


@pytest.mark.parametrize("case,field,value,status", [
    ("d_state", "d_state", 8, _lib.SSM_ERR_UNSUPPORTED),
    ("d_conv", "d_conv", 3, _lib.SSM_ERR_UNSUPPORTED),
    ("batch", "batch", 0, _lib.SSM_ERR_INVALID_ARG),
    ("seqlen", "seqlen", -1, _lib.SSM_ERR_INVALID_ARG),
    ("d_inner", "d_inner", 12, _lib.SSM_ERR_INVALID_ARG),
    ("dt_min", "dt_min", 0.0, _lib.SSM_ERR_INVALID_ARG),
    ("dt_order", "dt_max", 1e-5, _lib.SSM_ERR_INVALID_ARG),
    ("io_dtype", "io_dtype", 7, _lib.SSM_ERR_INVALID_ARG),
    ("disc", "discretization", 5, _lib.SSM_ERR_INVALID_ARG),
    ("x_tok", "x_tok_stride", 36, _lib.SSM_ERR_INVALID_ARG),
    ("x_tok_small", "x_tok_stride", 16, _lib.SSM_ERR_INVALID_ARG),
    ("bc_tok", "bc_tok_stride", 8, _lib.SSM_ERR_INVALID_ARG),
    ("bc_seq", "bc_seq_stride", 18, _lib.SSM_ERR_INVALID_ARG),
])
def test_prefill_rejects_bad_dims(lib, case, field, value, status):
    assert call_prefill(lib, valid_dims(**{field: value}), fake_weights()) == status
    assert lib.ssm_last_error() != b""


def test_prefill_rejects_bad_pointers(lib):
    d, w = valid_dims(), fake_weights()
    assert call_prefill(lib, None, w) == _lib.SSM_ERR_INVALID_ARG
    assert call_prefill(lib, d, None) == _lib.SSM_ERR_INVALID_ARG
    for k in ("x", "z", "B", "C", "dt", "y", "cout", "sout"):
        assert call_prefill(lib, d, w, {k: None}) == _lib.SSM_ERR_INVALID_ARG, k
        assert b"NULL" in lib.ssm_last_error(), k
    for k in ("x", "z", "B", "C", "y", "cout"):
        assert call_prefill(lib, d, w, {k: FAKE + 2}) == _lib.SSM_ERR_INVALID_ARG, k
    assert call_prefill(lib, d, w, {"y": FAKE}) == _lib.SSM_ERR_INVALID_ARG  # y aliases x
    w2 = fake_weights()
    w2.A_log = None
    assert call_prefill(lib, d, w2) == _lib.SSM_ERR_INVALID_ARG
    assert b"A_log" in lib.ssm_last_error()


def test_decode_rejects_bad_arguments(lib):
    w = fake_weights()
    d = valid_dims(d_state=32)
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4096, FAKE, FAKE, None]
    assert lib.ssm_decode_step(ctypes.byref(d), ctypes.byref(w), *args) == _lib.SSM_ERR_UNSUPPORTED
    d = valid_dims()
    bad = list(args)
    bad[7] = FAKE + 4  # ssm_state must be 16-byte aligned
    assert lib.ssm_decode_step(ctypes.byref(d), ctypes.byref(w), *bad) == _lib.SSM_ERR_INVALID_ARG
    bad = list(args)
    bad[5] = FAKE  # y aliases x
    assert lib.ssm_decode_step(ctypes.byref(d), ctypes.byref(w), *bad) == _lib.SSM_ERR_INVALID_ARG


def test_workspace_is_zero_for_the_single_pass_kernel(lib):
    assert lib.ssm_prefill_workspace_bytes(ctypes.byref(valid_dims())) == 0
    assert lib.ssm_prefill_workspace_bytes(None) == 0


def test_binding_refuses_cpu_tensors(lib):
    x = torch.zeros(1, 8, 8, dtype=torch.bfloat16)
    p = {n: torch.zeros(8, 4) if n == "conv_w" else torch.zeros(8, 16) if n == "A_log" else torch.zeros(8)
         for n in api.PARAM_NAMES}
    with pytest.raises(RuntimeError, match="no CPU path"):
        api.prefill(x, x, torch.zeros(1, 8, 16), torch.zeros(1, 8, 16), torch.zeros(1, 8), p)
    with pytest.raises(RuntimeError, match="no CPU path"):
        api.segment_summary(x, torch.zeros(1, 8, 16), torch.zeros(1, 8), p)
    with pytest.raises(RuntimeError, match="no CPU path"):
        api.segment_carry(torch.zeros(1, 1, 17, 8), p)


def test_host_workspace_bytes_cover_two_chunk_slots(lib):
    def slot(b, T, E, es):
        al = lambda v: (v + 255) // 256 * 256  # noqa: E731
        return 3 * al(b * T * E * es) + 2 * al(b * T * 64) + al(b * T * 4)

    d = valid_dims()  # b=2, L=64, E=32, bf16
    assert lib.ssm_prefill_host_workspace_bytes(ctypes.byref(d), 16) == 2 * slot(2, 16, 32, 2)
    # chunk 0 selects 4096 tokens, clipped to the sequence length
    assert lib.ssm_prefill_host_workspace_bytes(ctypes.byref(d), 0) == 2 * slot(2, 64, 32, 2)
    assert lib.ssm_prefill_host_workspace_bytes(ctypes.byref(d), 1000) == 2 * slot(2, 64, 32, 2)
    d32 = api.make_dims(1, 5000, 64, torch.float32)
    assert lib.ssm_prefill_host_workspace_bytes(ctypes.byref(d32), 0) == 2 * slot(1, 4096, 64, 4)
    assert lib.ssm_prefill_host_workspace_bytes(ctypes.byref(d), -1) == 0
    assert lib.ssm_prefill_host_workspace_bytes(ctypes.byref(valid_dims(d_state=8)), 16) == 0
    assert lib.ssm_prefill_host_workspace_bytes(None, 16) == 0


def call_prefill_host(lib, dims, weights, ptrs=None, ws_bytes=1 << 20, chunk=16):
    p = dict(x=FAKE, z=FAKE, B=FAKE, C=FAKE, dt=FAKE, cin=None, sin=None, y=FAKE + 4096, cout=FAKE, sout=FAKE,
             ws=FAKE)
    p.update(ptrs or {})
    return lib.ssm_prefill_host(ctypes.byref(dims) if dims is not None else None,
                                ctypes.byref(weights) if weights is not None else None, p["x"], p["z"], p["B"], p["C"],
                                p["dt"], p["cin"], p["sin"], p["y"], p["cout"], p["sout"], p["ws"], ws_bytes, chunk,
                                None)


def test_prefill_host_rejects_bad_arguments_before_any_work(lib):
    d, w = valid_dims(), fake_weights()
    assert call_prefill_host(lib, valid_dims(d_state=8), w) == _lib.SSM_ERR_UNSUPPORTED
    assert call_prefill_host(lib, d, None) == _lib.SSM_ERR_INVALID_ARG
    assert call_prefill_host(lib, d, w, chunk=-3) == _lib.SSM_ERR_INVALID_ARG
    assert b"chunk_tokens" in lib.ssm_last_error()
    for k in ("x", "z", "B", "C", "dt", "y", "cout", "sout", "ws"):
        assert call_prefill_host(lib, d, w, {k: None}) == _lib.SSM_ERR_INVALID_ARG, k
        assert b"NULL" in lib.ssm_last_error(), k
    assert call_prefill_host(lib, d, w, {"y": FAKE}) == _lib.SSM_ERR_INVALID_ARG  # y aliases x
    assert call_prefill_host(lib, d, w, {"ws": FAKE + 16}) == _lib.SSM_ERR_INVALID_ARG  # not 256-byte aligned
    need = lib.ssm_prefill_host_workspace_bytes(ctypes.byref(d), 16)
    assert call_prefill_host(lib, d, w, ws_bytes=need - 1) == _lib.SSM_ERR_INVALID_ARG
    assert b"workspace" in lib.ssm_last_error()


def test_host_binding_refuses_host_parameters(lib):
    x = torch.zeros(1, 8, 8, dtype=torch.bfloat16)
    p = {n: torch.zeros(8, 4) if n == "conv_w" else torch.zeros(8, 16) if n == "A_log" else torch.zeros(8)
         for n in api.PARAM_NAMES}
    with pytest.raises(RuntimeError, match="CUDA tensor"):
        api.prefill_host(x, x, torch.zeros(1, 8, 16), torch.zeros(1, 8, 16), torch.zeros(1, 8), p,
                         conv_cache_out=torch.zeros(1, 3, 8, dtype=torch.bfloat16))


def test_block_forward_rejects_bad_arguments_before_any_work(lib):
    w = fake_weights()
    pw = _lib.SsmBlockWeights(FAKE, FAKE, FAKE)
    ws_need = lib.ssm_block_workspace_bytes(ctypes.byref(api.make_block_dims(2, 64, 32, 64)))
    assert ws_need > 0

    def call(dims, proj=pw, hidden=FAKE, out=FAKE + 4096, ws=FAKE, ws_bytes=ws_need):
        return lib.ssm_block_forward(ctypes.byref(dims) if dims is not None else None, ctypes.byref(w),
                                     ctypes.byref(proj) if proj is not None else None, hidden, None, None, out, FAKE,
                                     FAKE, ws, ws_bytes, None)

    d = api.make_block_dims(2, 64, 32, 64)
    d32 = api.make_block_dims(2, 64, 32, 64)
    d32.io_dtype = _lib.SSM_F32
    assert call(d32) == _lib.SSM_ERR_UNSUPPORTED
    assert b"bf16" in lib.ssm_last_error()
    assert call(None) == _lib.SSM_ERR_INVALID_ARG
    bad = api.make_block_dims(2, 64, 30, 64)  # d_model not a multiple of 8
    assert call(bad) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, proj=None) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, proj=_lib.SsmBlockWeights(FAKE, None, FAKE)) == _lib.SSM_ERR_INVALID_ARG
    assert b"w_x" in lib.ssm_last_error()
    assert call(d, hidden=None) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, out=FAKE) == _lib.SSM_ERR_INVALID_ARG  # out aliases hidden
    assert call(d, ws_bytes=ws_need - 1) == _lib.SSM_ERR_INVALID_ARG
    assert lib.ssm_block_workspace_bytes(ctypes.byref(d32)) == 0


def test_segment_summary_workspace_and_argument_checks(lib):
    d = valid_dims()  # b=2, T=64, E=32
    assert lib.ssm_segment_summary_workspace_bytes(ctypes.byref(d)) == 2 * 1 * 17 * 32 * 4
    d300 = valid_dims(seqlen=300)
    assert lib.ssm_segment_summary_workspace_bytes(ctypes.byref(d300)) == 2 * 2 * 17 * 32 * 4
    assert lib.ssm_segment_summary_workspace_bytes(ctypes.byref(valid_dims(seqlen=0))) == 0
    assert lib.ssm_segment_summary_workspace_bytes(None) == 0
    w = fake_weights()
    ws = lib.ssm_segment_summary_workspace_bytes(ctypes.byref(d))

    def call(dims, x=FAKE, B=FAKE, dt=FAKE, cin=None, summ=FAKE, work=FAKE + 8192, nbytes=ws):
        return lib.ssm_segment_summary(ctypes.byref(dims) if dims else None, ctypes.byref(w), x, B, dt, cin, summ,
                                       work, nbytes, None)

    assert call(None) == _lib.SSM_ERR_INVALID_ARG
    assert call(valid_dims(d_state=8)) == _lib.SSM_ERR_UNSUPPORTED
    for k in ("x", "B", "dt", "summ"):
        assert call(d, **{k: None}) == _lib.SSM_ERR_INVALID_ARG, k
        assert b"NULL" in lib.ssm_last_error(), k
    assert call(d, summ=FAKE + 4) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, cin=FAKE + 2) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, nbytes=ws - 4) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, work=None) == _lib.SSM_ERR_INVALID_ARG
    assert b"workspace" in lib.ssm_last_error()


def test_segment_carry_argument_checks(lib):
    d, w = valid_dims(), fake_weights()

    def call(dims, summ=FAKE, count=2, sin=None, sout=FAKE):
        return lib.ssm_segment_carry(ctypes.byref(dims) if dims else None, ctypes.byref(w), summ, count, sin, sout,
                                     None)

    assert call(None) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, count=-1) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, summ=None) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, sout=None) == _lib.SSM_ERR_INVALID_ARG
    assert call(d, sin=FAKE + 2) == _lib.SSM_ERR_INVALID_ARG
    assert call(valid_dims(d_conv=3)) == _lib.SSM_ERR_UNSUPPORTED


def test_selftest_rejects_bad_limits_on_the_host(lib):
    for bad in (0, 999, 2_000_000_001):
        assert lib.ssm_selftest_bounded_wait(bad, None) == _lib.SSM_ERR_INVALID_ARG


def test_prefill_kernel_choice_on_the_host(lib):
    """The automatic launch shape, on the host for a 148-SM GPU: kernel 5 up
    to one CTA (32 channels of one sequence) per SM; kernel 4 up to 64 CTAs
    per SM, unless every CTA runs per-state exponentials (ZOH, or decay_path
    1), where kernel 5 stays; kernel 3 beyond; an explicit kernel wins; a
    rejected tuning or shape gives 0."""
    k = lambda b, E, **kw: api.prefill_kernel(b, 1024, E, num_sms=148, **kw)
    assert k(1, 32) == 5 and k(1, 4736) == 5 and k(2, 2368) == 5  # 1, 148, 148 CTAs
    assert k(1, 4768) == 4 and k(1, 7680) == 4 and k(8, 5120) == 4  # 149, 240, 1280 CTAs
    assert k(1, 7680, discretization="zoh") == 5
    assert k(1, 7680, tuning={"decay_path": 1}) == 5
    assert k(64 * 148, 32) == 4 and k(64 * 148 + 1, 32) == 3
    assert k(64 * 148 + 1, 32, discretization="zoh") == 3
    assert k(256, 7680) == 3  # the decode prompt's 61440 CTAs
    assert k(1, 7680, tuning={"kernel": 3}) == 3 and k(1, 32, tuning={"kernel": 4}) == 4
    assert k(1, 7680, tuning={"kernel": 2}) == 0
    assert k(1, 7680, tuning={"decay_path": 2}) == 0
    assert k(1, 7684) == 0  # E not a multiple of 8
    assert api.prefill_kernel(1, 1024, 7680, num_sms=74) == 4 and api.prefill_kernel(1, 1024, 2368, num_sms=74) == 5
