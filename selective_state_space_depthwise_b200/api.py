"""PyTorch-facing calls of the C ABI (include/ssm.h).

Each function reads sizes and strides off the tensors, allocates missing
outputs with torch (device memory is PyTorch's job here), and makes exactly
one C call on the current CUDA stream. Every step of the block core runs in
the library's CUDA kernels; tensors that are not on a CUDA device are
rejected -- there is no CPU path.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

_DTYPES = {torch.float32: _lib.SSM_F32, torch.bfloat16: _lib.SSM_BF16}
_DISC = {"euler": _lib.SSM_DISC_EULER_B, "euler_b": _lib.SSM_DISC_EULER_B, "zoh": _lib.SSM_DISC_ZOH}
PARAM_NAMES = ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(name, t, device):
    if t is None:
        return
    if not t.is_cuda:
        raise RuntimeError(f"{name} must be a CUDA tensor: the block core has no CPU path")
    if t.device != device:
        raise RuntimeError(f"{name} is on {t.device}, expected {device}")


def _weights(params, E, device):
    for n in PARAM_NAMES:
        t = params[n]
        _need_cuda(n, t, device)
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous float32")
    if params["conv_w"].shape != (E, 4) or params["A_log"].shape != (E, 16):
        raise ValueError("conv_w must be [E, 4] and A_log [E, 16]")
    for n in ("conv_b", "w_dt", "dt_bias", "D"):
        if params[n].shape != (E,):
            raise ValueError(f"{n} must be [E]")
    w = _lib.SsmWeights()
    for n in PARAM_NAMES:
        setattr(w, n, params[n].data_ptr())
    return w


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _tuning_ref(tuning):
    """ssm_tuning from a dict {"kernel": k, "decay_path": d} (None: defaults)."""
    if not tuning:
        return None
    unknown = set(tuning) - {"kernel", "decay_path"}
    if unknown:
        raise ValueError(f"unknown tuning keys {sorted(unknown)} (kernel, decay_path)")
    return ctypes.byref(_lib.SsmTuning(int(tuning.get("kernel", 0)), int(tuning.get("decay_path", 0))))


def make_dims(batch, seqlen, E, io_dtype, dt_min=1e-4, dt_max=1.0, discretization="euler", **strides):
    d = _lib.SsmDims()
    d.batch, d.seqlen, d.d_inner, d.d_state, d.d_conv = batch, seqlen, E, 16, 4
    d.dt_min, d.dt_max = dt_min, dt_max
    d.io_dtype = _DTYPES[io_dtype] if isinstance(io_dtype, torch.dtype) else int(io_dtype)
    d.discretization = _DISC[discretization]
    for k, v in strides.items():
        setattr(d, k, int(v))
    return d


def workspace_bytes(batch, seqlen, E, io_dtype=torch.bfloat16) -> int:
    lib = _lib.load()
    return int(lib.ssm_prefill_workspace_bytes(ctypes.byref(make_dims(batch, seqlen, E, io_dtype))))


def prefill_kernel(batch, seqlen, E, io_dtype=torch.bfloat16, discretization="euler", tuning=None,
                   num_sms=0) -> int:
    """The prefill kernel (3, 4 or 5) `prefill` launches for this shape and
    tuning on a GPU of num_sms SMs (0: the current device's); 0 where the call
    would be rejected. Host-only for num_sms > 0."""
    lib = _lib.load()
    dims = make_dims(batch, seqlen, E, io_dtype, discretization=discretization)
    return int(lib.ssm_prefill_kernel(ctypes.byref(dims), _tuning_ref(tuning), int(num_sms)))


def prefill(x, z, B, C, dt_raw, params, *, conv_cache_in=None, ssm_state_in=None, y=None, conv_cache_out=None,
            ssm_state_out=None, dt_min=1e-4, dt_max=1.0, discretization="euler", tuning=None, stream=None):
    """Full-sequence block core. x, z: [b, L, E] (last dim contiguous; token and
    sequence strides are passed through); B, C: [b, L, 16]; dt_raw: [b, L].
    Returns (y [b, L, E], conv_cache_out [b, 3, E], ssm_state_out [b, E, 16])."""
    lib = _lib.load()
    b, L, E = x.shape
    dev = x.device
    for n, t in (("x", x), ("z", z), ("B", B), ("C", C), ("dt_raw", dt_raw), ("conv_cache_in", conv_cache_in),
                 ("ssm_state_in", ssm_state_in), ("y", y), ("conv_cache_out", conv_cache_out),
                 ("ssm_state_out", ssm_state_out)):
        _need_cuda(n, t, dev)
    if x.dtype not in _DTYPES or z.dtype != x.dtype:
        raise ValueError("x and z must share an io dtype (float32 or bfloat16)")
    if z.shape != (b, L, E) or B.shape != (b, L, 16) or C.shape != (b, L, 16) or dt_raw.shape != (b, L):
        raise ValueError("shape mismatch: z [b,L,E], B/C [b,L,16], dt_raw [b,L]")
    if x.stride(2) != 1 or z.stride(2) != 1 or B.stride(2) != 1 or dt_raw.stride(1) != 1:
        raise ValueError("the innermost dimension of x, z, B, C, dt_raw must be contiguous")
    if B.stride() != C.stride():
        raise ValueError("B and C must share strides")
    if y is None:
        y = torch.empty((b, L, E), dtype=x.dtype, device=dev)
    if conv_cache_out is None:
        conv_cache_out = torch.empty((b, 3, E), dtype=x.dtype, device=dev)
    if ssm_state_out is None:
        ssm_state_out = torch.empty((b, E, 16), dtype=torch.float32, device=dev)
    for n, t, shp, dt in (("conv_cache_out", conv_cache_out, (b, 3, E), x.dtype),
                          ("ssm_state_out", ssm_state_out, (b, E, 16), torch.float32),
                          ("conv_cache_in", conv_cache_in, (b, 3, E), x.dtype),
                          ("ssm_state_in", ssm_state_in, (b, E, 16), torch.float32)):
        if t is not None and (t.shape != shp or t.dtype != dt or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous {dt} tensor of shape {shp}")
    if y.shape != (b, L, E) or y.dtype != x.dtype or y.stride(2) != 1:
        raise ValueError("y must be [b, L, E] in the io dtype with a contiguous last dim")
    dims = make_dims(b, L, E, x.dtype, dt_min, dt_max, discretization,
                     x_tok_stride=x.stride(1), x_seq_stride=x.stride(0), z_tok_stride=z.stride(1),
                     z_seq_stride=z.stride(0), y_tok_stride=y.stride(1), y_seq_stride=y.stride(0),
                     bc_tok_stride=B.stride(1), bc_seq_stride=B.stride(0), dt_seq_stride=dt_raw.stride(0))
    w = _weights(params, E, dev)
    ws = int(lib.ssm_prefill_workspace_bytes(ctypes.byref(dims)))
    work = torch.empty(ws, dtype=torch.uint8, device=dev) if ws else None
    st = lib.ssm_prefill_ex(ctypes.byref(dims), ctypes.byref(w), _ptr(x), _ptr(z), _ptr(B), _ptr(C), _ptr(dt_raw),
                            _ptr(conv_cache_in), _ptr(ssm_state_in), _ptr(y), _ptr(conv_cache_out),
                            _ptr(ssm_state_out), _ptr(work), ws, _tuning_ref(tuning), _stream(stream))
    _lib.check(st)
    return y, conv_cache_out, ssm_state_out


def host_workspace_bytes(batch, seqlen, E, io_dtype=torch.bfloat16, chunk_tokens=0) -> int:
    lib = _lib.load()
    return int(lib.ssm_prefill_host_workspace_bytes(ctypes.byref(make_dims(batch, seqlen, E, io_dtype)),
                                                    int(chunk_tokens)))


def prefill_host(x, z, B, C, dt_raw, params, *, conv_cache_in=None, ssm_state_in=None, y=None, conv_cache_out=None,
                 ssm_state_out=None, dt_min=1e-4, dt_max=1.0, discretization="euler", chunk_tokens=0, workspace=None,
                 stream=None, static_scratch=False):
    """Full-sequence block core with the token tensors in host memory
    (ssm_prefill_host): x, z, B, C, dt_raw and y are pinned CPU tensors
    (pageable ones are refused), shaped and strided as for `prefill`; the parameters and
    the caches are CUDA tensors on the current device. The copies and kernels
    are only enqueued: synchronise `stream` before reading y. With
    static_scratch=True the call goes to ssm_prefill_host_static, which takes
    no workspace and allocates nothing (its chunk buffers are the library's
    static device scratch).
    Returns (y [b, L, E] on the host, conv_cache_out, ssm_state_out)."""
    lib = _lib.load()
    b, L, E = x.shape
    dev = params["A_log"].device
    for n, t in (("x", x), ("z", z), ("B", B), ("C", C), ("dt_raw", dt_raw), ("y", y)):
        if t is not None and t.is_cuda:
            raise RuntimeError(f"{n} must be a host tensor for prefill_host (use prefill for device tensors)")
    for n, t in (("conv_cache_in", conv_cache_in), ("ssm_state_in", ssm_state_in),
                 ("conv_cache_out", conv_cache_out), ("ssm_state_out", ssm_state_out)):
        _need_cuda(n, t, dev)
    if x.dtype not in _DTYPES or z.dtype != x.dtype:
        raise ValueError("x and z must share an io dtype (float32 or bfloat16)")
    if z.shape != (b, L, E) or B.shape != (b, L, 16) or C.shape != (b, L, 16) or dt_raw.shape != (b, L):
        raise ValueError("shape mismatch: z [b,L,E], B/C [b,L,16], dt_raw [b,L]")
    if x.stride(2) != 1 or z.stride(2) != 1 or B.stride(2) != 1 or dt_raw.stride(1) != 1:
        raise ValueError("the innermost dimension of x, z, B, C, dt_raw must be contiguous")
    if B.stride() != C.stride():
        raise ValueError("B and C must share strides")
    if y is None:
        y = torch.empty((b, L, E), dtype=x.dtype, pin_memory=True)
    if conv_cache_out is None:
        conv_cache_out = torch.empty((b, 3, E), dtype=x.dtype, device=dev)
    if ssm_state_out is None:
        ssm_state_out = torch.empty((b, E, 16), dtype=torch.float32, device=dev)
    if y.shape != (b, L, E) or y.dtype != x.dtype or y.stride(2) != 1:
        raise ValueError("y must be [b, L, E] in the io dtype with a contiguous last dim")
    dims = make_dims(b, L, E, x.dtype, dt_min, dt_max, discretization,
                     x_tok_stride=x.stride(1), x_seq_stride=x.stride(0), z_tok_stride=z.stride(1),
                     z_seq_stride=z.stride(0), y_tok_stride=y.stride(1), y_seq_stride=y.stride(0),
                     bc_tok_stride=B.stride(1), bc_seq_stride=B.stride(0), dt_seq_stride=dt_raw.stride(0))
    w = _weights(params, E, dev)
    if static_scratch:
        st = lib.ssm_prefill_host_static(ctypes.byref(dims), ctypes.byref(w), _ptr(x), _ptr(z), _ptr(B), _ptr(C),
                                         _ptr(dt_raw), _ptr(conv_cache_in), _ptr(ssm_state_in), _ptr(y),
                                         _ptr(conv_cache_out), _ptr(ssm_state_out), int(chunk_tokens), _stream(stream))
        _lib.check(st)
        return y, conv_cache_out, ssm_state_out
    ws = int(lib.ssm_prefill_host_workspace_bytes(ctypes.byref(dims), int(chunk_tokens)))
    if workspace is None or workspace.numel() < ws:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
    st = lib.ssm_prefill_host(ctypes.byref(dims), ctypes.byref(w), _ptr(x), _ptr(z), _ptr(B), _ptr(C), _ptr(dt_raw),
                              _ptr(conv_cache_in), _ptr(ssm_state_in), _ptr(y), _ptr(conv_cache_out),
                              _ptr(ssm_state_out), _ptr(workspace), workspace.numel(), int(chunk_tokens),
                              _stream(stream))
    _lib.check(st)
    return y, conv_cache_out, ssm_state_out


def segment_summary_workspace_bytes(batch, seqlen, E, io_dtype=torch.bfloat16) -> int:
    lib = _lib.load()
    return int(lib.ssm_segment_summary_workspace_bytes(ctypes.byref(make_dims(batch, seqlen, E, io_dtype))))


def segment_summary(x, B, dt_raw, params, *, conv_cache_in=None, summary=None, workspace=None, dt_min=1e-4,
                    dt_max=1.0, discretization="euler", stream=None):
    """Summary of one segment of a sequence for the sequence-parallel prefill
    (ssm_segment_summary): x [b, T, E] (last dim contiguous), B [b, T, 16],
    dt_raw [b, T]; conv_cache_in [b, 3, E] = raw x rows before the segment, or
    None for zeros. Returns summary [b, 17, E] fp32: the zero-start final
    state in rows 0..15, the dt sum in row 16."""
    lib = _lib.load()
    b, T, E = x.shape
    dev = x.device
    for n, t in (("x", x), ("B", B), ("dt_raw", dt_raw), ("conv_cache_in", conv_cache_in), ("summary", summary),
                 ("workspace", workspace)):
        _need_cuda(n, t, dev)
    if x.dtype not in _DTYPES:
        raise ValueError("x must be float32 or bfloat16")
    if B.shape != (b, T, 16) or dt_raw.shape != (b, T):
        raise ValueError("shape mismatch: B [b,T,16], dt_raw [b,T]")
    if x.stride(2) != 1 or B.stride(2) != 1 or dt_raw.stride(1) != 1:
        raise ValueError("the innermost dimension of x, B, dt_raw must be contiguous")
    if conv_cache_in is not None and (conv_cache_in.shape != (b, 3, E) or conv_cache_in.dtype != x.dtype
                                      or not conv_cache_in.is_contiguous()):
        raise ValueError("conv_cache_in must be a contiguous [b, 3, E] tensor in the io dtype")
    if summary is None:
        summary = torch.empty((b, 17, E), dtype=torch.float32, device=dev)
    if summary.shape != (b, 17, E) or summary.dtype != torch.float32 or not summary.is_contiguous():
        raise ValueError("summary must be a contiguous float32 [b, 17, E] tensor")
    dims = make_dims(b, T, E, x.dtype, dt_min, dt_max, discretization, x_tok_stride=x.stride(1),
                     x_seq_stride=x.stride(0), bc_tok_stride=B.stride(1), bc_seq_stride=B.stride(0),
                     dt_seq_stride=dt_raw.stride(0))
    ws = int(lib.ssm_segment_summary_workspace_bytes(ctypes.byref(dims)))
    if workspace is None and ws:
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
    if ws and workspace.numel() * workspace.element_size() < ws:
        raise ValueError(f"workspace needs {ws} bytes")
    w = _weights(params, E, dev)
    st = lib.ssm_segment_summary(ctypes.byref(dims), ctypes.byref(w), _ptr(x), _ptr(B), _ptr(dt_raw),
                                 _ptr(conv_cache_in), _ptr(summary), _ptr(workspace) if ws else None, ws,
                                 _stream(stream))
    _lib.check(st)
    return summary


def segment_carry(summaries, params, *, ssm_state_in=None, out=None, stream=None):
    """State entering the segment after the summarised ones
    (ssm_segment_carry): summaries [count, b, 17, E] fp32 (count may be 0);
    ssm_state_in [b, E, 16] = the state before segment 0, or None for zeros.
    Returns [b, E, 16] fp32 (out may alias ssm_state_in)."""
    lib = _lib.load()
    count, b, rows, E = summaries.shape
    dev = summaries.device
    for n, t in (("summaries", summaries), ("ssm_state_in", ssm_state_in), ("out", out)):
        _need_cuda(n, t, dev)
    if rows != 17 or summaries.dtype != torch.float32 or not summaries.is_contiguous():
        raise ValueError("summaries must be a contiguous float32 [count, b, 17, E] tensor")
    if out is None:
        out = torch.empty((b, E, 16), dtype=torch.float32, device=dev)
    for n, t in (("ssm_state_in", ssm_state_in), ("out", out)):
        if t is not None and (t.shape != (b, E, 16) or t.dtype != torch.float32 or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous float32 [b, E, 16] tensor")
    dims = make_dims(b, 0, E, torch.float32)
    w = _weights(params, E, dev)
    st = lib.ssm_segment_carry(ctypes.byref(dims), ctypes.byref(w), _ptr(summaries) if count else None, int(count),
                               _ptr(ssm_state_in), _ptr(out), _stream(stream))
    _lib.check(st)
    return out


PROJ_NAMES = ("W_in", "W_x", "W_out")


def make_block_dims(batch, seqlen, d_model, E, dt_min=1e-4, dt_max=1.0, discretization="euler"):
    d = _lib.SsmBlockDims()
    d.batch, d.seqlen, d.d_model, d.d_inner, d.d_state, d.d_conv = batch, seqlen, d_model, E, 16, 4
    d.dt_min, d.dt_max = dt_min, dt_max
    d.io_dtype = _lib.SSM_BF16
    d.discretization = _DISC[discretization]
    return d


def block_workspace_bytes(batch, seqlen, d_model, E) -> int:
    lib = _lib.load()
    return int(lib.ssm_block_workspace_bytes(ctypes.byref(make_block_dims(batch, seqlen, d_model, E))))


def block_forward(hidden, params, proj, *, conv_cache_in=None, ssm_state_in=None, out=None, conv_cache_out=None,
                  ssm_state_out=None, dt_min=1e-4, dt_max=1.0, discretization="euler", workspace=None, stream=None):
    """The whole block forward (ssm_block_forward): hidden [b, L, D] bf16 ->
    out [b, L, D] bf16, with proj = {"W_in": [2E, D], "W_x": [33, E],
    "W_out": [D, E]} bf16 and the core's parameters in `params`.
    Returns (out, conv_cache_out [b, 3, E], ssm_state_out [b, E, 16])."""
    lib = _lib.load()
    b, L, Dm = hidden.shape
    dev = hidden.device
    E = proj["W_x"].shape[1]
    for n, t in (("hidden", hidden), ("out", out), ("conv_cache_in", conv_cache_in), ("ssm_state_in", ssm_state_in),
                 ("conv_cache_out", conv_cache_out), ("ssm_state_out", ssm_state_out)):
        _need_cuda(n, t, dev)
    for n in PROJ_NAMES:
        _need_cuda(n, proj[n], dev)
        if proj[n].dtype != torch.bfloat16 or not proj[n].is_contiguous():
            raise ValueError(f"{n} must be a contiguous bfloat16 tensor")
    if proj["W_in"].shape != (2 * E, Dm) or proj["W_x"].shape != (33, E) or proj["W_out"].shape != (Dm, E):
        raise ValueError("W_in must be [2E, D], W_x [33, E] and W_out [D, E]")
    if hidden.dtype != torch.bfloat16 or not hidden.is_contiguous():
        raise ValueError("hidden must be a contiguous bfloat16 tensor")
    if out is None:
        out = torch.empty((b, L, Dm), dtype=torch.bfloat16, device=dev)
    if conv_cache_out is None:
        conv_cache_out = torch.empty((b, 3, E), dtype=torch.bfloat16, device=dev)
    if ssm_state_out is None:
        ssm_state_out = torch.empty((b, E, 16), dtype=torch.float32, device=dev)
    dims = make_block_dims(b, L, Dm, E, dt_min, dt_max, discretization)
    w = _weights(params, E, dev)
    pw = _lib.SsmBlockWeights(proj["W_in"].data_ptr(), proj["W_x"].data_ptr(), proj["W_out"].data_ptr())
    ws = int(lib.ssm_block_workspace_bytes(ctypes.byref(dims)))
    if workspace is None or workspace.numel() < ws:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
    st = lib.ssm_block_forward(ctypes.byref(dims), ctypes.byref(w), ctypes.byref(pw), _ptr(hidden),
                               _ptr(conv_cache_in), _ptr(ssm_state_in), _ptr(out), _ptr(conv_cache_out),
                               _ptr(ssm_state_out), _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(st)
    return out, conv_cache_out, ssm_state_out


def proj_gemm_workspace_bytes(M, N, K) -> int:
    lib = _lib.load()
    return int(lib.ssm_proj_gemm_workspace_bytes(int(M), int(N), int(K)))


def proj_gemm(A, W, *, out=None, workspace=None, stream=None):
    """One projection of the block (ssm_proj_gemm): out = A @ W^T with A [M, K]
    and W [N, K] contiguous bf16 CUDA tensors; returns out [M, N] bf16. The
    cut-tile scratch, when the shape needs one, is `workspace` or allocated."""
    lib = _lib.load()
    M, K = A.shape
    N = W.shape[0]
    dev = A.device
    for n, t in (("A", A), ("W", W), ("out", out)):
        _need_cuda(n, t, dev)
        if t is not None and (t.dtype != torch.bfloat16 or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous bfloat16 tensor")
    if W.shape[1] != K:
        raise ValueError("A [M, K] and W [N, K] must share K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    if out.shape != (M, N):
        raise ValueError("out must be [M, N]")
    ws = int(lib.ssm_proj_gemm_workspace_bytes(M, N, K))
    if ws and (workspace is None or workspace.numel() * workspace.element_size() < ws):
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
    _lib.check(lib.ssm_proj_gemm(_ptr(A), _ptr(W), _ptr(out), M, N, K, _ptr(workspace) if ws else None, ws,
                                 _stream(stream)))
    return out


def ssd_chunk_scan(cb, x, dt, dA_cumsum, C, prev_states, D=None, *, out=None, stream=None):
    """Mamba-2 chunk-scan output (ssm_ssd_chunk_scan). cb [b, nc, G, cs, cs],
    x [b, L, H, P], C [b, L, G, N], prev_states [b, nc, H, P, N]: bf16;
    dt, dA_cumsum [b, H, nc, cs] and D [H]: fp32. Returns out [b, L, H, P] bf16."""
    lib = _lib.load()
    b, L, H, P = x.shape
    _, nc, G, cs, _ = cb.shape
    N = C.shape[-1]
    dev = x.device
    for n, t in (("cb", cb), ("x", x), ("dt", dt), ("dA_cumsum", dA_cumsum), ("C", C), ("prev_states", prev_states),
                 ("D", D), ("out", out)):
        _need_cuda(n, t, dev)
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    for n, t in (("cb", cb), ("x", x), ("C", C), ("prev_states", prev_states)):
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{n} must be bfloat16")
    for n, t in (("dt", dt), ("dA_cumsum", dA_cumsum), ("D", D)):
        if t is not None and t.dtype != torch.float32:
            raise ValueError(f"{n} must be float32")
    if (cb.shape != (b, nc, G, cs, cs) or C.shape != (b, L, G, N) or prev_states.shape != (b, nc, H, P, N)
            or dt.shape != (b, H, nc, cs) or dA_cumsum.shape != dt.shape or (D is not None and D.shape != (H,))):
        raise ValueError("shape mismatch between the chunk-scan operands")
    if out is None:
        out = torch.empty_like(x)
    d = _lib.SsmSsdDims(b, L, H, P, G, N, cs)
    st = lib.ssm_ssd_chunk_scan(ctypes.byref(d), _ptr(cb), _ptr(x), _ptr(dt), _ptr(dA_cumsum), _ptr(C),
                                _ptr(prev_states), _ptr(D), _ptr(out), _stream(stream))
    _lib.check(st)
    return out


def decode_step(x, z, B, C, dt_raw, params, conv_cache, ssm_state, *, y=None, dt_min=1e-4, dt_max=1.0,
                discretization="euler", stream=None):
    """One-token block core. x, z: [b, E] (last dim contiguous); B, C: [b, 16];
    dt_raw: [b]; conv_cache [b, 3, E] and ssm_state [b, E, 16] are updated in
    place. Returns y [b, E]."""
    lib = _lib.load()
    b, E = x.shape
    dev = x.device
    for n, t in (("x", x), ("z", z), ("B", B), ("C", C), ("dt_raw", dt_raw), ("conv_cache", conv_cache),
                 ("ssm_state", ssm_state), ("y", y)):
        _need_cuda(n, t, dev)
    if x.dtype not in _DTYPES or z.dtype != x.dtype or conv_cache.dtype != x.dtype:
        raise ValueError("x, z and conv_cache must share an io dtype")
    if z.shape != (b, E) or B.shape != (b, 16) or C.shape != (b, 16) or dt_raw.shape != (b,):
        raise ValueError("shape mismatch: z [b,E], B/C [b,16], dt_raw [b]")
    if x.stride(1) != 1 or z.stride(1) != 1 or B.stride(1) != 1 or B.stride() != C.stride():
        raise ValueError("innermost dims must be contiguous and B, C share strides")
    if conv_cache.shape != (b, 3, E) or not conv_cache.is_contiguous():
        raise ValueError("conv_cache must be a contiguous [b, 3, E] tensor")
    if ssm_state.shape != (b, E, 16) or ssm_state.dtype != torch.float32 or not ssm_state.is_contiguous():
        raise ValueError("ssm_state must be a contiguous float32 [b, E, 16] tensor")
    if y is None:
        y = torch.empty((b, E), dtype=x.dtype, device=dev)
    dims = make_dims(b, 1, E, x.dtype, dt_min, dt_max, discretization, x_seq_stride=x.stride(0),
                     z_seq_stride=z.stride(0), y_seq_stride=y.stride(0), bc_seq_stride=B.stride(0),
                     dt_seq_stride=dt_raw.stride(0))
    w = _weights(params, E, dev)
    st = lib.ssm_decode_step(ctypes.byref(dims), ctypes.byref(w), _ptr(x), _ptr(z), _ptr(B), _ptr(C), _ptr(dt_raw),
                             _ptr(y), _ptr(conv_cache), _ptr(ssm_state), _stream(stream))
    _lib.check(st)
    return y


def check_device_error(stream=None):
    """ssm_check_device_error: synchronises `stream`, then raises SsmError
    (status SSM_ERR_DEVICE) if a kernel's bounded wait gave up since the last
    check, clearing the device error word."""
    lib = _lib.load()
    _lib.check(lib.ssm_check_device_error(_stream(stream)))


def selftest_bounded_wait(limit_ns=1_000_000, stream=None):
    """ssm_selftest_bounded_wait: a kernel whose wait can never complete gives
    up after limit_ns and reports through the device error word."""
    lib = _lib.load()
    _lib.check(lib.ssm_selftest_bounded_wait(int(limit_ns), _stream(stream)))
