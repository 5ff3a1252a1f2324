"""ctypes view of the C ABI in include/ssm.h (libssm.so).

Argument marshalling only: structures mirror the header, functions keep the
header's names. Loading fails loudly if the library is missing; there is no
fallback implementation anywhere in the package.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libssm.so")

SSM_OK, SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_CUDA, SSM_ERR_DEVICE = 0, 1, 2, 3, 4
SSM_F32, SSM_BF16 = 0, 1
SSM_DISC_EULER_B, SSM_DISC_ZOH = 0, 1

# Every symbol include/ssm.h declares (checked by the CPU test suite).
SSM_HOST_STATIC_SCRATCH_BYTES = 128 << 20  # include/ssm.h
SSM_SELFTEST_WAIT_CODE = 99  # include/ssm.h

EXPORTED = (
    "ssm_prefill",
    "ssm_prefill_ex",
    "ssm_prefill_workspace_bytes",
    "ssm_prefill_kernel",
    "ssm_prefill_host",
    "ssm_prefill_host_workspace_bytes",
    "ssm_prefill_host_static",
    "ssm_block_forward",
    "ssm_block_workspace_bytes",
    "ssm_proj_gemm",
    "ssm_proj_gemm_workspace_bytes",
    "ssm_ssd_chunk_scan",
    "ssm_segment_summary",
    "ssm_segment_summary_workspace_bytes",
    "ssm_segment_carry",
    "ssm_decode_step",
    "ssm_check_device_error",
    "ssm_selftest_bounded_wait",
    "ssm_status_string",
    "ssm_last_error",
    "ssm_version",
)


class SsmDims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("d_inner", ctypes.c_int64),
        ("d_state", ctypes.c_int32),
        ("d_conv", ctypes.c_int32),
        ("dt_min", ctypes.c_float),
        ("dt_max", ctypes.c_float),
        ("io_dtype", ctypes.c_int32),
        ("discretization", ctypes.c_int32),
        ("x_tok_stride", ctypes.c_int64),
        ("x_seq_stride", ctypes.c_int64),
        ("z_tok_stride", ctypes.c_int64),
        ("z_seq_stride", ctypes.c_int64),
        ("y_tok_stride", ctypes.c_int64),
        ("y_seq_stride", ctypes.c_int64),
        ("bc_tok_stride", ctypes.c_int64),
        ("bc_seq_stride", ctypes.c_int64),
        ("dt_seq_stride", ctypes.c_int64),
    ]


class SsmBlockDims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("d_model", ctypes.c_int64),
        ("d_inner", ctypes.c_int64),
        ("d_state", ctypes.c_int32),
        ("d_conv", ctypes.c_int32),
        ("dt_min", ctypes.c_float),
        ("dt_max", ctypes.c_float),
        ("io_dtype", ctypes.c_int32),
        ("discretization", ctypes.c_int32),
    ]


class SsmBlockWeights(ctypes.Structure):
    _fields_ = [("w_in", ctypes.c_void_p), ("w_x", ctypes.c_void_p), ("w_out", ctypes.c_void_p)]


class SsmSsdDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate",
                                             "chunk_size")]


class SsmWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D")]


class SsmTuning(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("decay_path", ctypes.c_int32)]


class SsmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load libssm.so and declare the signatures. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libssm.so not built at {path}: run __graft_entry__.build() (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    p, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    dims_p, w_p, tun_p = ctypes.POINTER(SsmDims), ctypes.POINTER(SsmWeights), ctypes.POINTER(SsmTuning)
    lib.ssm_prefill.argtypes = [dims_p, w_p] + [p] * 10 + [p, sz, p]
    lib.ssm_prefill.restype = st
    lib.ssm_prefill_ex.argtypes = [dims_p, w_p] + [p] * 10 + [p, sz, tun_p, p]
    lib.ssm_prefill_ex.restype = st
    lib.ssm_prefill_workspace_bytes.argtypes = [dims_p]
    lib.ssm_prefill_workspace_bytes.restype = sz
    lib.ssm_prefill_kernel.argtypes = [dims_p, tun_p, ctypes.c_int32]
    lib.ssm_prefill_kernel.restype = ctypes.c_int32
    lib.ssm_prefill_host.argtypes = [dims_p, w_p] + [p] * 10 + [p, sz, ctypes.c_int64, p]
    lib.ssm_prefill_host.restype = st
    lib.ssm_prefill_host_static.argtypes = [dims_p, w_p] + [p] * 10 + [ctypes.c_int64, p]
    lib.ssm_prefill_host_static.restype = st
    lib.ssm_prefill_host_workspace_bytes.argtypes = [dims_p, ctypes.c_int64]
    lib.ssm_prefill_host_workspace_bytes.restype = sz
    bdims_p, bw_p = ctypes.POINTER(SsmBlockDims), ctypes.POINTER(SsmBlockWeights)
    lib.ssm_block_forward.argtypes = [bdims_p, w_p, bw_p] + [p] * 6 + [p, sz, p]
    lib.ssm_block_forward.restype = st
    lib.ssm_block_workspace_bytes.argtypes = [bdims_p]
    lib.ssm_block_workspace_bytes.restype = sz
    i64 = ctypes.c_int64
    lib.ssm_proj_gemm.argtypes = [p, p, p, i64, i64, i64, p, sz, p]
    lib.ssm_proj_gemm.restype = st
    lib.ssm_proj_gemm_workspace_bytes.argtypes = [i64, i64, i64]
    lib.ssm_proj_gemm_workspace_bytes.restype = sz
    lib.ssm_ssd_chunk_scan.argtypes = [ctypes.POINTER(SsmSsdDims)] + [p] * 8 + [p]
    lib.ssm_ssd_chunk_scan.restype = st
    lib.ssm_segment_summary.argtypes = [dims_p, w_p] + [p] * 6 + [sz, p]
    lib.ssm_segment_summary.restype = st
    lib.ssm_segment_summary_workspace_bytes.argtypes = [dims_p]
    lib.ssm_segment_summary_workspace_bytes.restype = sz
    lib.ssm_segment_carry.argtypes = [dims_p, w_p, p, ctypes.c_int64, p, p, p]
    lib.ssm_segment_carry.restype = st
    lib.ssm_decode_step.argtypes = [dims_p, w_p] + [p] * 8 + [p]
    lib.ssm_decode_step.restype = st
    lib.ssm_check_device_error.argtypes = [p]
    lib.ssm_check_device_error.restype = st
    lib.ssm_selftest_bounded_wait.argtypes = [ctypes.c_int64, p]
    lib.ssm_selftest_bounded_wait.restype = st
    lib.ssm_status_string.argtypes = [st]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_last_error.argtypes = []
    lib.ssm_last_error.restype = ctypes.c_char_p
    lib.ssm_version.argtypes = []
    lib.ssm_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def check(status: int):
    if status != SSM_OK:
        lib = load()
        raise SsmError(status, f"{lib.ssm_status_string(status).decode()}: {lib.ssm_last_error().decode()}")
