"""ctypes mirror of include/kda.h. Argument marshalling only.

Loading fails loudly (ImportError) when libkda.so is missing: there is no
fallback implementation behind this binding.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

KDA_OK = 0
KDA_ERR_INVALID_ARGUMENT = 1
KDA_ERR_UNSUPPORTED = 2
KDA_ERR_CUDA = 3
KDA_ERR_TIMEOUT = 4
KDA_ERR_WORKSPACE = 5

KDA_DTYPE_F32 = 0
KDA_DTYPE_BF16 = 1

KDA_GATE_LOG = 0
KDA_GATE_SOFTPLUS = 1
KDA_GATE_SAFE = 2

KDA_DEBUG_STALL_FIRST_WAIT = 1

_vp = ctypes.c_void_p
_fp = ctypes.POINTER(ctypes.c_float)
_i32p = ctypes.POINTER(ctypes.c_int32)


class ChunkArgs(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
        ("Dk", ctypes.c_int), ("Dv", ctypes.c_int),
        ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp),
        ("o", _vp),
        ("scale", ctypes.c_float),
        ("initial_state", _vp), ("final_state", _vp),
        ("cu_seqlens", _vp), ("cu_seqlens_host", _vp),
        ("N", ctypes.c_int),
        ("use_qk_l2norm", ctypes.c_int),
        ("has_lower_bound", ctypes.c_int), ("lower_bound", ctypes.c_float),
        ("chunk_size", ctypes.c_int),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        ("gate_mode", ctypes.c_int), ("A_log", _vp), ("dt_bias", _vp),
        ("beta_is_prob", ctypes.c_int),
        ("debug_flags", ctypes.c_uint),
    ]


class StepArgs(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("N", ctypes.c_int), ("H", ctypes.c_int), ("Dk", ctypes.c_int), ("Dv", ctypes.c_int),
        ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp),
        ("state", _vp), ("o", _vp),
        ("scale", ctypes.c_float),
        ("use_qk_l2norm", ctypes.c_int),
        ("has_lower_bound", ctypes.c_int), ("lower_bound", ctypes.c_float),
        ("gate_mode", ctypes.c_int), ("A_log", _vp), ("dt_bias", _vp),
        ("beta_is_prob", ctypes.c_int),
        ("state_out", _vp),
    ]


class TokenArgs(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("N", ctypes.c_int), ("H", ctypes.c_int), ("Dk", ctypes.c_int), ("Dv", ctypes.c_int),
        ("conv_kernel", ctypes.c_int),
        ("x", _vp), ("conv_w", _vp), ("conv_state", _vp), ("g", _vp), ("beta", _vp),
        ("state", _vp), ("g_out", _vp), ("norm_eps", ctypes.c_float), ("o", _vp),
        ("scale", ctypes.c_float),
        ("use_qk_l2norm", ctypes.c_int),
        ("has_lower_bound", ctypes.c_int), ("lower_bound", ctypes.c_float),
        ("gate_mode", ctypes.c_int), ("A_log", _vp), ("dt_bias", _vp),
        ("beta_is_prob", ctypes.c_int),
        ("state_out", _vp),
    ]


class BwdArgs(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
        ("Dk", ctypes.c_int), ("Dv", ctypes.c_int),
        ("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp),
        ("dout", _vp),
        ("scale", ctypes.c_float),
        ("initial_state", _vp), ("dfinal_state", _vp),
        ("dq", _vp), ("dk", _vp), ("dv", _vp), ("dg", _vp), ("dbeta", _vp),
        ("dinitial_state", _vp),
        ("cu_seqlens", _vp), ("cu_seqlens_host", _vp),
        ("N", ctypes.c_int),
        ("use_qk_l2norm", ctypes.c_int),
        ("has_lower_bound", ctypes.c_int), ("lower_bound", ctypes.c_float),
        ("beta_is_prob", ctypes.c_int),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
    ]


# every symbol include/kda.h declares
EXPORTS = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_chunk_fwd_status",
           "kda_chunk_fwd_noalloc", "kda_chunk_fwd_noalloc_status",
           "kda_recurrent_step", "kda_decode_token", "kda_chunk_bwd_workspace_size", "kda_chunk_bwd",
           "kda_status_string", "kda_last_cuda_error", "kda_launch_count", "kda_version")

_lib = None


def load():
    """Load libkda.so (once) and declare its prototypes."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m kimi_delta_attention_20_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.kda_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(ChunkArgs),
                                                 ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_chunk_fwd_workspace_size.restype = ctypes.c_int
    lib.kda_chunk_fwd.argtypes = [ctypes.POINTER(ChunkArgs), _vp]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(ChunkArgs), _vp]
    lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    for name in ("kda_chunk_fwd_status", "kda_chunk_fwd_noalloc_status"):
        getattr(lib, name).argtypes = [ctypes.POINTER(ChunkArgs), _vp]
        getattr(lib, name).restype = ctypes.c_int
    lib.kda_recurrent_step.argtypes = [ctypes.POINTER(StepArgs), _vp]
    lib.kda_recurrent_step.restype = ctypes.c_int
    lib.kda_decode_token.argtypes = [ctypes.POINTER(TokenArgs), _vp]
    lib.kda_decode_token.restype = ctypes.c_int
    lib.kda_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(BwdArgs), ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_chunk_bwd_workspace_size.restype = ctypes.c_int
    lib.kda_chunk_bwd.argtypes = [ctypes.POINTER(BwdArgs), _vp]
    lib.kda_chunk_bwd.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_last_cuda_error.argtypes = []
    lib.kda_last_cuda_error.restype = ctypes.c_int
    lib.kda_launch_count.argtypes = []
    lib.kda_launch_count.restype = ctypes.c_ulonglong
    lib.kda_version.argtypes = []
    lib.kda_version.restype = ctypes.c_int
    _lib = lib
    return lib


class KDAError(RuntimeError):
    def __init__(self, status: int, what: str):
        lib = load()
        msg = lib.kda_status_string(status).decode()
        if status == KDA_ERR_CUDA:
            msg += f" (cudaError {lib.kda_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")
        self.status = status


def check(status: int, what: str):
    if status != KDA_OK:
        raise KDAError(status, what)
