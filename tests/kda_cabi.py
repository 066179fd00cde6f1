"""Argument structs of the C ABI built straight from torch tensors, for the tests
that call libkda.so through ctypes without the Python binding."""
from __future__ import annotations

import ctypes

import torch

from kimi_delta_attention_20_b200 import _abi


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def chunk_args(d, o, S, *, lower_bound=None, l2=True, chunk_size=64, workspace=None, debug_flags=0):
    """kda_chunk_args for the device tensors in ``d`` (q, k, v, g, beta [B, T, H, D],
    optional initial_state, cu_seqlens with its host copy cu_host) writing o and S."""
    a = _abi.ChunkArgs()
    a.dtype = _abi.KDA_DTYPE_BF16 if d["q"].dtype == torch.bfloat16 else _abi.KDA_DTYPE_F32
    B, T, H, Dk = d["q"].shape
    a.B, a.T, a.H, a.Dk, a.Dv = B, T, H, Dk, d["v"].shape[-1]
    for name in ("q", "k", "v", "g", "beta"):
        setattr(a, name, _p(d[name]))
    a.o = _p(o)
    a.scale = float("nan")
    a.initial_state = _p(d.get("initial_state"))
    a.final_state = _p(S)
    if d.get("cu_seqlens") is not None:
        a.cu_seqlens = _p(d["cu_seqlens"])
        a.cu_seqlens_host = _p(d["cu_host"])
        a.N = d["cu_host"].numel() - 1
    else:
        a.N = B
    a.use_qk_l2norm = int(l2)
    a.has_lower_bound = int(lower_bound is not None)
    a.lower_bound = float(lower_bound) if lower_bound is not None else 0.0
    a.chunk_size = chunk_size
    if workspace is not None:
        a.workspace = _p(workspace)
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a.debug_flags = debug_flags
    return a


def to_device(inp, device="cuda"):
    """The drawn inputs on the device, cu_seqlens as int32 with its host copy."""
    d = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    if inp.get("cu_seqlens") is not None:
        d["cu_host"] = inp["cu_seqlens"].to(torch.int32).cpu().contiguous()
        d["cu_seqlens"] = d["cu_seqlens"].to(torch.int32).contiguous()
    return d


def stream_ptr():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
