"""Python entry points over the C ABI: `chunk_kda` and `recurrent_step`.

PyTorch supplies device memory and the current stream; every step of the
computation runs in the library's CUDA kernels. Tensors must live on a CUDA
device; there is no CPU path.
"""
from __future__ import annotations

import ctypes
import math
import warnings
from typing import Optional, Tuple

import torch

from . import _abi

_DTYPES = {torch.float32: _abi.KDA_DTYPE_F32, torch.bfloat16: _abi.KDA_DTYPE_BF16}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(name, t):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def chunk_kda(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
              beta: torch.Tensor, *, scale: Optional[float] = None,
              initial_state: Optional[torch.Tensor] = None, output_final_state: bool = False,
              use_qk_l2norm_in_kernel: bool = False, lower_bound: Optional[float] = None,
              chunk_size: int = 64, cu_seqlens: Optional[torch.Tensor] = None,
              out: Optional[torch.Tensor] = None, final_state_out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None
              ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise KDA forward (the `chunk_kda` boundary of page
    "K3/kda/ops/api.py", without backend dispatch or in-kernel gate).

    q, k, g: [B, T, H, Dk]; v: [B, T, H, Dv]; beta: [B, T, H] LOGITS.
    g is the per-channel log-decay (<= 0); ``lower_bound`` clamps it from
    below. ``cu_seqlens`` (int32, [N+1], B == 1) packs N sequences.
    Returns (o [B, T, H, Dv], final_state [N, H, Dk, Dv] fp32 or None).
    """
    lib = _abi.load()
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta)):
        _need_cuda(name, t)
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype for t in (k, v, g, beta)):
        raise ValueError("q, k, v, g, beta must share one dtype: float32 or bfloat16")
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, Dk]")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape != (B, T, H, Dv) or beta.shape != (B, T, H):
        raise ValueError("shape mismatch among q, k, v, g, beta")
    if not use_qk_l2norm_in_kernel:
        warnings.warn(
            "use_qk_l2norm_in_kernel=False: the chunkwise form relies on unit-norm keys; "
            "unnormalised keys can make the output grow without bound.",
            RuntimeWarning, stacklevel=2)
    if lower_bound is not None and not lower_bound < 0:
        raise ValueError("lower_bound must be negative")
    if chunk_size not in (0, 64):
        raise ValueError("chunk_size must be 64")
    cu_host = None
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("cu_seqlens requires B == 1")
        cu_host = cu_seqlens.detach().to("cpu", torch.int32).contiguous()
        cu_dev = cu_seqlens.to(q.device, torch.int32).contiguous()
        N = cu_host.numel() - 1
    else:
        cu_dev = None
        N = B
    if initial_state is not None:
        _need_cuda("initial_state", initial_state)
        if initial_state.dtype != torch.float32 or initial_state.shape != (N, H, Dk, Dv):
            raise ValueError(f"initial_state must be float32 [{N}, {H}, {Dk}, {Dv}]")
    o = out if out is not None else torch.empty(B, T, H, Dv, dtype=q.dtype, device=q.device)
    fs = None
    if output_final_state:
        fs = final_state_out if final_state_out is not None else torch.empty(
            N, H, Dk, Dv, dtype=torch.float32, device=q.device)
    a = _abi.ChunkArgs()
    a.dtype = _DTYPES[q.dtype]
    a.B, a.T, a.H, a.Dk, a.Dv = B, T, H, Dk, Dv
    a.q, a.k, a.v, a.g, a.beta, a.o = (_ptr(t) for t in (q, k, v, g, beta, o))
    a.scale = float("nan") if scale is None else float(scale)
    a.initial_state = _ptr(initial_state)
    a.final_state = _ptr(fs)
    a.cu_seqlens = _ptr(cu_dev)
    a.cu_seqlens_host = _ptr(cu_host)
    a.N = N
    a.use_qk_l2norm = int(bool(use_qk_l2norm_in_kernel))
    a.has_lower_bound = int(lower_bound is not None)
    a.lower_bound = float(lower_bound) if lower_bound is not None else 0.0
    a.chunk_size = int(chunk_size)
    nbytes = ctypes.c_size_t(0)
    _abi.check(lib.kda_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(nbytes)),
               "kda_chunk_fwd_workspace_size")
    if nbytes.value:
        if workspace is None or workspace.numel() * workspace.element_size() < nbytes.value:
            workspace = torch.empty(nbytes.value, dtype=torch.uint8, device=q.device)
        a.workspace = _ptr(workspace)
        a.workspace_bytes = nbytes.value
    with torch.cuda.device(q.device):
        _abi.check(lib.kda_chunk_fwd(ctypes.byref(a), _stream(q.device)), "kda_chunk_fwd")
    return o, fs


def chunk_workspace_bytes(B, T, H, Dk, Dv, *, dtype=torch.bfloat16, N=None, varlen=False):
    """Workspace bytes kda_chunk_fwd needs for this geometry."""
    lib = _abi.load()
    a = _abi.ChunkArgs()
    a.dtype = _DTYPES[dtype]
    a.B, a.T, a.H, a.Dk, a.Dv = B, T, H, Dk, Dv
    a.N = N if N is not None else B
    a.cu_seqlens = ctypes.c_void_p(1) if varlen else None  # only its presence is read
    nbytes = ctypes.c_size_t(0)
    _abi.check(lib.kda_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(nbytes)),
               "kda_chunk_fwd_workspace_size")
    return nbytes.value


def recurrent_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                   beta: torch.Tensor, state: torch.Tensor, *, scale: Optional[float] = None,
                   use_qk_l2norm_in_kernel: bool = True, lower_bound: Optional[float] = None,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One decode token per sequence (page "atlas_core/kimi_k3/kda.rs",
    `kda_recurrent_step`, which always normalises q and k).

    q, k, g: [N, H, Dk]; v: [N, H, Dv]; beta: [N, H] logits; state:
    [N, H, Dk, Dv] fp32, updated IN PLACE. Returns o [N, H, Dv].
    """
    lib = _abi.load()
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("state", state)):
        _need_cuda(name, t)
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype for t in (k, v, g, beta)):
        raise ValueError("q, k, v, g, beta must share one dtype: float32 or bfloat16")
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape != (N, H, Dv) or beta.shape != (N, H):
        raise ValueError("shape mismatch among q, k, v, g, beta")
    if state.dtype != torch.float32 or state.shape != (N, H, Dk, Dv):
        raise ValueError(f"state must be float32 [{N}, {H}, {Dk}, {Dv}]")
    if lower_bound is not None and not lower_bound < 0:
        raise ValueError("lower_bound must be negative")
    o = out if out is not None else torch.empty(N, H, Dv, dtype=q.dtype, device=q.device)
    a = _abi.StepArgs()
    a.dtype = _DTYPES[q.dtype]
    a.N, a.H, a.Dk, a.Dv = N, H, Dk, Dv
    a.q, a.k, a.v, a.g, a.beta, a.state, a.o = (_ptr(t) for t in (q, k, v, g, beta, state, o))
    a.scale = float("nan") if scale is None else float(scale)
    a.use_qk_l2norm = int(bool(use_qk_l2norm_in_kernel))
    a.has_lower_bound = int(lower_bound is not None)
    a.lower_bound = float(lower_bound) if lower_bound is not None else 0.0
    with torch.cuda.device(q.device):
        _abi.check(lib.kda_recurrent_step(ctypes.byref(a), _stream(q.device)), "kda_recurrent_step")
    return o
