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


def _seqlens(cu_seqlens, cu_seqlens_cpu, device):
    """Device and host copies of the varlen offsets (int32, [N + 1]).

    The library validates the offsets and orders its work from the host copy
    during the call, and its kernels read the device copy. A CPU ``cu_seqlens``
    is that host copy and goes to the device by an asynchronous copy from pinned
    memory; a CUDA ``cu_seqlens`` with ``cu_seqlens_cpu`` (its host copy) costs no
    copy at all. Only a CUDA ``cu_seqlens`` without a host copy needs a blocking
    device-to-host read, which stalls the host until the stream reaches it.
    """
    if cu_seqlens is None:
        if cu_seqlens_cpu is not None:
            raise ValueError("cu_seqlens_cpu needs cu_seqlens")
        return None, None
    if cu_seqlens_cpu is not None:
        if cu_seqlens_cpu.is_cuda:
            raise ValueError("cu_seqlens_cpu must be a CPU tensor")
        if cu_seqlens_cpu.shape != cu_seqlens.shape:
            raise ValueError("cu_seqlens_cpu must have the shape of cu_seqlens")
        host = cu_seqlens_cpu.to(torch.int32).contiguous()
    elif not cu_seqlens.is_cuda:
        host = cu_seqlens.to(torch.int32).contiguous()
    else:
        host = cu_seqlens.detach().to("cpu", torch.int32).contiguous()  # blocking
    if cu_seqlens.is_cuda:
        if cu_seqlens.device != device:
            raise ValueError(f"cu_seqlens must be on {device}")
        dev = cu_seqlens.to(torch.int32).contiguous()
    else:
        dev = host.pin_memory().to(device, non_blocking=True)
    return dev, host


def _gate_fields(a, device, H, Dk, A_log, dt_bias, use_gate_in_kernel, safe_gate,
                 lower_bound, use_beta_sigmoid_in_kernel):
    """Gate and beta fields of the C argument struct (page "K3/kda/ops/api.py",
    `use_gate_in_kernel`, `safe_gate`, `use_beta_sigmoid_in_kernel`)."""
    if lower_bound is not None and not lower_bound < 0:
        raise ValueError("lower_bound must be negative")
    a.beta_is_prob = int(not use_beta_sigmoid_in_kernel)
    if not use_gate_in_kernel:
        a.gate_mode = _abi.KDA_GATE_LOG
        a.has_lower_bound = int(lower_bound is not None)
        a.lower_bound = float(lower_bound) if lower_bound is not None else 0.0
        return
    if A_log is None:
        raise ValueError("A_log is required when use_gate_in_kernel=True")
    _need_cuda("A_log", A_log)
    if A_log.dtype != torch.float32 or A_log.numel() != H or A_log.device != device:
        raise ValueError(f"A_log must be float32 with {H} elements on {device}")
    if dt_bias is not None:
        _need_cuda("dt_bias", dt_bias)
        if dt_bias.dtype != torch.float32 or dt_bias.numel() != H * Dk or dt_bias.device != device:
            raise ValueError(f"dt_bias must be float32 with {H}x{Dk} elements on {device}")
    a.A_log = _ptr(A_log)
    a.dt_bias = _ptr(dt_bias)
    if safe_gate:
        if lower_bound is None:
            raise ValueError("lower_bound is required when safe_gate=True")
        a.gate_mode = _abi.KDA_GATE_SAFE
        a.has_lower_bound = 1
        a.lower_bound = float(lower_bound)
    else:  # the unbounded form takes no lower bound
        a.gate_mode = _abi.KDA_GATE_SOFTPLUS
        a.has_lower_bound = 0
        a.lower_bound = 0.0


def _chunk_kda_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
              beta: torch.Tensor, *, A_log: Optional[torch.Tensor] = None,
              dt_bias: Optional[torch.Tensor] = None, scale: Optional[float] = None,
              initial_state: Optional[torch.Tensor] = None, output_final_state: bool = False,
              use_qk_l2norm_in_kernel: bool = False, use_gate_in_kernel: bool = False,
              use_beta_sigmoid_in_kernel: bool = True, safe_gate: bool = False,
              lower_bound: Optional[float] = None,
              chunk_size: int = 64, cu_seqlens: Optional[torch.Tensor] = None,
              cu_seqlens_cpu: Optional[torch.Tensor] = None,
              out: Optional[torch.Tensor] = None, final_state_out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None
              ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise KDA forward (the `chunk_kda` boundary of page
    "K3/kda/ops/api.py", without backend dispatch).

    q, k, g: [B, T, H, Dk]; v: [B, T, H, Dv]; beta: [B, T, H].
    beta holds LOGITS (sigmoid in the kernel) unless use_beta_sigmoid_in_kernel
    is False, when it holds probabilities used as given. Note the default: the
    logit form is this operator's boundary, where api.py defaults to False.
    g is the per-channel log-decay (<= 0), clamped below by ``lower_bound``;
    with use_gate_in_kernel it is the gate input instead and the kernel forms
    -exp(A_log) softplus(g + dt_bias), or with safe_gate
    lower_bound * sigmoid(exp(A_log) (g + dt_bias)) (A_log: [H] fp32,
    dt_bias: [H, Dk] fp32 or None; the unbounded form ignores lower_bound).
    ``cu_seqlens`` (int32, [N+1], B == 1) packs N sequences; it may be a CPU
    tensor (uploaded asynchronously) or a CUDA tensor, and a CUDA one should come
    with ``cu_seqlens_cpu``, its host copy: without it every call reads the
    offsets back with a blocking device-to-host copy. ``chunk_size``
    <= 32 selects 32-token chunks (CUDA-core kernel), anything else 64.
    Returns (o [B, T, H, Dv], final_state [N, H, Dk, Dv] fp32 or None).

    When autograd is on and q, k, v, g, beta or initial_state requires grad, the
    call is recorded for the backward (``chunk_kda_bwd``): gradients flow to
    those inputs (the log-decay form; in-kernel gate forms raise).
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
    if not isinstance(chunk_size, int) or chunk_size < 0:
        raise ValueError("chunk_size must be a non-negative int")
    chunk_size = 32 if 0 < chunk_size <= 32 else 64  # api.py's 32-or-64 rule
    if cu_seqlens is not None and B != 1:
        raise ValueError("cu_seqlens requires B == 1")
    cu_dev, cu_host = _seqlens(cu_seqlens, cu_seqlens_cpu, q.device)
    N = B if cu_host is None else cu_host.numel() - 1
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
    _gate_fields(a, q.device, H, Dk, A_log, dt_bias, use_gate_in_kernel, safe_gate, lower_bound,
                 use_beta_sigmoid_in_kernel)
    a.chunk_size = int(chunk_size)
    nbytes = ctypes.c_size_t(0)
    _abi.check(lib.kda_chunk_fwd_workspace_size(ctypes.byref(a), ctypes.byref(nbytes)),
               "kda_chunk_fwd_workspace_size")
    if nbytes.value:
        # a caller's workspace is passed as is: the library runs the fastest kernel it
        # allows (the per-chunk records of the two-pass kernel need the full size, the
        # single-pass kernel 256 bytes) and rejects one too small for any
        if workspace is None:
            workspace = torch.empty(nbytes.value, dtype=torch.uint8, device=q.device)
        _need_cuda("workspace", workspace)
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel() * workspace.element_size()
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


def chunk_bwd_workspace_bytes(B, T, H, Dk, Dv, *, dtype=torch.bfloat16, N=None, varlen=False):
    """Workspace bytes kda_chunk_bwd needs for this geometry."""
    lib = _abi.load()
    a = _abi.BwdArgs()
    a.dtype = _DTYPES[dtype]
    a.B, a.T, a.H, a.Dk, a.Dv = B, T, H, Dk, Dv
    a.N = N if N is not None else B
    a.cu_seqlens = ctypes.c_void_p(1) if varlen else None  # only its presence is read
    nbytes = ctypes.c_size_t(0)
    _abi.check(lib.kda_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(nbytes)),
               "kda_chunk_bwd_workspace_size")
    return nbytes.value


def _check_state_out(state: torch.Tensor, state_out: Optional[torch.Tensor]):
    if state_out is None:
        return
    _need_cuda("state_out", state_out)
    if state_out.dtype != torch.float32 or state_out.shape != state.shape or not state_out.is_contiguous():
        raise ValueError(f"state_out must be a contiguous float32 tensor of shape {tuple(state.shape)}")


def recurrent_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                   beta: torch.Tensor, state: torch.Tensor, *, A_log: Optional[torch.Tensor] = None,
                   dt_bias: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                   use_qk_l2norm_in_kernel: bool = True, use_gate_in_kernel: bool = False,
                   use_beta_sigmoid_in_kernel: bool = True, safe_gate: bool = False,
                   lower_bound: Optional[float] = None,
                   out: Optional[torch.Tensor] = None,
                   state_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One decode token per sequence (page "atlas_core/kimi_k3/kda.rs",
    `kda_recurrent_step`, which always normalises q and k).

    q, k, g: [N, H, Dk]; v: [N, H, Dv]; beta: [N, H] logits (or probabilities
    with use_beta_sigmoid_in_kernel=False); state: [N, H, Dk, Dv] fp32, updated
    IN PLACE, or only read when ``state_out`` (a second fp32 [N, H, Dk, Dv]
    buffer, disjoint from ``state``) receives the new state. Gate arguments as in
    ``chunk_kda``. Returns o [N, H, Dv].
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
    _check_state_out(state, state_out)
    o = out if out is not None else torch.empty(N, H, Dv, dtype=q.dtype, device=q.device)
    a = _abi.StepArgs()
    a.dtype = _DTYPES[q.dtype]
    a.N, a.H, a.Dk, a.Dv = N, H, Dk, Dv
    a.q, a.k, a.v, a.g, a.beta, a.state, a.o = (_ptr(t) for t in (q, k, v, g, beta, state, o))
    a.state_out = _ptr(state_out)
    a.scale = float("nan") if scale is None else float(scale)
    a.use_qk_l2norm = int(bool(use_qk_l2norm_in_kernel))
    _gate_fields(a, q.device, H, Dk, A_log, dt_bias, use_gate_in_kernel, safe_gate, lower_bound,
                 use_beta_sigmoid_in_kernel)
    with torch.cuda.device(q.device):
        _abi.check(lib.kda_recurrent_step(ctypes.byref(a), _stream(q.device)), "kda_recurrent_step")
    return o


def decode_token(x: torch.Tensor, conv_w: torch.Tensor, conv_state: torch.Tensor, g: torch.Tensor,
                 beta: torch.Tensor, state: torch.Tensor, *, g_out: Optional[torch.Tensor] = None,
                 norm_eps: float = 1e-6, A_log: Optional[torch.Tensor] = None,
                 dt_bias: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                 use_qk_l2norm_in_kernel: bool = True, use_gate_in_kernel: bool = False,
                 use_beta_sigmoid_in_kernel: bool = True, safe_gate: bool = False,
                 lower_bound: Optional[float] = None,
                 out: Optional[torch.Tensor] = None,
                 state_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One serving decode token per sequence in one launch (page
    "atlas_core/kimi_k3/kda.rs": `conv_update` + SiLU, `kda_recurrent_step`, and
    `full_rank_output_gate` when ``g_out`` is given).

    x: [N, H*(2 Dk + Dv)] pre-conv projections q | k | v; conv_w: [H*(2 Dk + Dv), K]
    fp32; conv_state: [N, H*(2 Dk + Dv), K] fp32, oldest input first, updated IN
    PLACE; g: [N, H, Dk]; beta: [N, H]; state: [N, H, Dk, Dv] fp32, updated IN PLACE
    unless ``state_out`` is given (as in ``recurrent_step``); g_out: [N, H, Dv] or None. ``norm_eps`` is the RMSNorm epsilon of the output
    gate (1e-6 by default, the norm epsilon of the KDA model configs). Gate and beta
    arguments as in ``recurrent_step``. Returns o [N, H, Dv]: the gated, normalised
    output with ``g_out``, else the recurrent step's output.
    """
    lib = _abi.load()
    for name, t in (("x", x), ("conv_w", conv_w), ("conv_state", conv_state), ("g", g), ("beta", beta),
                    ("state", state)):
        _need_cuda(name, t)
    if x.dtype not in _DTYPES or any(t.dtype != x.dtype for t in (g, beta)):
        raise ValueError("x, g, beta must share one dtype: float32 or bfloat16")
    if g_out is not None:
        _need_cuda("g_out", g_out)
        if g_out.dtype != x.dtype:
            raise ValueError("g_out must have the dtype of x")
    if state.dtype != torch.float32 or state.dim() != 4:
        raise ValueError("state must be float32 [N, H, Dk, Dv]")
    N, H, Dk, Dv = state.shape
    C = H * (2 * Dk + Dv)
    if x.shape != (N, C):
        raise ValueError(f"x must be [{N}, {C}] (q | k | v of H={H}, Dk={Dk}, Dv={Dv})")
    if conv_w.dtype != torch.float32 or conv_w.dim() != 2 or conv_w.shape[0] != C:
        raise ValueError(f"conv_w must be float32 [{C}, K]")
    K = conv_w.shape[1]
    if conv_state.dtype != torch.float32 or conv_state.shape != (N, C, K):
        raise ValueError(f"conv_state must be float32 [{N}, {C}, {K}]")
    if g.shape != (N, H, Dk) or beta.shape != (N, H):
        raise ValueError("g must be [N, H, Dk] and beta [N, H]")
    if g_out is not None and g_out.shape != (N, H, Dv):
        raise ValueError(f"g_out must be [{N}, {H}, {Dv}]")
    _check_state_out(state, state_out)
    for name, t in (("x", x), ("conv_w", conv_w), ("conv_state", conv_state), ("g", g), ("beta", beta),
                    ("state", state)) + ((("g_out", g_out),) if g_out is not None else ()):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    o = out if out is not None else torch.empty(N, H, Dv, dtype=x.dtype, device=x.device)
    a = _abi.TokenArgs()
    a.dtype = _DTYPES[x.dtype]
    a.N, a.H, a.Dk, a.Dv, a.conv_kernel = N, H, Dk, Dv, K
    a.x, a.conv_w, a.conv_state, a.g, a.beta, a.state, a.o = (
        _ptr(t) for t in (x, conv_w, conv_state, g, beta, state, o))
    a.g_out = _ptr(g_out) if g_out is not None else None
    a.state_out = _ptr(state_out)
    a.norm_eps = float(norm_eps)
    a.scale = float("nan") if scale is None else float(scale)
    a.use_qk_l2norm = int(bool(use_qk_l2norm_in_kernel))
    _gate_fields(a, x.device, H, Dk, A_log, dt_bias, use_gate_in_kernel, safe_gate, lower_bound,
                 use_beta_sigmoid_in_kernel)
    with torch.cuda.device(x.device):
        _abi.check(lib.kda_decode_token(ctypes.byref(a), _stream(x.device)), "kda_decode_token")
    return o


def chunk_kda_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                  dout: torch.Tensor, *, dfinal_state: Optional[torch.Tensor] = None,
                  initial_state: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                  use_qk_l2norm_in_kernel: bool = False, use_beta_sigmoid_in_kernel: bool = True,
                  lower_bound: Optional[float] = None, cu_seqlens: Optional[torch.Tensor] = None,
                  cu_seqlens_cpu: Optional[torch.Tensor] = None,
                  want_dinitial_state: bool = True, workspace: Optional[torch.Tensor] = None):
    """Gradients of ``chunk_kda`` (log-decay gate, the derivatives of the token
    recurrence of page "atlas_core/kimi_k3/kda.rs"; the pages give no backward
    formulas). Arguments as ``chunk_kda`` plus ``dout`` [B, T, H, Dv] (cotangent of
    o) and ``dfinal_state`` [N, H, Dk, Dv] fp32 (cotangent of the final state) or
    None. Returns (dq, dk, dv, dg, dbeta, dinitial_state or None); gradients have
    the dtype of q, dinitial_state is fp32. The gradient of g is zero where the
    lower bound is taken (g < lower_bound).
    """
    lib = _abi.load()
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta), ("dout", dout)):
        _need_cuda(name, t)
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype for t in (k, v, g, beta)):
        raise ValueError("q, k, v, g, beta must share one dtype: float32 or bfloat16")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape != (B, T, H, Dv) or beta.shape != (B, T, H):
        raise ValueError("shape mismatch among q, k, v, g, beta")
    dout = dout.to(q.dtype).contiguous()
    if dout.shape != v.shape:
        raise ValueError("dout must have the shape of v")
    if cu_seqlens is not None and B != 1:
        raise ValueError("cu_seqlens requires B == 1")
    cu_dev, cu_host = _seqlens(cu_seqlens, cu_seqlens_cpu, q.device)
    N = B if cu_host is None else cu_host.numel() - 1
    for name, t in (("initial_state", initial_state), ("dfinal_state", dfinal_state)):
        if t is not None:
            _need_cuda(name, t)
            if t.dtype != torch.float32 or t.shape != (N, H, Dk, Dv):
                raise ValueError(f"{name} must be float32 [{N}, {H}, {Dk}, {Dv}]")
    if dfinal_state is not None:
        dfinal_state = dfinal_state.contiguous()
    grads = [torch.empty_like(t) for t in (q, k, v, g, beta)]
    dS0 = torch.empty(N, H, Dk, Dv, dtype=torch.float32, device=q.device) if want_dinitial_state else None
    a = _abi.BwdArgs()
    a.dtype = _DTYPES[q.dtype]
    a.B, a.T, a.H, a.Dk, a.Dv = B, T, H, Dk, Dv
    a.q, a.k, a.v, a.g, a.beta, a.dout = (_ptr(t) for t in (q, k, v, g, beta, dout))
    a.scale = float("nan") if scale is None else float(scale)
    a.initial_state, a.dfinal_state = _ptr(initial_state), _ptr(dfinal_state)
    a.dq, a.dk, a.dv, a.dg, a.dbeta = (_ptr(t) for t in grads)
    a.dinitial_state = _ptr(dS0)
    a.cu_seqlens, a.cu_seqlens_host, a.N = _ptr(cu_dev), _ptr(cu_host), N
    a.use_qk_l2norm = int(bool(use_qk_l2norm_in_kernel))
    a.has_lower_bound = int(lower_bound is not None)
    a.lower_bound = float(lower_bound) if lower_bound is not None else 0.0
    a.beta_is_prob = int(not use_beta_sigmoid_in_kernel)
    nbytes = ctypes.c_size_t(0)
    _abi.check(lib.kda_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(nbytes)), "kda_chunk_bwd_workspace_size")
    if workspace is None or workspace.numel() * workspace.element_size() < nbytes.value:
        workspace = torch.empty(max(nbytes.value, 16), dtype=torch.uint8, device=q.device)
    a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        _abi.check(lib.kda_chunk_bwd(ctypes.byref(a), _stream(q.device)), "kda_chunk_bwd")
    return (*grads, dS0)


class _ChunkKDA(torch.autograd.Function):
    """chunk_kda recorded for autograd: forward by kda_chunk_fwd, backward by kda_chunk_bwd."""

    @staticmethod
    def forward(ctx, q, k, v, g, beta, initial_state, kw):
        o, fs = _chunk_kda_fwd(q, k, v, g, beta, initial_state=initial_state, output_final_state=True, **kw)
        ctx.save_for_backward(q, k, v, g, beta, initial_state)
        ctx.kw = kw
        return o, fs

    @staticmethod
    def backward(ctx, do, dfs):
        q, k, v, g, beta, S0 = ctx.saved_tensors
        kw = ctx.kw
        if do is None:
            do = torch.zeros(v.shape, dtype=v.dtype, device=v.device)
        dq, dk, dv, dg, db, dS0 = chunk_kda_bwd(
            q, k, v, g, beta, do, dfinal_state=dfs, initial_state=S0, scale=kw.get("scale"),
            use_qk_l2norm_in_kernel=kw.get("use_qk_l2norm_in_kernel", False),
            use_beta_sigmoid_in_kernel=kw.get("use_beta_sigmoid_in_kernel", True),
            lower_bound=kw.get("lower_bound"), cu_seqlens=kw.get("cu_seqlens"),
            cu_seqlens_cpu=kw.get("cu_seqlens_cpu"),
            want_dinitial_state=S0 is not None and ctx.needs_input_grad[5])
        return dq, dk, dv, dg, db, dS0, None


def chunk_kda(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
              beta: torch.Tensor, *, initial_state: Optional[torch.Tensor] = None,
              output_final_state: bool = False, **kw) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    tensors = (q, k, v, g, beta, initial_state)
    if torch.is_grad_enabled() and any(t is not None and t.requires_grad for t in tensors):
        if kw.get("use_gate_in_kernel") or kw.get("A_log") is not None:
            raise NotImplementedError("gradients of the in-kernel gate forms are not provided; pass the log-decay g")
        for name in ("out", "final_state_out"):
            if kw.get(name) is not None:
                raise ValueError(f"{name} cannot be used when gradients are recorded")
        o, fs = _ChunkKDA.apply(q, k, v, g, beta, initial_state, kw)
        return o, (fs if output_final_state else None)
    return _chunk_kda_fwd(q, k, v, g, beta, initial_state=initial_state, output_final_state=output_final_state, **kw)


chunk_kda.__doc__ = _chunk_kda_fwd.__doc__
