"""CPU fp64 oracle for Kimi Delta Attention (KDA).

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers allowed; the product
library never imports this package and this package never imports the
product library.

Two independently written C implementations back it (compiled on first use
with the host C compiler, or ahead of time by ``build()``):

* ``recurrent`` -- form R, the token-by-token recurrence of page
  "atlas_core/kimi_k3/kda.rs" (module doc and ``kda_recurrent_step``): the
  definition, written out.
* ``chunkwise`` -- form C, the chunk-at-a-time WY/UT form that the
  ``chunk_kda`` boundary of page "K3/kda/ops/api.py" computes, derived here
  from the same recurrence. It exists to cross-check form R.
* ``gate`` -- the in-kernel forget gate of the same boundary (``A_log``,
  ``dt_bias``, unbounded or safe form), in fp64 numpy, as page
  "atlas_core/kimi_k3/kda.rs" writes it in ``bounded_gate``.
* ``conv_update``, ``output_gate``, ``decode_token`` -- the serving decode token
  of the same page (``conv_update``, ``kda_decode_token``,
  ``full_rank_output_gate``): causal depthwise conv + SiLU, then form R for one
  token, then sigmoid(gate) * RMSNorm, in fp64 numpy.
* ``backward`` -- the gradients of the forward (dq, dk, dv, dg, dbeta and the
  initial-state gradient) for an output cotangent and an optional final-state
  cotangent: reverse-mode differentiation (torch autograd) of an fp64 torch
  restatement of the same recurrence; small cases only.

Both take packed inputs: q, k, g of shape [T_total, H, d_k], v of shape
[T_total, H, d_v], beta logits [T_total, H], ``cu_seqlens`` int offsets
[N+1] (sequence n is tokens cu_seqlens[n]..cu_seqlens[n+1]), and optional
initial states [N, H, d_k, d_v] (row = key channel). Inputs of any float
dtype are widened exactly to fp64; results come back as fp64 numpy arrays.
A [B, T, H, D] batch is the same thing with cu_seqlens = [0, T, 2T, ...].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SOURCES = ("kda_recurrent.c", "kda_chunkwise.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle's C sources into ``oracle/libkda_oracle.so``."""
    srcs = [os.path.join(_HERE, s) for s in _SOURCES]
    if not force and os.path.exists(_LIB_PATH):
        newest = max(os.path.getmtime(s) for s in srcs)
        if os.path.getmtime(_LIB_PATH) >= newest:
            return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    # IEEE semantics are part of the definition (sigmoid(-inf) = 0, exp(-inf) = 0),
    # so no fast-math.
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-Wall", "-Wextra", "-o", tmp, *srcs, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            i64p = ctypes.POINTER(ctypes.c_int64)
            common = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, i64p,
                      dp, dp, dp, dp, dp, ctypes.c_double, dp, dp, dp,
                      ctypes.c_int, ctypes.c_int, ctypes.c_double]
            lib.kda_oracle_recurrent.argtypes = common + [ctypes.c_int, ctypes.c_int]
            lib.kda_oracle_recurrent.restype = ctypes.c_int
            lib.kda_oracle_chunkwise.argtypes = common + [ctypes.c_int, ctypes.c_int, ctypes.c_int]
            lib.kda_oracle_chunkwise.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor; bf16 -> fp64 is exact
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _prep(q, k, v, g, beta, cu_seqlens, initial_state):
    q, k, v, g, beta = (_f64(t) for t in (q, k, v, g, beta))
    if q.ndim == 4:  # [B, T, H, D] -> packed
        B, T = q.shape[:2]
        if cu_seqlens is not None and B != 1:
            raise ValueError("cu_seqlens needs B == 1")
        if cu_seqlens is None:
            cu_seqlens = np.arange(B + 1, dtype=np.int64) * T
        q, k, v, g = (t.reshape(B * T, *t.shape[2:]) for t in (q, k, v, g))
        beta = beta.reshape(B * T, -1)
    Ttot, H, Dk = q.shape
    Dv = v.shape[-1]
    if cu_seqlens is None:
        cu_seqlens = np.array([0, Ttot], dtype=np.int64)
    if hasattr(cu_seqlens, "detach"):
        cu_seqlens = cu_seqlens.detach().cpu().numpy()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.size - 1
    if cu[0] != 0 or cu[-1] != Ttot or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at T_total")
    for name, t, shp in (("k", k, (Ttot, H, Dk)), ("v", v, (Ttot, H, Dv)),
                         ("g", g, (Ttot, H, Dk)), ("beta", beta, (Ttot, H))):
        if t.shape != shp:
            raise ValueError(f"{name} has shape {t.shape}, expected {shp}")
    S0 = _f64(initial_state)
    if S0 is not None and S0.shape != (N, H, Dk, Dv):
        raise ValueError(f"initial_state has shape {S0.shape}, expected {(N, H, Dk, Dv)}")
    return q, k, v, g, beta, cu, S0, N, H, Dk, Dv


def _threads(nthreads):
    if nthreads and nthreads > 0:
        return int(nthreads)
    return os.cpu_count() or 1


def softplus(x):
    """log(1 + e^x) in the overflow-free split max(x, 0) + log1p(e^-|x|)
    (page "atlas_core/kimi_k3/kda.rs", `softplus`)."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def gate(g_in, A_log, dt_bias=None, lower_bound=None):
    """In-kernel forget gate in log space for inputs g_in [..., H, Dk].

    With x = g_in + dt_bias (dt_bias [H, Dk] or None) and rate = exp(A_log[h]):
      lower_bound None: g = -rate * softplus(x)                (unbounded form)
      lower_bound lb:   g = lb * sigmoid(rate * x)             (safe form)
    (page "atlas_core/kimi_k3/kda.rs", `bounded_gate`; page "K3/kda/ops/api.py",
    `use_gate_in_kernel` / `safe_gate`).
    """
    x = _f64(g_in)
    if dt_bias is not None:
        x = x + _f64(dt_bias)
    rate = np.exp(_f64(A_log)).reshape(-1, 1)
    if lower_bound is None:
        return -rate * softplus(x)
    return float(lower_bound) / (1.0 + np.exp(-rate * x))


def _gate_prep(g, gate_form, A_log, dt_bias, lower_bound):
    """The log-decay the recurrence uses, and the lower bound left to clamp it.

    gate_form None: g is the log-decay (clamped by lower_bound inside the recurrence).
    gate_form "softplus" / "safe": g is the gate input, turned into the log-decay by
    ``gate`` above (page "K3/kda/ops/api.py", ``use_gate_in_kernel``; the
    unbounded form takes no lower bound, the safe form needs one).
    """
    if gate_form is None:
        return g, lower_bound
    if gate_form not in ("softplus", "safe"):
        raise ValueError("gate_form must be None, 'softplus' or 'safe'")
    if A_log is None:
        raise ValueError("the in-kernel gate needs A_log")
    if gate_form == "safe" and lower_bound is None:
        raise ValueError("the safe gate needs lower_bound")
    g = _f64(g)
    H, Dk = g.shape[-2], g.shape[-1]
    dt = None if dt_bias is None else _f64(dt_bias).reshape(H, Dk)
    return gate(g, _f64(A_log).reshape(H), dt, lower_bound if gate_form == "safe" else None), None


def recurrent(q, k, v, g, beta, *, scale=None, initial_state=None, cu_seqlens=None,
              use_qk_l2norm=True, lower_bound=None, beta_is_logit=True,
              gate_form=None, A_log=None, dt_bias=None, nthreads=0):
    """Form R (the definition). Returns (o [T_total,H,d_v], final_state [N,H,d_k,d_v]).

    ``beta`` holds logits (sigmoid applied per token) unless ``beta_is_logit`` is
    False (then probabilities, used as given); ``g`` holds per-channel log-decays,
    ``lower_bound`` clamps g from below, ``scale`` defaults to 1/sqrt(d_k). With
    ``gate_form`` = "softplus" or "safe", ``g`` is the gate input instead (see
    ``_gate_prep``).
    """
    g, lower_bound = _gate_prep(g, gate_form, A_log, dt_bias, lower_bound)
    q, k, v, g, beta, cu, S0, N, H, Dk, Dv = _prep(q, k, v, g, beta, cu_seqlens, initial_state)
    if scale is None:
        scale = 1.0 / np.sqrt(Dk)
    o = np.zeros((q.shape[0], H, Dv))
    S = np.zeros((N, H, Dk, Dv))
    rc = _load().kda_oracle_recurrent(
        N, H, Dk, Dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(S0), _ptr(o), _ptr(S),
        int(bool(use_qk_l2norm)), int(lower_bound is not None),
        float(lower_bound if lower_bound is not None else 0.0), int(bool(beta_is_logit)),
        _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_recurrent failed ({rc})")
    return o, S


def chunkwise(q, k, v, g, beta, *, scale=None, initial_state=None, cu_seqlens=None,
              use_qk_l2norm=True, lower_bound=None, beta_is_logit=True,
              gate_form=None, A_log=None, dt_bias=None, chunk_size=64, nthreads=0):
    """Form C (chunkwise WY/UT). Same arguments and results as ``recurrent``."""
    g, lower_bound = _gate_prep(g, gate_form, A_log, dt_bias, lower_bound)
    q, k, v, g, beta, cu, S0, N, H, Dk, Dv = _prep(q, k, v, g, beta, cu_seqlens, initial_state)
    if scale is None:
        scale = 1.0 / np.sqrt(Dk)
    o = np.zeros((q.shape[0], H, Dv))
    S = np.zeros((N, H, Dk, Dv))
    rc = _load().kda_oracle_chunkwise(
        N, H, Dk, Dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(S0), _ptr(o), _ptr(S),
        int(bool(use_qk_l2norm)), int(lower_bound is not None),
        float(lower_bound if lower_bound is not None else 0.0), int(bool(beta_is_logit)),
        int(chunk_size), _threads(nthreads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_chunkwise failed ({rc})")
    return o, S


# --------------------------------------------------------------------------- decode token

def silu(x):
    """x * sigmoid(x) in fp64 (page "atlas_core/kimi_k3/kda.rs", `conv_update`)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def conv_update(state, x, w):
    """Causal depthwise convolution + SiLU over one new sample per channel.

    ``state`` [..., C, K] holds each channel's last K inputs, oldest first; it is
    shifted one slot towards the start, ``x`` [..., C] is written into the last
    slot, and y[c] = silu(sum_k w[c, k] state[c, k]) with ``w`` [C, K]
    (page "atlas_core/kimi_k3/kda.rs", `conv_update`). Returns (y, new_state) in
    fp64; the input state is not modified.
    """
    st = _f64(state).copy()
    xs = _f64(x)
    ww = _f64(w)
    st[..., :-1] = st[..., 1:]
    st[..., -1] = xs
    return silu(np.sum(ww * st, axis=-1)), st


def output_gate(core, g, head_dim, eps):
    """Full-rank output gate: sigmoid(g) * RMSNorm(core) per head of ``head_dim``
    channels, RMSNorm(x) = x / sqrt(mean(x^2) + eps), no weight (page
    "atlas_core/kimi_k3/kda.rs", `full_rank_output_gate`)."""
    c = _f64(core)
    gg = _f64(g)
    shp = c.shape
    c = c.reshape(*shp[:-1], -1, head_dim)
    gg = gg.reshape(*shp[:-1], -1, head_dim)
    inv = 1.0 / np.sqrt(np.mean(c * c, axis=-1, keepdims=True) + float(eps))
    return (c * inv / (1.0 + np.exp(-gg))).reshape(shp)


def decode_token(x, conv_w, conv_state, g, beta, state, *, H, Dk, Dv, scale=None,
                 use_qk_l2norm=True, lower_bound=None, beta_is_logit=True, gate_form=None,
                 A_log=None, dt_bias=None, g_out=None, norm_eps=1e-6):
    """One decode token for N sequences (page "atlas_core/kimi_k3/kda.rs",
    `kda_decode_token`, with `full_rank_output_gate` when ``g_out`` is given):
    the conv update + SiLU over the pre-conv projections ``x`` [N, H*(2Dk+Dv)]
    laid out q | k | v, then the recurrent step (form R) on that token from
    ``state`` [N, H, Dk, Dv], then, with ``g_out`` [N, H*Dv], the output gate.

    ``conv_w`` [H*(2Dk+Dv), K], ``conv_state`` [N, H*(2Dk+Dv), K]; ``g`` [N, H, Dk]
    and ``beta`` [N, H] as in ``recurrent``. Returns (o [N, H, Dv],
    new_conv_state, new_state), fp64.
    """
    y, cs = conv_update(conv_state, x, conv_w)
    N = y.shape[0]
    qd, vd = H * Dk, H * Dv
    q = y[:, :qd].reshape(N, H, Dk)
    k = y[:, qd:2 * qd].reshape(N, H, Dk)
    v = y[:, 2 * qd:2 * qd + vd].reshape(N, H, Dv)
    cu = np.arange(N + 1, dtype=np.int64)  # one token per sequence
    o, S = recurrent(q, k, v, _f64(g).reshape(N, H, Dk), _f64(beta).reshape(N, H), scale=scale,
                     initial_state=state, cu_seqlens=cu, use_qk_l2norm=use_qk_l2norm,
                     lower_bound=lower_bound, beta_is_logit=beta_is_logit, gate_form=gate_form,
                     A_log=A_log, dt_bias=dt_bias)
    if g_out is not None:
        o = output_gate(o.reshape(N, H * Dv), _f64(g_out).reshape(N, H * Dv), Dv, norm_eps).reshape(N, H, Dv)
    return o, cs, S


# --------------------------------------------------------------------------- backward

def backward(q, k, v, g, beta, do, *, dS_final=None, scale=None, initial_state=None, cu_seqlens=None,
             use_qk_l2norm=True, lower_bound=None, beta_is_logit=True):
    """Gradients of the chunkwise forward: given the output cotangent ``do``
    [T_total, H, d_v] (and optionally ``dS_final`` [N, H, d_k, d_v] for the final
    states), returns (dq, dk, dv, dg, dbeta, dS0) as fp64 numpy arrays, dS0 of the
    initial states [N, H, d_k, d_v] (zeros when none are given).

    The forward is the recurrence of page "atlas_core/kimi_k3/kda.rs" (module doc,
    `l2norm_rows`, `kda_recurrent_step`) written out token by token in fp64 torch
    operations, with the clamp g <- max(g, lower_bound) and beta a logit (sigmoid)
    or a probability as in ``recurrent``; the gradients are its reverse-mode
    derivatives (torch autograd: the definition differentiated, no other form).
    Python loops over tokens: small cases only.
    """
    import torch

    def t64(x, grad=False):
        if x is None:
            return None
        a = torch.from_numpy(_f64(x).copy())
        return a.requires_grad_(grad)

    q, k, v, g, beta, cu, S0, N, H, Dk, Dv = _prep(q, k, v, g, beta, cu_seqlens, initial_state)
    dO = _f64(do).reshape(q.shape[0], H, Dv)
    tq, tk, tv, tg, tb = (t64(x, True) for x in (q, k, v, g, beta))
    tS0 = t64(S0 if S0 is not None else np.zeros((N, H, Dk, Dv)), True)
    if scale is None:
        scale = 1.0 / np.sqrt(Dk)
    outs, finals = [], []
    for n in range(N):
        S = tS0[n]
        for t in range(int(cu[n]), int(cu[n + 1])):
            qt, kt = tq[t], tk[t]
            if use_qk_l2norm:
                qt = qt / torch.sqrt((qt * qt).sum(-1, keepdim=True) + 1e-6)
                kt = kt / torch.sqrt((kt * kt).sum(-1, keepdim=True) + 1e-6)
            gt = tg[t] if lower_bound is None else torch.clamp(tg[t], min=float(lower_bound))
            b = torch.sigmoid(tb[t]) if beta_is_logit else tb[t]
            S = torch.exp(gt)[..., :, None] * S                      # decay along the key axis
            delta = b[:, None] * (tv[t] - torch.einsum("hkv,hk->hv", S, kt))
            S = S + kt[..., :, None] * delta[..., None, :]
            outs.append((t, scale * torch.einsum("hkv,hk->hv", S, qt)))
        finals.append(S)
    loss = sum((o * torch.from_numpy(dO[t])).sum() for t, o in outs)
    if dS_final is not None:
        dSf = _f64(dS_final).reshape(N, H, Dk, Dv)
        loss = loss + sum((finals[n] * torch.from_numpy(dSf[n])).sum() for n in range(N))
    if not torch.is_tensor(loss):  # no tokens and no final-state cotangent
        z = lambda a: np.zeros(a.shape)
        return z(q), z(k), z(v), z(g), z(beta), np.zeros((N, H, Dk, Dv))
    grads = torch.autograd.grad(loss, (tq, tk, tv, tg, tb, tS0), allow_unused=True)
    return tuple(np.zeros(x.shape) if gr is None else gr.detach().numpy()
                 for gr, x in zip(grads, (tq, tk, tv, tg, tb, tS0)))
