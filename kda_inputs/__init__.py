"""Seeded synthetic inputs for KDA, shared by the tests, the benchmark and the
smoke check.

This module only draws random tensors; it holds none of the operator's
arithmetic and imports neither the CUDA library nor the oracle. The recipe
follows the five workloads the operator is measured on (chunk forward on
three geometries plus a tiny fp32 case, and a batched decode step):

* q, k, v ~ N(0, 1); q and k are L2-normalised inside the operator.
* gate input: g = -exp(a_h) * softplus(z), z ~ N(0, 1) per element,
  a_h ~ U(-2, 0.5) per head (the unbounded gate of page
  "atlas_core/kimi_k3/kda.rs", `bounded_gate` with lower_bound None, used
  here only to draw realistic log-decays); clamped workloads pass
  lower_bound = -5 to the operator, which applies the clamp.
* decode: g = -5 * sigmoid(N(0, 1)).
* in-kernel gate cases: the raw gate input z ~ N(0, 1) is passed as g, with
  A_log = log(U(1, 16)) per head and dt_bias = the inverse softplus of
  dt = exp(U(log 1e-3, log 1e-1)) per channel (the initialisation page
  "KDA ⇄ FLA Parity in Primus", section "What changed and why" (A), names
  as FLA's; `draw_gate_params`).
* beta logits ~ N(0, 1); beta probabilities (cases that pass beta as given)
  ~ U(0, 1).
* initial states ~ N(0, 1) * 0.1, fp32.

Everything is drawn in fp32 with one ``torch.Generator`` seeded with the
workload index, in the fixed order q, k, v, z, a_h, beta, initial_state,
then cast once (round-to-nearest-even) to the workload dtype. The cast
tensors are what both the CUDA path and the oracle consume. The draw is
device-specific (a CUDA generator gives different numbers from a CPU one),
so tests that compare against the oracle copy the drawn tensors to the host.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch
import torch.nn.functional as F


@dataclasses.dataclass(frozen=True)
class ChunkWorkload:
    name: str
    B: int
    T: int
    H: int
    Dk: int
    Dv: int
    dtype: torch.dtype
    seed: int
    init_state: bool
    final_state: bool
    lower_bound: Optional[float]
    seqlens: Optional[Sequence[int]] = None  # varlen packing (B must be 1)
    scale: Optional[float] = None
    chunk_size: int = 64
    gate_in_kernel: bool = False   # g holds the gate input; A_log / dt_bias drawn too
    beta_prob: bool = False        # beta holds probabilities instead of logits

    @property
    def tokens(self) -> int:
        return self.B * self.T

    @property
    def n_seqs(self) -> int:
        return len(self.seqlens) if self.seqlens is not None else self.B


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    N: int
    H: int
    Dk: int
    Dv: int
    steps: int
    dtype: torch.dtype
    seed: int
    lower_bound: Optional[float] = None


CHUNK_WORKLOADS = {
    0: ChunkWorkload("tiny-fp32 B1 T128 H2 d32", 1, 128, 2, 32, 32, torch.float32, 0,
                     init_state=False, final_state=True, lower_bound=None,
                     scale=1.0 / math.sqrt(32)),
    1: ChunkWorkload("twin B4 T2048 H8 d32", 4, 2048, 8, 32, 32, torch.bfloat16, 1,
                     init_state=True, final_state=True, lower_bound=None),
    2: ChunkWorkload("B1 T8192 H16 d128 lb-5", 1, 8192, 16, 128, 128, torch.bfloat16, 2,
                     init_state=False, final_state=True, lower_bound=-5.0),
    4: ChunkWorkload("varlen 4096/8192/12288/7168 H96 d128 lb-5", 1, 31744, 96, 128, 128,
                     torch.bfloat16, 4, init_state=True, final_state=True, lower_bound=-5.0,
                     seqlens=(4096, 8192, 12288, 7168)),
    # one KDA layer of the 300M pure-KDA model in training: micro-batch 128 x 2048 tokens,
    # 8 heads, d_k 32, d_v 64, in-kernel unbounded gate, beta already a probability
    5: ChunkWorkload("300M layer B128 T2048 H8 dk32 dv64 gate-in-kernel", 128, 2048, 8, 32, 64,
                     torch.bfloat16, 5, init_state=False, final_state=False, lower_bound=None,
                     gate_in_kernel=True, beta_prob=True),
}

DECODE_WORKLOADS = {
    3: DecodeWorkload("decode N64 H96 d128 x256", 64, 96, 128, 128, 256, torch.bfloat16, 3),
}


def _gen(device, seed):
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return gen


def draw_chunk(B, T, H, Dk, Dv, *, dtype=torch.bfloat16, seed=0, device="cpu",
               seqlens=None, init_state=False, gate="unbounded", beta="logit"):
    """Draw one chunk-forward input set.

    Returns a dict with q, k, g [B,T,H,Dk], v [B,T,H,Dv], beta [B,T,H],
    initial_state [N,H,Dk,Dv] fp32 or None, cu_seqlens int32 [N+1] or None.
    ``gate`` is "unbounded" (-exp(a_h) softplus(z)), "decode" (-5 sigmoid(z))
    or "input" (z itself, for the in-kernel gate). ``beta`` is "logit"
    (N(0, 1)) or "prob" (U(0, 1)).
    """
    gen = _gen(device, seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    q = torch.randn(B, T, H, Dk, **f32)
    k = torch.randn(B, T, H, Dk, **f32)
    v = torch.randn(B, T, H, Dv, **f32)
    z = torch.randn(B, T, H, Dk, **f32)
    a_h = torch.rand(H, **f32) * 2.5 - 2.0
    beta_t = torch.randn(B, T, H, **f32)
    if beta == "prob":
        beta_t = torch.rand(B, T, H, **f32)
    elif beta != "logit":
        raise ValueError(beta)
    if gate == "unbounded":
        g = -torch.exp(a_h).view(1, 1, H, 1) * F.softplus(z)
    elif gate == "decode":
        g = -5.0 * torch.sigmoid(z)
    elif gate == "input":
        g = z
    else:
        raise ValueError(gate)
    del z
    cu = None
    N = B
    if seqlens is not None:
        if B != 1 or sum(seqlens) != T:
            raise ValueError("varlen packing needs B == 1 and sum(seqlens) == T")
        N = len(seqlens)
        cu = torch.zeros(N + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(list(seqlens), dtype=torch.int64), 0).to(torch.int32)
        cu = cu.to(device)
    S0 = torch.randn(N, H, Dk, Dv, **f32) * 0.1 if init_state else None
    out = dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), g=g.to(dtype),
               beta=beta_t.to(dtype), initial_state=S0, cu_seqlens=cu)
    return out


def draw_gate_params(H, Dk, *, seed=0, device="cpu"):
    """Parameters of the in-kernel gate, fp32: A_log [H] = log(U(1, 16)) and
    dt_bias [H, Dk] = inverse softplus of dt = exp(U(log 1e-3, log 1e-1))
    (dt floored at 1e-4), the initialisation named for FLA's KDA layer."""
    gen = _gen(device, 1000 + int(seed))
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    A_log = torch.log(torch.rand(H, **f32) * 15.0 + 1.0)
    lo, hi = math.log(1e-3), math.log(1e-1)
    dt = torch.exp(torch.rand(H, Dk, **f32) * (hi - lo) + lo).clamp_min(1e-4)
    dt_bias = dt + torch.log(-torch.expm1(-dt))
    return dict(A_log=A_log, dt_bias=dt_bias)


def chunk_inputs(idx_or_wl, device="cpu"):
    """Inputs of a named chunk-forward workload (see CHUNK_WORKLOADS)."""
    wl = CHUNK_WORKLOADS[idx_or_wl] if isinstance(idx_or_wl, int) else idx_or_wl
    out = draw_chunk(wl.B, wl.T, wl.H, wl.Dk, wl.Dv, dtype=wl.dtype, seed=wl.seed,
                     device=device, seqlens=wl.seqlens, init_state=wl.init_state,
                     gate="input" if wl.gate_in_kernel else "unbounded",
                     beta="prob" if wl.beta_prob else "logit")
    if wl.gate_in_kernel:
        out.update(draw_gate_params(wl.H, wl.Dk, seed=wl.seed, device=device))
    return out


def draw_decode(N, H, Dk, Dv, steps, *, dtype=torch.bfloat16, seed=3, device="cpu",
                gate="decode", beta="logit"):
    """Decode inputs: initial state [N,H,Dk,Dv] fp32 ~ 0.1 N(0,1), then per step
    q, k [steps,N,H,Dk], v [steps,N,H,Dv], g = -5 sigmoid(z) [steps,N,H,Dk]
    (or z itself with gate="input"), beta [steps,N,H] logits (or U(0, 1)
    probabilities with beta="prob")."""
    gen = _gen(device, seed)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    S0 = torch.randn(N, H, Dk, Dv, **f32) * 0.1
    q = torch.randn(steps, N, H, Dk, **f32).to(dtype)
    k = torch.randn(steps, N, H, Dk, **f32).to(dtype)
    v = torch.randn(steps, N, H, Dv, **f32).to(dtype)
    z = torch.randn(steps, N, H, Dk, **f32)
    if gate == "decode":
        g = (-5.0 * torch.sigmoid(z)).to(dtype)
    elif gate == "input":
        g = z.to(dtype)
    else:
        raise ValueError(gate)
    beta_t = torch.randn(steps, N, H, **f32)
    if beta == "prob":
        beta_t = torch.rand(steps, N, H, **f32)
    elif beta != "logit":
        raise ValueError(beta)
    return dict(state=S0, q=q, k=k, v=v, g=g, beta=beta_t.to(dtype))


def decode_inputs(idx_or_wl, device="cpu", steps=None):
    wl = DECODE_WORKLOADS[idx_or_wl] if isinstance(idx_or_wl, int) else idx_or_wl
    return draw_decode(wl.N, wl.H, wl.Dk, wl.Dv, wl.steps if steps is None else steps,
                       dtype=wl.dtype, seed=wl.seed, device=device)


def draw_token(N, H, Dk, Dv, K, steps, *, dtype=torch.bfloat16, seed=0, device="cpu", gate="decode"):
    """Serving decode-token inputs: pre-conv projections x [steps, N, H*(2Dk+Dv)] ~ N(0,1),
    conv weights [H*(2Dk+Dv), K] ~ N(0, 1/K), conv windows [N, H*(2Dk+Dv), K] ~ N(0,1),
    gates [steps, N, H, Dk] = -5 sigmoid(z) (or z itself with gate="input"), beta
    logits [steps, N, H], output-gate inputs [steps, N, H, Dv] ~ N(0,1), and the
    initial state [N, H, Dk, Dv] ~ 0.1 N(0,1) fp32. Drawn in that order with one
    generator seeded with ``seed``, on ``device``; token tensors cast to ``dtype``."""
    gen = torch.Generator(device=device).manual_seed(seed)
    C = H * (2 * Dk + Dv)
    rn = lambda *shape: torch.randn(*shape, generator=gen, device=device)
    x = rn(steps, N, C).to(dtype)
    w = rn(C, K) / K ** 0.5
    cs = rn(N, C, K)
    z = rn(steps, N, H, Dk)
    g = (z if gate == "input" else -5.0 * torch.sigmoid(z)).to(dtype)
    beta = rn(steps, N, H).to(dtype)
    g_out = rn(steps, N, H, Dv).to(dtype)
    S0 = rn(N, H, Dk, Dv) * 0.1
    return dict(x=x, w=w, cs=cs, g=g, beta=beta, g_out=g_out, S0=S0)
