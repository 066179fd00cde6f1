"""Tolerances and oracle plumbing shared by the GPU parity tests.

Tolerances (the operator's stated bars, applied to o and the final state
separately):
  * fp32 inputs: max|got - want| <= 1e-4 * max(max|want|, 1e-6), the
    scale-relative shape of page "memra-engine tests/kda_fixture_gpu.rs"
    (`check`, `scale_of`) with the 1e-4 bar;
  * bf16 inputs: ||got - want||_F / ||want||_F <= 2e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def check(name, got, want, dtype):
    got, want = _np(got), _np(want)
    assert got.shape == want.shape, f"{name}: shape {got.shape} vs {want.shape}"
    assert np.all(np.isfinite(got)), f"{name}: non-finite values from the GPU"
    if dtype == torch.float32:
        scale = max(float(np.abs(want).max(initial=0.0)), 1e-6)
        err = float(np.abs(got - want).max(initial=0.0))
        assert err <= TOL_F32 * scale, f"{name}: max abs err {err:.3e} > {TOL_F32:.0e} * {scale:.3e}"
        return err / scale
    den = float(np.linalg.norm(want))
    err = float(np.linalg.norm(got - want))
    rel = err / max(den, 1e-30)
    assert rel <= TOL_BF16, f"{name}: rel Frobenius err {rel:.3e} > {TOL_BF16:.0e}"
    return rel


def oracle_chunk(inp, *, heads=None, seqs=None, scale=None, lower_bound=None, l2=True,
                 beta_is_logit=True, gate_form=None, A_log=None, dt_bias=None):
    """Form R on (a subset of) a chunk-forward input dict; returns per-sequence
    (o [T_n, h, Dv], S [h, Dk, Dv]) lists over the chosen sequences and heads.
    The gate arguments are those of ``oracle.recurrent`` (A_log [H], dt_bias
    [H, Dk] over all heads; the chosen heads are taken from them)."""
    q, k, v, g, beta = (inp[n] for n in ("q", "k", "v", "g", "beta"))
    B, T, H, _ = q.shape
    cu = inp.get("cu_seqlens")
    if cu is not None:
        cu = cu.cpu().numpy().astype(np.int64)
        bounds = [(int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]
        flat = lambda x: x[0]
    else:
        bounds = [(n * T, (n + 1) * T) for n in range(B)]
        flat = lambda x: x.reshape(B * T, *x.shape[2:])
    hs = list(range(H)) if heads is None else list(heads)
    ns = list(range(len(bounds))) if seqs is None else list(seqs)
    S0 = inp.get("initial_state")
    if A_log is not None:
        A_log = _np(A_log).reshape(H)[hs]
    if dt_bias is not None:
        dt_bias = _np(dt_bias).reshape(H, -1)[hs]
    out = []
    for n in ns:
        a, b = bounds[n]
        sl = lambda x: flat(x)[a:b][:, hs]
        s0 = None if S0 is None else S0[n:n + 1, hs]
        o, S = oracle.recurrent(sl(q), sl(k), sl(v), sl(g), flat(beta)[a:b][:, hs], scale=scale,
                                initial_state=s0, use_qk_l2norm=l2, lower_bound=lower_bound,
                                beta_is_logit=beta_is_logit, gate_form=gate_form, A_log=A_log,
                                dt_bias=dt_bias)
        out.append((a, b, o, S[0]))
    return out
