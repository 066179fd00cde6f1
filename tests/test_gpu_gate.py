"""GPU parity of the in-kernel gate and of beta given as a probability.

The `chunk_kda` boundary of page "K3/kda/ops/api.py" can form the log-decay in
the kernel from the gate input (`use_gate_in_kernel`, `A_log`, `dt_bias`, the
unbounded softplus form or `safe_gate` with a lower bound) and can take beta
as a probability (`use_beta_sigmoid_in_kernel=False`); page
"atlas_core/kimi_k3/kda.rs" writes the gate as `bounded_gate`. Both sides
consume the same drawn tensors; the oracle applies the gate in fp64.
"""
import math

import numpy as np
import pytest
import torch

import kda_inputs as KI
import oracle
from kda_check import check
from test_gpu_parity import DEV, compare_chunk, kda_mod

pytestmark = pytest.mark.gpu


def gate_kwargs(form, params, *, with_dt=True, lb=-5.0):
    kw = dict(use_gate_in_kernel=True, A_log=params["A_log"].to(DEV),
              dt_bias=params["dt_bias"].to(DEV) if with_dt else None)
    okw = dict(gate_form=form, A_log=params["A_log"], dt_bias=params["dt_bias"] if with_dt else None)
    if form == "safe":
        kw.update(safe_gate=True, lower_bound=lb)
    return kw, okw, (lb if form == "safe" else None)


def run(inp, *, final=True, **kw):
    kda = kda_mod()
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    return kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"],
                         initial_state=d.get("initial_state"), output_final_state=final,
                         use_qk_l2norm_in_kernel=True, cu_seqlens=d.get("cu_seqlens"), **kw)


# tensor-core path (bf16, d 128) over ragged varlen sequences, and the CUDA-core
# path (fp32 and bf16 at d 32 / 64)
GEOMS = [
    ("tc", torch.bfloat16, 128, (1, 63, 64, 65, 200, 330)),
    ("simt-f32", torch.float32, 32, (1, 64, 130, 77)),
    ("simt-bf16", torch.bfloat16, 64, (65, 128, 5)),
]


@pytest.mark.parametrize("form", ["softplus", "safe"])
@pytest.mark.parametrize("with_dt", [True, False])
@pytest.mark.parametrize("geom", GEOMS, ids=[g[0] for g in GEOMS])
def test_chunk_in_kernel_gate(geom, form, with_dt):
    tag, dtype, d, seqlens = geom
    H = 4
    inp = KI.draw_chunk(1, sum(seqlens), H, d, d, dtype=dtype, seed=31, seqlens=seqlens,
                        init_state=True, gate="input")
    params = KI.draw_gate_params(H, d, seed=31)
    kw, okw, lb = gate_kwargs(form, params, with_dt=with_dt)
    o, S = run(inp, **kw)
    compare_chunk(inp, o, S, dtype, lower_bound=lb, tag=f"{tag}-{form}", **okw)


@pytest.mark.parametrize("geom", GEOMS, ids=[g[0] for g in GEOMS])
def test_chunk_beta_probability(geom):
    tag, dtype, d, seqlens = geom
    H = 3
    inp = KI.draw_chunk(1, sum(seqlens), H, d, d, dtype=dtype, seed=32, seqlens=seqlens,
                        init_state=True, beta="prob")
    o, S = run(inp, use_beta_sigmoid_in_kernel=False, lower_bound=-5.0)
    compare_chunk(inp, o, S, dtype, lower_bound=-5.0, beta_is_logit=False, tag=f"{tag}-prob")


def test_chunk_gate_and_beta_probability_together():
    H, d, seqlens = 2, 128, (96, 160)
    inp = KI.draw_chunk(1, sum(seqlens), H, d, d, dtype=torch.bfloat16, seed=33, seqlens=seqlens,
                        gate="input", beta="prob")
    params = KI.draw_gate_params(H, d, seed=33)
    kw, okw, lb = gate_kwargs("safe", params)
    o, S = run(inp, use_beta_sigmoid_in_kernel=False, **kw)
    compare_chunk(inp, o, S, torch.bfloat16, lower_bound=lb, beta_is_logit=False, tag="both", **okw)


def test_chunk_steep_in_kernel_gate_takes_exact_fallback():
    """rate e^A_log = 60 on a large gate input: per-block spans far above the
    factorisation's limit, so the chunks go through the exact CUDA-core blocks."""
    H, d, T = 2, 128, 256
    inp = KI.draw_chunk(1, T, H, d, d, dtype=torch.bfloat16, seed=34, gate="input")
    inp["g"] = (inp["g"].float() + 2.0).to(torch.bfloat16)
    params = dict(A_log=torch.full((H,), math.log(60.0)), dt_bias=torch.zeros(H, d))
    kw, okw, _ = gate_kwargs("softplus", params)
    o, S = run(inp, **kw)
    assert torch.isfinite(o).all()
    compare_chunk(inp, o, S, torch.bfloat16, tag="steep-gate", **okw)


def test_workload_d128_T8192_safe_gate_in_kernel():
    """The d 128, T 8192, H 16 workload with its lower bound -5 applied through the
    safe in-kernel gate instead of a clamp; sampled heads checked."""
    wl = KI.CHUNK_WORKLOADS[2]
    inp = KI.draw_chunk(wl.B, wl.T, wl.H, wl.Dk, wl.Dv, dtype=wl.dtype, seed=wl.seed, device=DEV,
                        gate="input")
    params = KI.draw_gate_params(wl.H, wl.Dk, seed=wl.seed)
    kw, okw, lb = gate_kwargs("safe", params, lb=wl.lower_bound)
    o, S = run(inp, **kw)
    compare_chunk(inp, o, S, wl.dtype, heads=[0, 7, 15], lower_bound=lb, tag="d128-safe", **okw)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mode", ["softplus", "safe", "prob"])
def test_decode_gate_and_beta_modes(dtype, mode):
    kda = kda_mod()
    N, H, d, steps = 3, 4, 128, 5
    inp = KI.draw_decode(N, H, d, d, steps, dtype=dtype, seed=35,
                         gate="input" if mode != "prob" else "decode",
                         beta="prob" if mode == "prob" else "logit")
    params = KI.draw_gate_params(H, d, seed=35)
    if mode == "prob":
        kw, okw = dict(use_beta_sigmoid_in_kernel=False), dict(beta_is_logit=False)
    else:
        kw, okw, lb = gate_kwargs(mode, params)
        okw["lower_bound"] = lb
    state = inp["state"].to(DEV).clone()
    outs = []
    for t in range(steps):
        outs.append(kda.recurrent_step(inp["q"][t].to(DEV), inp["k"][t].to(DEV), inp["v"][t].to(DEV),
                                       inp["g"][t].to(DEV), inp["beta"][t].to(DEV), state, **kw))
    for n in range(N):
        o_ref, S_ref = oracle.recurrent(inp["q"][:, n], inp["k"][:, n], inp["v"][:, n],
                                        inp["g"][:, n], inp["beta"][:, n],
                                        initial_state=inp["state"][n:n + 1], **okw)
        check(f"decode-{mode} o seq{n}", torch.stack([x[n] for x in outs]), o_ref, dtype)
        check(f"decode-{mode} S seq{n}", state[n], S_ref[0], dtype)


def test_gate_argument_errors():
    kda = kda_mod()
    inp = KI.draw_chunk(1, 64, 2, 128, 128, seed=36, device=DEV, gate="input")
    args = (inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"])
    with pytest.raises(ValueError):
        kda.chunk_kda(*args, use_qk_l2norm_in_kernel=True, use_gate_in_kernel=True)  # no A_log
    A = torch.zeros(2, device=DEV)
    with pytest.raises(ValueError):
        kda.chunk_kda(*args, use_qk_l2norm_in_kernel=True, use_gate_in_kernel=True, A_log=A,
                      safe_gate=True)  # safe gate needs a bound
    with pytest.raises(ValueError):
        kda.chunk_kda(*args, use_qk_l2norm_in_kernel=True, use_gate_in_kernel=True,
                      A_log=A.double())
    with pytest.raises(ValueError):
        kda.chunk_kda(*args, use_qk_l2norm_in_kernel=True, use_gate_in_kernel=True, A_log=A,
                      dt_bias=torch.zeros(3, device=DEV))
