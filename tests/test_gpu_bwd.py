"""GPU parity of the chunk_kda backward (kda_chunk_bwd) against the fp64 oracle
(`oracle.backward`, the derivatives of the token recurrence of page
"atlas_core/kimi_k3/kda.rs", pinned by finite differences), and of the autograd
route through `chunk_kda`. Lengths straddle the 16-token checkpoints of the
reverse sweep.
"""
import numpy as np
import pytest
import torch

import kda_inputs as KI
import oracle
from kda_check import check

pytestmark = pytest.mark.gpu

DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")


def draw(lens, H, Dk, Dv, dtype, seed, **kw):
    inp = KI.draw_chunk(1, sum(lens), H, Dk, Dv, dtype=dtype, seed=seed, seqlens=lens, init_state=True, **kw)
    gen = torch.Generator().manual_seed(seed + 1000)
    inp["do"] = torch.randn(inp["v"].shape, generator=gen).to(dtype)
    inp["dSf"] = torch.randn(inp["initial_state"].shape, generator=gen) * 0.5
    return inp


def run_and_compare(inp, dtype, *, lower_bound=None, l2=True, prob=False, final=True, tag=""):
    import kimi_delta_attention_20_b200 as kda
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    got = kda.chunk_kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["do"],
                            dfinal_state=d["dSf"] if final else None, initial_state=d["initial_state"],
                            use_qk_l2norm_in_kernel=l2, use_beta_sigmoid_in_kernel=not prob,
                            lower_bound=lower_bound, cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    want = oracle.backward(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], inp["beta"][0], inp["do"][0],
                           dS_final=inp["dSf"] if final else None, initial_state=inp["initial_state"],
                           cu_seqlens=inp["cu_seqlens"], use_qk_l2norm=l2, lower_bound=lower_bound,
                           beta_is_logit=not prob)
    for name, gt, wt in zip(NAMES, got, want):
        if name != "dS0":
            gt = gt[0]
        check(f"{tag} {name}", gt, wt, dtype)
    return got


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(32, 32), (64, 64), (128, 128), (32, 64), (128, 32)])
def test_backward_matches_oracle(dims, dtype):
    Dk, Dv = dims
    inp = draw((15, 16, 17, 1, 33), 2, Dk, Dv, dtype, seed=Dk + Dv)
    run_and_compare(inp, dtype, lower_bound=-5.0, tag=f"{dims}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_many_heads(dtype):
    """More CTAs than SMs (5 sequences x 8 heads x 4 column slices at d 128): the
    reverse sweep then runs one warp group per CTA doing both of its jobs in turn;
    fewer (the other tests) run the two groups side by side."""
    inp = draw((33, 17, 1, 16, 40), 8, 128, 128, dtype, seed=97)
    run_and_compare(inp, dtype, lower_bound=-5.0, tag="many heads")


@pytest.mark.parametrize("case", ["no_final", "no_l2", "prob", "clamp_active", "empty_seqs"])
def test_backward_options(case):
    dtype = torch.float32
    lens = (0, 20, 0, 9) if case == "empty_seqs" else (20, 9)
    inp = draw(lens, 2, 64, 64, dtype, seed=90 + len(case))
    kw = dict(lower_bound=-5.0)
    if case == "no_final":
        kw["final"] = False
    elif case == "no_l2":
        inp["k"] = (inp["k"].float() / 8.0).to(dtype)
        kw["l2"] = False
    elif case == "prob":
        inp["beta"] = torch.sigmoid(inp["beta"].float()).to(dtype)
        kw["prob"] = True
    elif case == "clamp_active":
        inp["g"] = (inp["g"].float() * 4.0).to(dtype)  # many gates below the bound
        kw["lower_bound"] = -1.0
    run_and_compare(inp, dtype, tag=case, **kw)


@pytest.mark.parametrize("case", ["d32_fp32_varlen", "d64_bf16", "d128_bf16", "d64_fp32_options"])
def test_backward_segments(case):
    """Few (sequence, head) chains of long sequences: the backward cuts every sequence
    into segments, gets each segment's entering state and leaving state cotangent from
    two widened runs and two chain walks, and sweeps the segments side by side. An
    empty sequence, a short one (trailing segments empty), initial states, the
    final-state cotangent and the initial-state gradient through the chains."""
    if case == "d32_fp32_varlen":
        inp = draw((700, 1500, 64, 0), 1, 32, 32, torch.float32, seed=140)
        run_and_compare(inp, torch.float32, lower_bound=-5.0, tag=case)
    elif case == "d64_bf16":
        inp = draw((300, 900), 2, 64, 64, torch.bfloat16, seed=141)
        run_and_compare(inp, torch.bfloat16, lower_bound=-5.0, tag=case)
    elif case == "d128_bf16":
        inp = draw((1000,), 2, 128, 128, torch.bfloat16, seed=142)
        run_and_compare(inp, torch.bfloat16, lower_bound=-5.0, tag=case)
    else:
        inp = draw((500, 260), 1, 64, 64, torch.float32, seed=143)
        inp["beta"] = torch.sigmoid(inp["beta"].float())
        run_and_compare(inp, torch.float32, final=False, prob=True, tag=case)


def test_autograd_through_chunk_kda():
    """loss.backward() through chunk_kda gives kda_chunk_bwd's gradients, which match the oracle."""
    import kimi_delta_attention_20_b200 as kda
    inp = draw((24, 40), 2, 32, 64, torch.float32, seed=95)
    leaves = {n: inp[n].to(DEV).requires_grad_(True) for n in ("q", "k", "v", "g", "beta", "initial_state")}
    o, S = kda.chunk_kda(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["beta"],
                         initial_state=leaves["initial_state"], output_final_state=True,
                         use_qk_l2norm_in_kernel=True, lower_bound=-5.0, cu_seqlens=inp["cu_seqlens"].to(DEV))
    loss = (o * inp["do"].to(DEV)).sum() + (S * inp["dSf"].to(DEV)).sum()
    loss.backward()
    want = oracle.backward(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], inp["beta"][0], inp["do"][0],
                           dS_final=inp["dSf"], initial_state=inp["initial_state"], cu_seqlens=inp["cu_seqlens"],
                           lower_bound=-5.0)
    for name, leaf, wt in zip(NAMES, ("q", "k", "v", "g", "beta", "initial_state"), want):
        gt = leaves[leaf].grad
        check(f"autograd {name}", gt if leaf == "initial_state" else gt[0], wt, torch.float32)


def test_autograd_rejects_in_kernel_gate():
    import kimi_delta_attention_20_b200 as kda
    inp = KI.draw_chunk(1, 8, 2, 32, 32, seed=96, device=DEV, gate="input")
    q = inp["q"].requires_grad_(True)
    params = KI.draw_gate_params(2, 32, seed=96, device=DEV)
    with pytest.raises(NotImplementedError):
        kda.chunk_kda(q, inp["k"], inp["v"], inp["g"], inp["beta"], use_gate_in_kernel=True,
                      A_log=params["A_log"], use_qk_l2norm_in_kernel=True)


def test_backward_full_size_sampled():
    """The backward leg of bench.py at its full size (B1 T8192 H16 d128, bf16, lower bound
    -5, output and final-state cotangents) in the launch configuration it times. The
    gradients of a head's last 1024 tokens depend on the rest of the sequence only
    through the state entering token 7168, so for heads 0 and 15 the oracle runs the
    forward recurrence to that state (`oracle.recurrent`) and the backward from there
    (`oracle.backward` with that initial state and the final-state cotangent)."""
    import kimi_delta_attention_20_b200 as kda
    wl = KI.CHUNK_WORKLOADS[2]
    inp = KI.chunk_inputs(wl)
    gen = torch.Generator().manual_seed(wl.seed + 1000)
    do = torch.randn(inp["v"].shape, generator=gen).to(wl.dtype)
    dSf = torch.randn(1, wl.H, wl.Dk, wl.Dv, generator=gen) * 0.5
    d = {n: inp[n].to(DEV) for n in ("q", "k", "v", "g", "beta")}
    got = kda.chunk_kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], do.to(DEV), dfinal_state=dSf.to(DEV),
                            use_qk_l2norm_in_kernel=True, lower_bound=wl.lower_bound)
    torch.cuda.synchronize()
    t_split = wl.T - 1024
    for h in (0, wl.H - 1):
        sl = lambda x: x[0, :, h:h + 1]
        pre = [sl(inp[n])[:t_split] for n in ("q", "k", "v", "g", "beta")]
        _, S_mid = oracle.recurrent(*pre, lower_bound=wl.lower_bound)
        post = [sl(inp[n])[t_split:] for n in ("q", "k", "v", "g", "beta")]
        want = oracle.backward(*post, sl(do)[t_split:], dS_final=dSf[:, h:h + 1], initial_state=S_mid,
                               lower_bound=wl.lower_bound)
        for name, gt, wt in zip(NAMES[:5], got[:5], want[:5]):
            check(f"full-size h{h} {name}", gt[0, t_split:, h:h + 1], wt, wl.dtype)
