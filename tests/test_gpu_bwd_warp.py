"""GPU parity of the micro-chunk backward (bf16, d_k = 32, d_v 32 or 64, a gate lower bound
>= -10, many chains: one warp per (sequence, head) over 16-token micro-chunks) against
the fp64 oracle (`oracle.backward`, the derivatives of the token recurrence of page
"atlas_core/kimi_k3/kda.rs", pinned by finite differences), with the options of the
`chunk_kda` boundary of page "K3/kda/ops/api.py"."""
import pytest
import torch

import kda_inputs as KI
import oracle
from kda_check import check

pytestmark = pytest.mark.gpu

DEV = "cuda"
DT = torch.bfloat16
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")
# 32 sequences x 8 heads = 256 (sequence, head) chains: the form's threshold
LENS = (1, 15, 16, 17, 31, 33, 40, 0, 64, 65, 7, 48, 2, 20, 50, 16, 3, 29, 61, 44, 12, 35, 9, 58, 25, 0, 47, 33, 18, 63, 5, 70)
H = 8


def draw(dv, seed, init=True, lens=LENS):
    inp = KI.draw_chunk(1, sum(lens), H, 32, dv, dtype=DT, seed=seed, seqlens=lens, init_state=init)
    gen = torch.Generator().manual_seed(seed + 1000)
    inp["do"] = torch.randn(inp["v"].shape, generator=gen).to(DT)
    inp["dSf"] = torch.randn(len(lens), H, 32, dv, generator=gen) * 0.5
    return inp


def run_and_compare(inp, *, lower_bound=-5.0, l2=True, prob=False, final=True, tag=""):
    import kimi_delta_attention_20_b200 as kda
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    got = kda.chunk_kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["do"],
                            dfinal_state=d["dSf"] if final else None, initial_state=d.get("initial_state"),
                            use_qk_l2norm_in_kernel=l2, use_beta_sigmoid_in_kernel=not prob,
                            lower_bound=lower_bound, cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    want = oracle.backward(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], inp["beta"][0], inp["do"][0],
                           dS_final=inp["dSf"] if final else None, initial_state=inp.get("initial_state"),
                           cu_seqlens=inp["cu_seqlens"], use_qk_l2norm=l2, lower_bound=lower_bound,
                           beta_is_logit=not prob)
    for name, gt, wt in zip(NAMES, got, want):
        if name != "dS0":
            gt = gt[0]
        check(f"{tag} {name}", gt, wt, DT)


def test_warp_bwd_path_taken():
    """Two launches: the micro-chunk forward saving the states, then the backward."""
    import kimi_delta_attention_20_b200 as kda
    from kimi_delta_attention_20_b200 import _abi
    inp = draw(64, seed=600)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    lib = _abi.load()
    n0 = lib.kda_launch_count()
    kda.chunk_kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["do"], dfinal_state=d["dSf"],
                      initial_state=d["initial_state"], lower_bound=-5.0, cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    assert lib.kda_launch_count() - n0 == 2


@pytest.mark.parametrize("dv", [32, 64])
def test_warp_bwd_matches_oracle(dv):
    run_and_compare(draw(dv, seed=610 + dv), tag=f"d_v{dv}")


@pytest.mark.parametrize("case", ["no_final", "no_l2", "prob", "clamp_active", "no_initial", "bound_10"])
def test_warp_bwd_options(case):
    inp = draw(64, seed=620 + len(case), init=case != "no_initial")
    kw = {}
    if case == "no_final":
        kw["final"] = False
    elif case == "no_l2":
        inp["k"] = (inp["k"].float() / 6.0).to(DT)
        inp["q"] = (inp["q"].float() / 6.0).to(DT)
        kw["l2"] = False
    elif case == "prob":
        inp["beta"] = torch.sigmoid(inp["beta"].float()).to(DT)
        kw["prob"] = True
    elif case == "clamp_active":
        inp["g"] = (inp["g"].float() * 4.0).to(DT)
        kw["lower_bound"] = -1.0
    elif case == "bound_10":  # every gate at the bound the form accepts: factors up to e^80
        inp["g"] = torch.full_like(inp["g"], -10.0)
        kw["lower_bound"] = -10.0
    run_and_compare(inp, tag=case, **kw)


@pytest.mark.parametrize("dv", [32, 64])
def test_warp_bwd_many_chains(dv):
    """600 chains (75 ragged sequences x 8 heads): more than four per SM, so the saving forward
    is the split form (the entering states leave through its own transposing stores)."""
    lens = tuple((7 * i) % 41 + (i % 3) for i in range(75))
    run_and_compare(draw(dv, seed=640 + dv, lens=lens), tag=f"many d_v{dv}")
