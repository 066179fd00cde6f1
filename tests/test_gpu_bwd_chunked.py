"""GPU parity of the chunked tensor-core backward (bf16, d_k = d_v = 128, a gate lower
bound >= -5) against the fp64 oracle (`oracle.backward`, the derivatives of the token
recurrence of page "atlas_core/kimi_k3/kda.rs", pinned by finite differences): the
options of the `chunk_kda` boundary of page "K3/kda/ops/api.py" (no final-state
cotangent, no in-kernel L2 norm, beta as a probability, an active clamp, no initial
state), ragged chunk tails, empty sequences in a varlen batch, and the segment form of
the cotangent chain (few long sequences)."""
import pytest
import torch

import kda_inputs as KI
import oracle
from kda_check import check

pytestmark = pytest.mark.gpu

DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")
DTYPE = torch.bfloat16


def draw(lens, H, seed, init=True):
    inp = KI.draw_chunk(1, sum(lens), H, 128, 128, dtype=DTYPE, seed=seed, seqlens=lens, init_state=init)
    gen = torch.Generator().manual_seed(seed + 1000)
    inp["do"] = torch.randn(inp["v"].shape, generator=gen).to(DTYPE)
    inp["dSf"] = torch.randn(len(lens), H, 128, 128, generator=gen) * 0.5
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
        check(f"{tag} {name}", gt, wt, DTYPE)


def test_chunked_path_is_taken():
    """A bf16 d128 call with a lower bound of -5 launches the chunked form: the forward's
    four launches (set-up, intra-chunk pass, exact records, state pass with the saves),
    the cotangent chain and the chunk-local kernel -- not the token sweeps."""
    import kimi_delta_attention_20_b200 as kda
    from kimi_delta_attention_20_b200 import _abi
    inp = draw((200,), 2, seed=300)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    lib = _abi.load()
    n0 = lib.kda_launch_count()
    kda.chunk_kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["do"], dfinal_state=d["dSf"],
                      initial_state=d["initial_state"], lower_bound=-5.0)
    torch.cuda.synchronize()
    assert lib.kda_launch_count() - n0 == 6


@pytest.mark.parametrize("case", ["base", "no_final", "no_l2", "prob", "clamp_active", "no_initial"])
def test_chunked_options(case):
    lens = (70, 200, 1, 64)
    inp = draw(lens, 2, seed=310 + len(case), init=case != "no_initial")
    kw = {}
    if case == "no_final":
        kw["final"] = False
    elif case == "no_l2":
        inp["k"] = (inp["k"].float() / 8.0).to(DTYPE)
        inp["q"] = (inp["q"].float() / 8.0).to(DTYPE)
        kw["l2"] = False
    elif case == "prob":
        inp["beta"] = torch.sigmoid(inp["beta"].float()).to(DTYPE)
        kw["prob"] = True
    elif case == "clamp_active":
        inp["g"] = (inp["g"].float() * 4.0).to(DTYPE)  # many gates below the bound
        kw["lower_bound"] = -1.0
    run_and_compare(inp, tag=case, **kw)


def test_chunked_ragged_and_empty():
    """Chunk tails of every kind (1, 63, 64, 65, 127, 129 tokens) and empty sequences."""
    run_and_compare(draw((1, 63, 0, 64, 65, 0, 127, 129), 3, seed=320), tag="ragged")


def test_chunked_steepest_gates():
    """Every gate at the bound: the in-block factors reach e^{8 |lb|}."""
    inp = draw((300,), 2, seed=330)
    inp["g"] = torch.full_like(inp["g"], -5.0)
    run_and_compare(inp, tag="steep")


@pytest.mark.parametrize("lens", [(1500,), (700, 1500, 64, 0)])
def test_chunked_segments(lens):
    """Few long sequences: the cotangent chain runs over the forward's segments (from zero,
    back over M^T, then from the leaving cotangents); initial states, the final-state
    cotangent and the initial-state gradient cross every segment boundary."""
    run_and_compare(draw(lens, 2, seed=340 + len(lens)), tag=f"segments {lens}")
