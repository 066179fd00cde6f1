"""GPU parity of the fused serving decode token (conv update + SiLU, recurrent step,
output gate; page "atlas_core/kimi_k3/kda.rs": `conv_update`, `kda_decode_token`,
`full_rank_output_gate`) against the fp64 oracle, token after token so that both
the conv windows and the recurrent state are carried by the kernel.
"""
import numpy as np
import pytest
import torch

import kda_inputs as KI
import oracle
from kda_check import check

pytestmark = pytest.mark.gpu

DEV = "cuda"


def draw(N, H, Dk, Dv, K, steps, dtype, seed, gate="decode"):
    return KI.draw_token(N, H, Dk, Dv, K, steps, dtype=dtype, seed=seed, gate=gate)


def run_tokens(inp, steps, *, gated, oracle_kw=None, gpu_kw=None, eps=1e-6):
    import kimi_delta_attention_20_b200 as kda
    N, H, Dk, Dv = inp["S0"].shape
    cs_d = inp["cs"].clone().to(DEV)
    S_d = inp["S0"].clone().to(DEV)
    w_d = inp["w"].to(DEV)
    cs_o, S_o = inp["cs"].double().numpy(), inp["S0"].double().numpy()
    outs = []
    for t in range(steps):
        o = kda.decode_token(inp["x"][t].to(DEV), w_d, cs_d, inp["g"][t].to(DEV), inp["beta"][t].to(DEV), S_d,
                             g_out=inp["g_out"][t].to(DEV) if gated else None, norm_eps=eps, **(gpu_kw or {}))
        o_ref, cs_o, S_o = oracle.decode_token(inp["x"][t], inp["w"], cs_o, inp["g"][t], inp["beta"][t], S_o,
                                               H=H, Dk=Dk, Dv=Dv, g_out=inp["g_out"][t] if gated else None,
                                               norm_eps=eps, **(oracle_kw or {}))
        outs.append((o, o_ref))
    torch.cuda.synchronize()
    return outs, cs_d, cs_o, S_d, S_o


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("K", [4, 1, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(32, 32), (64, 64), (128, 128), (32, 64), (128, 32)])
def test_decode_token_matches_oracle(dims, dtype, K, gated):
    Dk, Dv = dims
    inp = draw(3, 2, Dk, Dv, K, 3, dtype, seed=Dk + 3 * Dv + K)
    outs, cs_d, cs_o, S_d, S_o = run_tokens(inp, 3, gated=gated)
    for t, (o, o_ref) in enumerate(outs):
        check(f"token {t} o", o, o_ref, dtype)
    # the windows hold inputs only: exact up to the input dtype's cast (fp32 holds them exactly)
    np.testing.assert_array_equal(cs_d.cpu().double().numpy(), cs_o)
    check("token state", S_d, S_o, dtype)


@pytest.mark.parametrize("form", ["softplus", "safe", "prob"])
def test_decode_token_gate_forms(form):
    H, D = 3, 64
    inp = draw(2, H, D, D, 4, 2, torch.bfloat16, seed=71, gate="input" if form != "prob" else "decode")
    params = KI.draw_gate_params(H, D, seed=71)
    gpu_kw, oracle_kw = {}, {}
    if form == "prob":
        inp["beta"] = torch.rand(inp["beta"].shape, generator=torch.Generator().manual_seed(72)).to(torch.bfloat16)
        gpu_kw = dict(use_beta_sigmoid_in_kernel=False)
        oracle_kw = dict(beta_is_logit=False)
    else:
        gpu_kw = dict(use_gate_in_kernel=True, A_log=params["A_log"].to(DEV), dt_bias=params["dt_bias"].to(DEV))
        oracle_kw = dict(gate_form=form, A_log=params["A_log"], dt_bias=params["dt_bias"])
        if form == "safe":
            gpu_kw.update(safe_gate=True, lower_bound=-5.0)
            oracle_kw.update(lower_bound=-5.0)
    outs, _, _, S_d, S_o = run_tokens(inp, 2, gated=True, oracle_kw=oracle_kw, gpu_kw=gpu_kw)
    for t, (o, o_ref) in enumerate(outs):
        check(f"{form} token {t} o", o, o_ref, torch.bfloat16)
    check(f"{form} state", S_d, S_o, torch.bfloat16)


def test_decode_token_output_gate_eps():
    """The RMSNorm epsilon is the caller's: 1e-6 and 1e-5 give different, each exact, outputs."""
    inp = draw(2, 2, 32, 32, 4, 1, torch.float32, seed=73)
    for eps in (1e-6, 1e-5, 0.0):
        outs, _, _, _, _ = run_tokens(inp, 1, gated=True, eps=eps)
        check(f"eps {eps}", outs[0][0], outs[0][1], torch.float32)


def test_decode_token_prefix_hit_on_gpu():
    """Page "atlas_core/kimi_k3/kda.rs" `prefix_hit_wrong_slot_diverges` at a supported
    head size: token 3 from the state saved after token 2 equals the sequential decode
    (bit for bit: same kernel, same inputs), from the state after token 1 it moves."""
    import kimi_delta_attention_20_b200 as kda
    H, D, K = 2, 32, 4
    C = 3 * H * D
    inp = draw(1, H, D, D, K, 3, torch.float32, seed=74)
    w = torch.full((C, K), 0.25, device=DEV)
    cs = torch.zeros(1, C, K, device=DEV)
    S = torch.zeros(1, H, D, D, device=DEV)
    snaps = []
    for t in range(2):
        kda.decode_token(inp["x"][t].to(DEV), w, cs, inp["g"][t].to(DEV), inp["beta"][t].to(DEV), S)
        snaps.append((cs.clone(), S.clone()))
    args = (inp["x"][2].to(DEV), w)
    rest = (inp["g"][2].to(DEV), inp["beta"][2].to(DEV))
    y_seq = kda.decode_token(*args, cs, *rest, S)
    cs_hit, S_hit = snaps[1][0].clone(), snaps[1][1].clone()
    y_hit = kda.decode_token(*args, cs_hit, *rest, S_hit)
    assert torch.equal(y_hit, y_seq) and torch.equal(cs_hit, cs) and torch.equal(S_hit, S)
    cs_w, S_w = snaps[0][0].clone(), snaps[0][1].clone()
    y_wrong = kda.decode_token(*args, cs_w, *rest, S_w)
    assert (y_wrong - y_hit).abs().max().item() > 1e-4


def test_decode_token_production_geometry_sampled():
    """The production layer (H 96, d 128, conv kernel 4, lower bound -5) for 64
    sequences, one token with the output gate; three sequences checked on all heads
    (sequences are independent)."""
    import kimi_delta_attention_20_b200 as kda
    N, H, D, K = 64, 96, 128, 4
    inp = draw(N, H, D, D, K, 1, torch.bfloat16, seed=75)
    cs = inp["cs"].clone().to(DEV)
    S = inp["S0"].clone().to(DEV)
    o = kda.decode_token(inp["x"][0].to(DEV), inp["w"].to(DEV), cs, inp["g"][0].to(DEV), inp["beta"][0].to(DEV),
                         S, g_out=inp["g_out"][0].to(DEV), lower_bound=-5.0)
    torch.cuda.synchronize()
    for n in (0, 31, 63):
        o_ref, cs_ref, S_ref = oracle.decode_token(
            inp["x"][0][n:n + 1], inp["w"], inp["cs"][n:n + 1], inp["g"][0][n:n + 1], inp["beta"][0][n:n + 1],
            inp["S0"][n:n + 1], H=H, Dk=D, Dv=D, g_out=inp["g_out"][0][n:n + 1], lower_bound=-5.0)
        check(f"prod o n{n}", o[n:n + 1], o_ref, torch.bfloat16)
        check(f"prod S n{n}", S[n:n + 1], S_ref, torch.bfloat16)
        np.testing.assert_array_equal(cs[n:n + 1].cpu().double().numpy(), cs_ref)


def test_decode_token_state_out_ping_pong():
    """The serving token with the new state written to a second buffer: the old state
    stays intact and the result is bit for bit the in-place one (conv windows are
    updated in place either way)."""
    import kimi_delta_attention_20_b200 as kda
    N, H, Dk, Dv, K, steps = 3, 2, 128, 128, 4, 4
    inp = draw(N, H, Dk, Dv, K, steps, torch.bfloat16, seed=9)
    w_d = inp["w"].to(DEV)
    cs_in, cs_pp = inp["cs"].clone().to(DEV), inp["cs"].clone().to(DEV)
    S_in = inp["S0"].clone().to(DEV)
    S_a, S_b = S_in.clone(), torch.empty_like(S_in)
    for t in range(steps):
        args = dict(g_out=inp["g_out"][t].to(DEV), norm_eps=1e-6)
        x, g, b = inp["x"][t].to(DEV), inp["g"][t].to(DEV), inp["beta"][t].to(DEV)
        o_in = kda.decode_token(x, w_d, cs_in, g, b, S_in, **args)
        before = S_a.clone()
        o_pp = kda.decode_token(x, w_d, cs_pp, g, b, S_a, state_out=S_b, **args)
        torch.cuda.synchronize()
        assert torch.equal(S_a, before), "the read-only state was written"
        assert torch.equal(o_in, o_pp)
        S_a, S_b = S_b, S_a
    assert torch.equal(S_in, S_a)
    assert torch.equal(cs_in, cs_pp)
