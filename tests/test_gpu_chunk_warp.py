"""GPU parity of the micro-chunk tensor-core forward (bf16, d_k 32 or 64, d_v 32 or 64:
16-token micro-chunks, one warp per (sequence, head) at d_k = 32, a CTA of two warps at
d_k = 64) against form R, the token recurrence of page "atlas_core/kimi_k3/kda.rs"
(`chunk_kda` of page "K3/kda/ops/api.py"). This form takes the bf16 calls of those
shapes that the segment form of the recurrence does not: many chains, short sequences,
or d_k != d_v."""
import pytest
import torch

import kda_inputs as KI
from kda_check import check, oracle_chunk

pytestmark = pytest.mark.gpu

DEV = "cuda"
DT = torch.bfloat16


def kda_mod():
    import kimi_delta_attention_20_b200 as kda
    return kda


def run(inp, **kw):
    kda = kda_mod()
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    return kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d.get("initial_state"),
                         output_final_state=True, cu_seqlens=d.get("cu_seqlens"), **kw)


def compare(inp, o, S, tag, **okw):
    ref = oracle_chunk({k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}, **okw)
    H = inp["q"].shape[2]
    B, T = inp["q"].shape[:2]
    o_flat = o.reshape(B * T, H, -1)
    for n, (a, b, o_ref, S_ref) in enumerate(ref):
        for h in range(H):
            if b > a:
                check(f"{tag} o seq{n} h{h}", o_flat[a:b][:, [h]], o_ref[:, [h]], DT)
            check(f"{tag} S seq{n} h{h}", S[n, [h]], S_ref[[h]], DT)


DIMS = [(32, 32), (32, 64), (64, 32), (64, 64)]


@pytest.mark.parametrize("dims", DIMS)
def test_warp_ragged_varlen(dims):
    """Micro-chunk tails of every kind and empty sequences in a varlen batch."""
    dk, dv = dims
    lens = [0, 1, 15, 16, 17, 33, 100, 0, 257, 64]
    inp = KI.draw_chunk(1, sum(lens), 3, dk, dv, dtype=DT, seed=500 + dk + dv, seqlens=lens, init_state=True)
    o, S = run(inp, use_qk_l2norm_in_kernel=True)
    compare(inp, o, S, f"ragged {dims}")


@pytest.mark.parametrize("dims", DIMS)
def test_warp_steep_gates(dims):
    """Gates that drop by up to ~100 per token: the middle-row split would leave the fp32
    range, so those micro-chunks take the exponent-difference products; others keep the
    tensor-core split."""
    dk, dv = dims
    inp = KI.draw_chunk(2, 120, 2, dk, dv, dtype=DT, seed=510 + dk + dv, init_state=True)
    g = inp["g"].float()
    g[:, 20:50] = g[:, 20:50] * 40.0
    inp["g"] = g.to(DT)
    o, S = run(inp, use_qk_l2norm_in_kernel=True)
    compare(inp, o, S, f"steep {dims}")


@pytest.mark.parametrize("dk", [32, 64])
@pytest.mark.parametrize("form", ["softplus", "safe"])
def test_warp_in_kernel_gate(form, dk):
    """The in-kernel gate forms (page "atlas_core/kimi_k3/kda.rs" `bounded_gate`)."""
    inp = KI.draw_chunk(2, 150, 4, dk, 64, dtype=DT, seed=520 + len(form) + dk, init_state=True, gate="input")
    gen = torch.Generator().manual_seed(521)
    A_log = torch.empty(4).uniform_(-2.0, 0.5, generator=gen)
    dt_bias = torch.randn(4, dk, generator=gen) * 0.5
    kw = dict(use_gate_in_kernel=True, A_log=A_log.to(DEV), dt_bias=dt_bias.to(DEV), use_qk_l2norm_in_kernel=True)
    okw = dict(gate_form=form, A_log=A_log, dt_bias=dt_bias)
    if form == "safe":
        kw.update(safe_gate=True, lower_bound=-5.0)
        okw["lower_bound"] = -5.0
    o, S = run(inp, **kw)
    compare(inp, o, S, f"gate {form}", **okw)


@pytest.mark.parametrize("dk", [32, 64])
def test_warp_options(dk):
    """beta as a probability, no in-kernel L2 norm, an explicit scale, no initial state."""
    inp = KI.draw_chunk(2, 90, 2, dk, 32, dtype=DT, seed=530 + dk, beta="prob")
    inp["k"] = (inp["k"].float() / 6.0).to(DT)
    with pytest.warns(RuntimeWarning):
        o, S = run(inp, use_qk_l2norm_in_kernel=False, use_beta_sigmoid_in_kernel=False, scale=0.37)
    compare(inp, o, S, "options", l2=False, beta_is_logit=False, scale=0.37)


@pytest.mark.parametrize("dk", [32, 64])
def test_warp_many_chains(dk):
    """1,024 chains (one wave), a sample of sequences checked on every head."""
    inp = KI.draw_chunk(64, 96, 16, dk, 64, dtype=DT, seed=540 + dk, init_state=True)
    o, S = run(inp, use_qk_l2norm_in_kernel=True, lower_bound=-5.0)
    sub = {n: inp[n][[0, 31, 63]] for n in ("q", "k", "v", "g", "beta")}
    sub["initial_state"] = inp["initial_state"][[0, 31, 63]]
    compare(sub, o[[0, 31, 63]], S[[0, 31, 63]], "many", lower_bound=-5.0)


@pytest.mark.parametrize("B", [37, 38])
def test_warp_forms_at_four_chains_per_sm(B):
    """The two d_k = 32 forms on either side of their switch: 592 chains (four per SM) take
    the producer/consumer form, 608 the split form; a sample of sequences on every head."""
    inp = KI.draw_chunk(B, 48, 16, 32, 64, dtype=DT, seed=550 + B, init_state=True)
    o, S = run(inp, use_qk_l2norm_in_kernel=True, lower_bound=-5.0)
    pick = [0, B // 2, B - 1]
    sub = {n: inp[n][pick] for n in ("q", "k", "v", "g", "beta")}
    sub["initial_state"] = inp["initial_state"][pick]
    compare(sub, o[pick], S[pick], f"B{B}", lower_bound=-5.0)


def test_warp_widened_run_split_form():
    """d_k = d_v = 32 with 296 chains of 256 tokens: the segment form cuts each sequence into
    four segments, so its widened run has 1,184 segment chains and takes the split form's
    widened variant (the [M | N] state, fp32 outputs); entering states cross every segment."""
    inp = KI.draw_chunk(37, 256, 8, 32, 32, dtype=DT, seed=560, init_state=True)
    o, S = run(inp, use_qk_l2norm_in_kernel=True)
    pick = [0, 18, 36]
    sub = {n: inp[n][pick] for n in ("q", "k", "v", "g", "beta")}
    sub["initial_state"] = inp["initial_state"][pick]
    compare(sub, o[pick], S[pick], "widened split")
