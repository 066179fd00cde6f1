"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every input is drawn by the seeded generators of kda_inputs and the same
(cast) tensors feed both sides. The named workloads run at their full sizes
and launch configuration; where the oracle would take too long on all heads
it checks a sample of (sequence, head) pairs, which is exact because pairs
are independent. Boundary lengths 1/7/63/64/65/130, decode-after-prefill
(t0, steps) pairs and split points come from page
"memra-engine tests/kda_fixture_gpu.rs" (gates 1-3).
"""
import math

import numpy as np
import pytest
import torch

import kda_inputs as KI
import oracle
from kda_check import check, oracle_chunk

pytestmark = pytest.mark.gpu

DEV = "cuda"


def kda_mod():
    import kimi_delta_attention_20_b200 as kda
    return kda


def run_chunk(inp, wl=None, *, scale=None, lower_bound=None, final=True, l2=True, **kw):
    kda = kda_mod()
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    return kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=scale,
                         initial_state=d.get("initial_state"), output_final_state=final,
                         use_qk_l2norm_in_kernel=l2, lower_bound=lower_bound,
                         cu_seqlens=d.get("cu_seqlens"), **kw)


def compare_chunk(inp, o, S, dtype, *, heads=None, seqs=None, scale=None, lower_bound=None,
                  l2=True, tag="", per_head=False, **okw):
    """o and the final states against form R, per sequence over the chosen heads, or
    with ``per_head`` per (sequence, head) so that no head hides under the others."""
    ref = oracle_chunk({k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()},
                       heads=heads, seqs=seqs, scale=scale, lower_bound=lower_bound, l2=l2, **okw)
    H = inp["q"].shape[2]
    hs = list(range(H)) if heads is None else list(heads)
    ns = list(range(len(ref))) if seqs is None else list(seqs)
    B, T = inp["q"].shape[:2]
    o_flat = o.reshape(B * T, H, -1)
    groups = [([h], [j]) for j, h in enumerate(hs)] if per_head else [(hs, list(range(len(hs))))]
    for (a, b, o_ref, S_ref), n in zip(ref, ns):
        for hg, jg in groups:
            name = f"seq{n} h{hg[0]}" if per_head else f"seq{n}"
            if b > a:
                check(f"{tag} o {name}", o_flat[a:b][:, hg], o_ref[:, jg], dtype)
            if S is not None:
                check(f"{tag} S {name}", S[n, hg], S_ref[jg], dtype)


# --- the named workloads, full size ------------------------------------------

def test_workload_tiny_fp32():
    wl = KI.CHUNK_WORKLOADS[0]
    inp = KI.chunk_inputs(wl, device="cpu")
    o, S = run_chunk(inp, scale=wl.scale)
    compare_chunk(inp, o, S, wl.dtype, scale=wl.scale, tag="tiny-fp32")


def test_workload_twin_d32():
    wl = KI.CHUNK_WORKLOADS[1]
    inp = KI.chunk_inputs(wl, device="cpu")
    o, S = run_chunk(inp)
    compare_chunk(inp, o, S, wl.dtype, tag="twin")


def test_workload_d128_T8192_clamped():
    wl = KI.CHUNK_WORKLOADS[2]
    inp = KI.chunk_inputs(wl, device=DEV)
    o, S = run_chunk(inp, lower_bound=wl.lower_bound)
    compare_chunk(inp, o, S, wl.dtype, heads=[0, 5, 11, 15], lower_bound=wl.lower_bound,
                  tag="d128", per_head=True)


def test_workload_varlen_H96():
    wl = KI.CHUNK_WORKLOADS[4]
    inp = KI.chunk_inputs(wl, device=DEV)
    o, S = run_chunk(inp, lower_bound=wl.lower_bound)
    # the first and the last head and eight drawn ones, each (sequence, head) on its own
    rng = np.random.default_rng(0)
    heads = sorted({0, 95} | set(rng.choice(np.arange(1, 95), size=8, replace=False).tolist()))
    compare_chunk(inp, o, S, wl.dtype, heads=heads, lower_bound=wl.lower_bound, tag="varlen",
                  per_head=True)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()


@pytest.mark.parametrize("case", ["batch", "varlen", "gate_forms"])
def test_segmented_state_chains(case):
    """Few (sequence, head) chains and long sequences: the two-pass forward cuts every
    sequence into chunk-aligned segments, runs pass 2 over them three times (transitions,
    offsets, outputs) and chains the segment states in between. Ragged last segments,
    an empty sequence and a one-chunk sequence (its trailing segments empty), initial
    and final states."""
    kw = dict(dtype=torch.bfloat16, init_state=True)
    if case == "batch":
        inp = KI.draw_chunk(2, 1100, 2, 128, 128, seed=120, **kw)
        okw, lb = {}, -5.0
    elif case == "varlen":
        inp = KI.draw_chunk(1, 2264, 3, 128, 128, seed=121, seqlens=(700, 1500, 64, 0), **kw)
        okw, lb = {}, None
    else:
        inp = KI.draw_chunk(1, 1400, 2, 128, 128, seed=122, gate="input", **kw)
        inp.update(KI.draw_gate_params(2, 128, seed=122))
        okw, lb = dict(gate_form="safe", A_log=inp["A_log"], dt_bias=inp["dt_bias"]), -5.0
    if case == "gate_forms":
        kda = kda_mod()
        d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        o, S = kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=d["initial_state"],
                             output_final_state=True, use_qk_l2norm_in_kernel=True, use_gate_in_kernel=True,
                             safe_gate=True, lower_bound=lb, A_log=d["A_log"], dt_bias=d["dt_bias"])
        sub = {k: v for k, v in inp.items() if k not in ("A_log", "dt_bias")}
        compare_chunk(sub, o, S, torch.bfloat16, lower_bound=lb, tag="seg-gate", **okw)
    else:
        o, S = run_chunk(inp, lower_bound=lb)
        compare_chunk(inp, o, S, torch.bfloat16, lower_bound=lb, tag=f"seg-{case}")


@pytest.mark.parametrize("case", ["d32_batch", "d64_varlen", "d32_fp32"])
def test_segmented_recurrent(case):
    """The recurrent forward (shapes without the tensor-core path) with few chains: every
    sequence is cut into segments, one run of the token recurrence over them carries the
    transition (from the identity, v = 0) and the offset (from zero) as one widened state,
    the segment states are chained, and the outputs are fixed up from the entering states.
    Empty trailing segments, an empty sequence, initial states."""
    if case == "d32_batch":
        inp = KI.draw_chunk(2, 1100, 2, 32, 32, seed=130, dtype=torch.bfloat16, init_state=True)
        lb, dt = -5.0, torch.bfloat16
    elif case == "d64_varlen":
        inp = KI.draw_chunk(1, 2264, 3, 64, 64, seed=131, dtype=torch.bfloat16, init_state=True,
                            seqlens=(700, 1500, 64, 0))
        lb, dt = None, torch.bfloat16
    else:
        inp = KI.draw_chunk(1, 3000, 1, 32, 32, seed=132, dtype=torch.float32, init_state=False)
        lb, dt = None, torch.float32
    o, S = run_chunk(inp, lower_bound=lb)
    compare_chunk(inp, o, S, dt, lower_bound=lb, tag=f"rseg-{case}")


def test_workload_300m_layer():
    """One layer of the 300M pure-KDA model (d_k 32, d_v 64, in-kernel gate, beta as a
    probability), full size; 6 of the 128 sequences checked on all 8 heads."""
    wl = KI.CHUNK_WORKLOADS[5]
    inp = KI.chunk_inputs(wl, device=DEV)
    kda = kda_mod()
    o, S = kda.chunk_kda(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                         A_log=inp["A_log"], dt_bias=inp["dt_bias"], use_qk_l2norm_in_kernel=True,
                         use_gate_in_kernel=True, use_beta_sigmoid_in_kernel=False)
    assert S is None and torch.isfinite(o).all()
    sub = {n: inp[n][[0, 17, 63, 64, 100, 127]].cpu() for n in ("q", "k", "v", "g", "beta")}
    sub["initial_state"] = None
    compare_chunk(sub, o[[0, 17, 63, 64, 100, 127]], None, wl.dtype, tag="300m",
                  gate_form="softplus", A_log=inp["A_log"].cpu(), dt_bias=inp["dt_bias"].cpu(),
                  beta_is_logit=False)


def test_workload_decode_256_steps():
    wl = KI.DECODE_WORKLOADS[3]
    kda = kda_mod()
    inp = KI.decode_inputs(wl, device=DEV)
    state = inp["state"].clone()
    outs = []
    for t in range(wl.steps):
        outs.append(kda.recurrent_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t],
                                       inp["beta"][t], state))
    o = torch.stack(outs).cpu()  # [steps, N, H, Dv]
    # 16 (sequence, head) pairs, the first and the last among them; every step's output
    # of each pair is checked on its own, and the pair's state after the 256 steps
    rng = np.random.default_rng(1)
    pairs = [(0, 0), (wl.N - 1, wl.H - 1)] + list(zip(rng.choice(wl.N, 14).tolist(),
                                                       rng.choice(wl.H, 14).tolist()))
    for n, h in pairs:
        sl = lambda x: x[:, n, h:h + 1].cpu()
        o_ref, S_ref = oracle.recurrent(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]),
                                        inp["beta"][:, n, h:h + 1].cpu(),
                                        initial_state=inp["state"][n:n + 1, h:h + 1].cpu())
        for t in range(wl.steps):
            check(f"decode o n{n} h{h} step{t}", o[t, n, h], o_ref[t, 0], wl.dtype)
        check(f"decode S n{n} h{h}", state[n, h], S_ref[0, 0], wl.dtype)


# --- boundaries, shapes, flags ------------------------------------------------

DIMS = [(32, 32), (64, 64), (128, 128), (32, 64), (32, 128), (128, 64)]


@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 130])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", DIMS)
def test_chunk_boundary_lengths(T, dtype, dims):
    Dk, Dv = dims
    inp = KI.draw_chunk(2, T, 3, Dk, Dv, dtype=dtype, seed=T * 31 + Dk + Dv, init_state=True)
    o, S = run_chunk(inp)
    compare_chunk(inp, o, S, dtype, tag=f"T{T}")


@pytest.mark.parametrize("T", [1, 31, 32, 33, 100])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(32, 64), (64, 32), (128, 128)])
def test_chunk_size_32(T, dtype, dims):
    """32-token chunks (api.py's chunk_size 32) give the same operator result."""
    Dk, Dv = dims
    inp = KI.draw_chunk(2, T, 3, Dk, Dv, dtype=dtype, seed=T * 17 + Dk, init_state=True)
    o, S = run_chunk(inp, chunk_size=32, lower_bound=-5.0)
    compare_chunk(inp, o, S, dtype, lower_bound=-5.0, tag=f"C32 T{T}")


def test_chunk_size_rule():
    """chunk sizes <= 32 select 32-token chunks, larger ones 64 (api.py's rule); both
    agree with each other to rounding on the same input."""
    inp = KI.draw_chunk(1, 150, 2, 32, 64, dtype=torch.float32, seed=77, init_state=True)
    o16, S16 = run_chunk(inp, chunk_size=16)
    o32, S32 = run_chunk(inp, chunk_size=32)
    o64, S64 = run_chunk(inp, chunk_size=100)
    assert torch.equal(o16, o32) and torch.equal(S16, S32)
    torch.testing.assert_close(o32, o64, rtol=1e-5, atol=1e-5)
    torch.testing.assert_close(S32, S64, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("lb", [None, -5.0, -0.5, -0.3, -2.7])
def test_chunk_lower_bound(lb):
    """Bounds that are bf16 values and bounds that are not (-0.3, -2.7: the clamped
    gate then carries a low-order part into the in-chunk sum)."""
    inp = KI.draw_chunk(1, 200, 2, 128, 128, dtype=torch.bfloat16, seed=5, init_state=True)
    o, S = run_chunk(inp, lower_bound=lb)
    compare_chunk(inp, o, S, torch.bfloat16, lower_bound=lb, tag=f"lb{lb}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_chunk_scale_and_no_l2norm(dtype):
    inp = KI.draw_chunk(1, 130, 2, 64, 64, dtype=dtype, seed=6)
    # keep unnormalised keys short so the delta rule stays contractive
    inp["k"] = (inp["k"].float() / 8.0).to(dtype)
    with pytest.warns(RuntimeWarning):
        o, S = run_chunk(inp, scale=0.37, l2=False)
    compare_chunk(inp, o, S, dtype, scale=0.37, l2=False, tag="nol2")


def test_chunk_varlen_ragged():
    lens = [0, 1, 64, 65, 130, 7, 0, 200]
    inp = KI.draw_chunk(1, sum(lens), 3, 128, 128, dtype=torch.bfloat16, seed=7,
                        seqlens=lens, init_state=True)
    o, S = run_chunk(inp, lower_bound=-5.0)
    compare_chunk(inp, o, S, torch.bfloat16, lower_bound=-5.0, tag="ragged")
    # zero-length sequences hand their initial state through unchanged
    for n in (0, 6):
        assert torch.equal(S[n].cpu(), inp["initial_state"][n])


def test_chunk_empty_sequence_batch():
    inp = KI.draw_chunk(2, 0, 2, 32, 32, dtype=torch.bfloat16, seed=8, init_state=True)
    o, S = run_chunk(inp)
    assert o.shape == (2, 0, 2, 32)
    assert torch.equal(S.cpu(), inp["initial_state"])


def test_chunk_final_state_in_place():
    inp = KI.draw_chunk(2, 97, 2, 128, 128, dtype=torch.bfloat16, seed=9, init_state=True)
    kda = kda_mod()
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    st = d["initial_state"].clone()
    o, S = kda.chunk_kda(d["q"], d["k"], d["v"], d["g"], d["beta"], initial_state=st,
                         output_final_state=True, final_state_out=st,
                         use_qk_l2norm_in_kernel=True)
    assert S.data_ptr() == st.data_ptr()
    compare_chunk(inp, o, S, torch.bfloat16, tag="inplace")


def test_chunk_without_final_state():
    inp = KI.draw_chunk(1, 70, 2, 32, 32, dtype=torch.bfloat16, seed=10, init_state=True)
    o, S = run_chunk(inp, final=False)
    assert S is None
    compare_chunk(inp, o, None, torch.bfloat16, tag="nofinal")


@pytest.mark.parametrize("split", [1, 2, 3, 63, 64, 65, 127])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_split_composition(split, dtype):
    """Two calls threaded through the state equal one call over T = 130."""
    inp = KI.draw_chunk(1, 130, 2, 128, 128, dtype=dtype, seed=11, init_state=True)
    o, S = run_chunk(inp)
    first = {k: (v[:, :split] if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
    second = {k: (v[:, split:] if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
    o1, S1 = run_chunk(first)
    second["initial_state"] = S1
    o2, S2 = run_chunk(second)
    check("split o", torch.cat([o1, o2], 1), o, dtype)
    check("split S", S2, S, dtype)
    compare_chunk(inp, torch.cat([o1, o2], 1), S2, dtype, tag=f"split{split}")


@pytest.mark.parametrize("t0,steps", [(1, 4), (7, 3), (63, 5), (64, 4), (65, 3)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_after_prefill(t0, steps, dtype):
    kda = kda_mod()
    T = t0 + steps
    inp = KI.draw_chunk(2, T, 3, 128, 128, dtype=dtype, seed=12 + t0, init_state=True)
    pre = {k: (v[:, :t0] if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
    o_pre, S = run_chunk(pre, lower_bound=-5.0)
    outs = [o_pre]
    for t in range(t0, T):
        x = {n: inp[n][:, t].to(DEV) for n in ("q", "k", "v", "g", "beta")}
        outs.append(kda.recurrent_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                                       lower_bound=-5.0)[:, None])
    compare_chunk(inp, torch.cat(outs, 1), S, dtype, lower_bound=-5.0, tag="prefill+decode")


@pytest.mark.parametrize("dims", DIMS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_shapes(dims, dtype):
    kda = kda_mod()
    Dk, Dv = dims
    inp = KI.draw_decode(5, 3, Dk, Dv, 6, dtype=dtype, seed=13)
    state = inp["state"].to(DEV)
    outs = []
    for t in range(6):
        outs.append(kda.recurrent_step(*(inp[n][t].to(DEV) for n in ("q", "k", "v", "g", "beta")),
                                       state, scale=0.25))
    o = torch.stack(outs)
    for n in range(5):
        o_ref, S_ref = oracle.recurrent(inp["q"][:, n], inp["k"][:, n], inp["v"][:, n],
                                        inp["g"][:, n], inp["beta"][:, n], scale=0.25,
                                        initial_state=inp["state"][n:n + 1])
        check(f"dec o n{n}", o[:, n], o_ref, dtype)
        check(f"dec S n{n}", state[n], S_ref[0], dtype)


def test_decode_noop_and_reset_tokens():
    """beta logit -inf with g = 0 leaves the state bit-identical; g = -inf with
    beta logit +inf replaces it by k^ v^T (oracle invariants, on the GPU)."""
    kda = kda_mod()
    N, H, D = 3, 2, 128
    S0 = torch.randn(N, H, D, D, device=DEV) * 0.1
    q = torch.randn(N, H, D, device=DEV)
    k = torch.randn(N, H, D, device=DEV)
    v = torch.randn(N, H, D, device=DEV)
    S = S0.clone()
    kda.recurrent_step(q, k, v, torch.zeros_like(q), torch.full((N, H), -math.inf, device=DEV), S)
    assert torch.equal(S, S0)
    kda.recurrent_step(q, k, v, torch.full_like(q, -math.inf), torch.full((N, H), math.inf,
                                                                          device=DEV), S)
    kh = k / torch.sqrt((k * k).sum(-1, keepdim=True) + 1e-6)
    torch.testing.assert_close(S, kh[..., :, None] * v[..., None, :], rtol=1e-5, atol=1e-6)


def test_decode_empty_batch():
    kda = kda_mod()
    z = torch.zeros(0, 2, 32, device=DEV)
    o = kda.recurrent_step(z, z, z, z, torch.zeros(0, 2, device=DEV), torch.zeros(0, 2, 32, 32, device=DEV))
    assert o.shape == (0, 2, 32)


def test_chunk_steep_gates_take_exact_path():
    """A chunk whose gate drops by more than the tensor-core split allows
    (here 9 per token over a whole chunk) is computed exactly for that chunk;
    its neighbours use the tensor-core split. Both must match the oracle."""
    inp = KI.draw_chunk(1, 200, 2, 128, 128, dtype=torch.bfloat16, seed=21, init_state=True)
    g = inp["g"].float()
    g[:, 64:128] = -9.0
    g[:, 150:160] = -9.5
    inp["g"] = g.to(torch.bfloat16)
    o, S = run_chunk(inp, lower_bound=-10.0)
    compare_chunk(inp, o, S, torch.bfloat16, lower_bound=-10.0, tag="steep")


def test_chunk_status_word_is_cleared():
    """The tensor-core path reports device-side timeouts in the first word of
    the workspace; a normal call leaves it zero."""
    inp = KI.draw_chunk(1, 130, 2, 128, 128, dtype=torch.bfloat16, seed=22)
    ws = torch.full((256,), 7, dtype=torch.uint8, device=DEV)
    run_chunk(inp, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0


# --- the single-pass tensor-core kernel ----------------------------------------
# kda_chunk_fwd runs the two-pass kernel when the workspace holds its per-chunk
# records and the single-pass kernel when only the 256-byte minimum is given;
# both must match the oracle on their own.

@pytest.mark.parametrize("lens", [(1,), (63,), (64,), (65,), (130,), (0, 1, 64, 65, 130, 7, 0, 200)])
def test_single_pass_kernel_lengths(lens):
    inp = KI.draw_chunk(1, sum(lens), 3, 128, 128, dtype=torch.bfloat16, seed=40 + sum(lens),
                        seqlens=lens, init_state=True)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    o, S = run_chunk(inp, lower_bound=-5.0, workspace=ws)
    compare_chunk(inp, o, S, torch.bfloat16, lower_bound=-5.0, tag=f"1pass {lens}")


def test_single_pass_kernel_steep_gates_and_gate_forms():
    inp = KI.draw_chunk(1, 200, 2, 128, 128, dtype=torch.bfloat16, seed=41, init_state=True)
    g = inp["g"].float()
    g[:, 64:128] = -9.0
    inp["g"] = g.to(torch.bfloat16)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    o, S = run_chunk(inp, lower_bound=-10.0, workspace=ws)
    compare_chunk(inp, o, S, torch.bfloat16, lower_bound=-10.0, tag="1pass steep")


def test_two_pass_and_single_pass_agree():
    """Both tensor-core kernels on one input: equal up to bf16 output rounding."""
    inp = KI.draw_chunk(1, 1000, 4, 128, 128, dtype=torch.bfloat16, seed=42,
                        seqlens=(300, 1, 699), init_state=True)
    o2, S2 = run_chunk(inp, lower_bound=-5.0)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    o1, S1 = run_chunk(inp, lower_bound=-5.0, workspace=ws)
    check("2pass vs 1pass o", o2, o1.double().cpu().numpy(), torch.bfloat16)
    check("2pass vs 1pass S", S2, S1.double().cpu().numpy(), torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_state_out_ping_pong(dtype):
    """The out-of-place step (two state buffers swapped each step, page "memra-engine
    tests/kda_fixture_gpu.rs", `state` / `state_alt`) leaves the old state intact and
    gives bit for bit the in-place result; both match the oracle."""
    kda = kda_mod()
    N, H, Dk, Dv, steps = 4, 3, 128, 64, 5
    inp = KI.draw_decode(N, H, Dk, Dv, steps, dtype=dtype, seed=21)
    S_in = inp["state"].to(DEV)
    S_a, S_b = S_in.clone(), torch.empty_like(S_in)
    o_in, o_pp = [], []
    for t in range(steps):
        args = [inp[n][t].to(DEV) for n in ("q", "k", "v", "g", "beta")]
        o_in.append(kda.recurrent_step(*args, S_in, lower_bound=-5.0))
        before = S_a.clone()
        o_pp.append(kda.recurrent_step(*args, S_a, lower_bound=-5.0, state_out=S_b))
        torch.cuda.synchronize()
        assert torch.equal(S_a, before), "the read-only state was written"
        S_a, S_b = S_b, S_a
    assert torch.equal(torch.stack(o_in), torch.stack(o_pp))
    assert torch.equal(S_in, S_a)
    o = torch.stack(o_pp)
    for n in range(N):
        o_ref, S_ref = oracle.recurrent(inp["q"][:, n], inp["k"][:, n], inp["v"][:, n], inp["g"][:, n],
                                        inp["beta"][:, n], lower_bound=-5.0, initial_state=inp["state"][n:n + 1])
        check(f"pp o n{n}", o[:, n], o_ref, dtype)
        check(f"pp S n{n}", S_a[n], S_ref[0], dtype)
