"""Pins for the CPU oracle: each test checks it against something other than
itself -- a hand-worked example, a closed form, a textbook special case, an
invariant, or the second independently written form.

The recurrence being pinned is the one of page "atlas_core/kimi_k3/kda.rs"
(module doc, `kda_recurrent_step`); the boundary (initial/final state,
chunk size, q/k L2 norm, lower bound) is the `chunk_kda` of page
"K3/kda/ops/api.py". Shapes use d_k != d_v where they can, so that a
transposed state or a decay on the wrong axis cannot pass by symmetry.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FORMS = ("recurrent", "chunkwise")


def run(form, *args, chunk_size=None, **kw):
    if form == "recurrent":
        return oracle.recurrent(*args, **kw)
    return oracle.chunkwise(*args, chunk_size=chunk_size or 3, **kw)


def _num(x):
    if isinstance(x, str):
        return {"ln(1/2)": math.log(0.5), "ln(3)": math.log(3.0)}[x]
    return float(x)


def rand_inputs(rng, T, H, Dk, Dv, gmin=-2.0):
    q = rng.standard_normal((T, H, Dk))
    k = rng.standard_normal((T, H, Dk))
    v = rng.standard_normal((T, H, Dv))
    g = rng.uniform(gmin, 0.0, (T, H, Dk))
    b = rng.standard_normal((T, H))
    return q, k, v, g, b


# --- worked example -------------------------------------------------------

@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("chunk", [1, 2, 3, 64])
def test_three_token_hand_example(form, chunk):
    """Hand-derived three tokens (tests/golden/three_token_hand.json)."""
    fx = json.load(open(os.path.join(GOLDEN, "three_token_hand.json")))
    conv = lambda a: np.array([[_num(x) for x in row] for row in a])[:, None, :]
    q, k, v, g = (conv(fx[n]) for n in ("q", "k", "v", "g"))
    b = np.array([_num(x) for x in fx["beta_logit"]])[:, None]
    o, S = run(form, q, k, v, g, b, scale=1.0, use_qk_l2norm=False, chunk_size=chunk)
    np.testing.assert_allclose(o[:, 0], np.array(fx["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], np.array(fx["final_state"]), rtol=0, atol=1e-14)
    # with the in-kernel L2 norm the inputs are already unit vectors, so each
    # normalised q or k shrinks by (1 + 1e-6)^(-1/2) and nothing else changes.
    o2, S2 = run(form, q, k, v, g, b, scale=1.0, use_qk_l2norm=True, chunk_size=chunk)
    np.testing.assert_allclose(o2[:, 0], np.array(fx["o"]), rtol=0, atol=1e-5)
    np.testing.assert_allclose(S2[0, 0], np.array(fx["final_state"]), rtol=0, atol=1e-5)


# --- closed forms -----------------------------------------------------------

@pytest.mark.parametrize("form", FORMS)
def test_single_token_from_zero_state(form):
    """One token from S=0: S = sigmoid(b) k^ v^T and o = scale sigmoid(b) (q^.k^) v."""
    rng = np.random.default_rng(1)
    q, k, v, g, b = rand_inputs(rng, 1, 2, 5, 3)
    o, S = run(form, q, k, v, g, b, scale=0.7)
    for h in range(2):
        qh = q[0, h] / np.linalg.norm(q[0, h])
        kh = k[0, h] / np.linalg.norm(k[0, h])
        sb = 1.0 / (1.0 + math.exp(-b[0, h]))
        np.testing.assert_allclose(S[0, h], sb * np.outer(kh, v[0, h]), atol=1e-6)
        np.testing.assert_allclose(o[0, h], 0.7 * sb * (qh @ kh) * v[0, h], atol=1e-6)


@pytest.mark.parametrize("form", FORMS)
def test_basis_keys_are_gated_causal_linear_attention(form):
    """Keys that are distinct standard basis vectors never interfere, so every
    delta equals sigmoid(b_s) v_s and the output is gated causal linear
    attention: o_t = scale sum_{s<=t} sigmoid(b_s) exp(sum_{s<u<=t} g_u[c_s]) q_t[c_s] v_s,
    with c_s the channel of key s. This fixes the decay axis (key channels),
    which decays a write receives (those of later tokens, and of the current
    token before the read) and the sign of the delta."""
    rng = np.random.default_rng(2)
    T, Dk, Dv = 6, 7, 4
    perm = rng.permutation(Dk)[:T]
    k = np.zeros((T, 1, Dk))
    k[np.arange(T), 0, perm] = 1.0
    q = rng.standard_normal((T, 1, Dk))
    v = rng.standard_normal((T, 1, Dv))
    g = rng.uniform(-1.5, 0.0, (T, 1, Dk))
    b = rng.standard_normal((T, 1))
    o, S = run(form, q, k, v, g, b, scale=1.3, use_qk_l2norm=False, chunk_size=4)
    sig = 1.0 / (1.0 + np.exp(-b[:, 0]))
    want = np.zeros((T, Dv))
    for t in range(T):
        for s in range(t + 1):
            c = perm[s]
            decay = math.exp(g[s + 1:t + 1, 0, c].sum())
            want[t] += 1.3 * sig[s] * decay * q[t, 0, c] * v[s, 0]
    np.testing.assert_allclose(o[:, 0], want, atol=1e-12)
    S_want = np.zeros((Dk, Dv))
    for s in range(T):
        c = perm[s]
        S_want[c] += sig[s] * math.exp(g[s + 1:, 0, c].sum()) * v[s, 0]
    np.testing.assert_allclose(S[0, 0], S_want, atol=1e-12)


@pytest.mark.parametrize("form", FORMS)
def test_zero_gate_orthonormal_keys_is_linear_attention(form):
    """g = 0 and orthonormal keys (T <= d_k): the textbook causal linear
    attention o = scale * tril(Q K^T) diag(sigmoid(b)) V, computed with a
    library QR and matmul."""
    rng = np.random.default_rng(3)
    T, Dk, Dv = 5, 8, 3
    Qm, _ = np.linalg.qr(rng.standard_normal((Dk, Dk)))
    k = Qm[:, :T].T.copy()[:, None, :]
    q = rng.standard_normal((T, 1, Dk))
    v = rng.standard_normal((T, 1, Dv))
    g = np.zeros((T, 1, Dk))
    b = rng.standard_normal((T, 1))
    o, _ = run(form, q, k, v, g, b, scale=0.5, use_qk_l2norm=False, chunk_size=2)
    sig = 1.0 / (1.0 + np.exp(-b[:, 0]))
    want = 0.5 * np.tril(q[:, 0] @ k[:, 0].T) @ (sig[:, None] * v[:, 0])
    np.testing.assert_allclose(o[:, 0], want, atol=1e-12)


@pytest.mark.parametrize("form", FORMS)
def test_transition_matrix_form(form):
    """Delta rule written as a product of generalised Householder transitions
    S_t = (I - b_t k_t k_t^T) diag(exp g_t) S_{t-1} + b_t k_t v_t^T, evaluated
    with dense numpy matrices; o_t = scale S_t^T q_t."""
    rng = np.random.default_rng(4)
    T, Dk, Dv = 9, 4, 6
    q, k, v, g, b = rand_inputs(rng, T, 1, Dk, Dv)
    S0 = rng.standard_normal((1, 1, Dk, Dv))
    o, S = run(form, q, k, v, g, b, scale=0.9, initial_state=S0, use_qk_l2norm=False,
               chunk_size=4)
    sig = 1.0 / (1.0 + np.exp(-b[:, 0]))
    St = S0[0, 0].copy()
    for t in range(T):
        kt = k[t, 0]
        A = (np.eye(Dk) - sig[t] * np.outer(kt, kt)) @ np.diag(np.exp(g[t, 0]))
        St = A @ St + sig[t] * np.outer(kt, v[t, 0])
        np.testing.assert_allclose(o[t, 0], 0.9 * St.T @ q[t, 0], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-10, atol=1e-10)


# --- invariants -------------------------------------------------------------

def test_noop_token_keeps_state():
    """g = 0 and beta logit = -inf (sigmoid exactly 0): S is unchanged and
    o = scale S^T q^. Form R only (form C needs finite gates)."""
    rng = np.random.default_rng(5)
    q, k, v, _, _ = rand_inputs(rng, 3, 2, 4, 5)
    g = np.zeros((3, 2, 4))
    b = np.full((3, 2), -np.inf)
    S0 = rng.standard_normal((1, 2, 4, 5))
    o, S = oracle.recurrent(q, k, v, g, b, scale=0.3, initial_state=S0)
    np.testing.assert_array_equal(S, S0)
    for t in range(3):
        for h in range(2):
            qh = q[t, h] / math.sqrt((q[t, h] ** 2).sum() + 1e-6)
            np.testing.assert_allclose(o[t, h], 0.3 * S0[0, h].T @ qh, atol=1e-12)


def test_full_reset_token():
    """g = -inf (decay to 0) and beta logit = +inf (sigmoid 1): S = k^ v^T."""
    rng = np.random.default_rng(6)
    q, k, v, _, _ = rand_inputs(rng, 1, 1, 4, 3)
    g = np.full((1, 1, 4), -np.inf)
    b = np.full((1, 1), np.inf)
    S0 = rng.standard_normal((1, 1, 4, 3))
    o, S = oracle.recurrent(q, k, v, g, b, initial_state=S0, use_qk_l2norm=False)
    np.testing.assert_allclose(S[0, 0], np.outer(k[0, 0], v[0, 0]), atol=1e-14)


@pytest.mark.parametrize("form", FORMS)
def test_pure_decay(form):
    """beta logit = -inf on every token: no writes, S_T = diag(exp(sum g)) S0."""
    rng = np.random.default_rng(7)
    q, k, v, g, _ = rand_inputs(rng, 7, 1, 3, 4)
    b = np.full((7, 1), -1e30)  # sigmoid underflows to exactly 0; finite for form C
    S0 = rng.standard_normal((1, 1, 3, 4))
    o, S = run(form, q, k, v, g, b, initial_state=S0, scale=1.0, use_qk_l2norm=False)
    np.testing.assert_allclose(S[0, 0], np.exp(g[:, 0].sum(0))[:, None] * S0[0, 0], atol=1e-13)
    G = np.cumsum(g[:, 0], axis=0)
    for t in range(7):
        np.testing.assert_allclose(o[t, 0], (np.exp(G[t])[:, None] * S0[0, 0]).T @ q[t, 0],
                                   atol=1e-13)


@pytest.mark.parametrize("form", FORMS)
def test_linearity_in_values_and_state(form):
    rng = np.random.default_rng(8)
    q, k, v, g, b = rand_inputs(rng, 11, 2, 4, 3)
    S0 = rng.standard_normal((1, 2, 4, 3))
    o1, S1 = run(form, q, k, v, g, b, initial_state=S0)
    o2, S2 = run(form, q, k, -2.5 * v, g, b, initial_state=-2.5 * S0)
    np.testing.assert_allclose(o2, -2.5 * o1, atol=1e-12)
    np.testing.assert_allclose(S2, -2.5 * S1, atol=1e-12)


@pytest.mark.parametrize("form", FORMS)
def test_head_and_sequence_permutation(form):
    rng = np.random.default_rng(9)
    lens = [5, 0, 9, 3]
    T = sum(lens)
    q, k, v, g, b = rand_inputs(rng, T, 3, 4, 2)
    S0 = rng.standard_normal((4, 3, 4, 2))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, S = run(form, q, k, v, g, b, initial_state=S0, cu_seqlens=cu)
    hp = [2, 0, 1]
    oh, Sh = run(form, q[:, hp], k[:, hp], v[:, hp], g[:, hp], b[:, hp],
                 initial_state=S0[:, hp], cu_seqlens=cu)
    np.testing.assert_allclose(oh, o[:, hp], atol=1e-13)
    np.testing.assert_allclose(Sh, S[:, hp], atol=1e-13)
    # reversed sequence order: each sequence moves with its own tokens and state
    order = [3, 2, 1, 0]
    idx = np.concatenate([np.arange(cu[n], cu[n + 1]) for n in order]).astype(int)
    cu_r = np.concatenate([[0], np.cumsum([lens[n] for n in order])])
    orr, Sr = run(form, q[idx], k[idx], v[idx], g[idx], b[idx],
                  initial_state=S0[order], cu_seqlens=cu_r)
    np.testing.assert_allclose(orr, o[idx], atol=1e-13)
    np.testing.assert_allclose(Sr, S[order], atol=1e-13)
    # the zero-length sequence hands its initial state straight through
    np.testing.assert_array_equal(S[1], S0[1])


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("split", [1, 2, 3, 63, 64, 65, 127])
def test_split_composition(form, split):
    """The final state of x[:a], fed as the initial state of x[a:], reproduces
    the single-shot outputs and final state (splits of T = 130 that straddle
    chunk 64, as page 'memra-engine tests/kda_fixture_gpu.rs' gate 3 does)."""
    rng = np.random.default_rng(10)
    q, k, v, g, b = rand_inputs(rng, 130, 1, 4, 3)
    S0 = rng.standard_normal((1, 1, 4, 3))
    kw = dict(chunk_size=64) if form == "chunkwise" else {}
    fn = oracle.recurrent if form == "recurrent" else oracle.chunkwise
    o, S = fn(q, k, v, g, b, initial_state=S0, **kw)
    oa, Sa = fn(q[:split], k[:split], v[:split], g[:split], b[:split], initial_state=S0, **kw)
    ob, Sb = fn(q[split:], k[split:], v[split:], g[split:], b[split:], initial_state=Sa, **kw)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, atol=1e-12)
    np.testing.assert_allclose(Sb, S, atol=1e-12)


@pytest.mark.parametrize("t0,steps", [(1, 4), (7, 3), (63, 5), (64, 4), (65, 3)])
def test_decode_after_prefill(t0, steps):
    """Chunkwise prefill of t0 tokens, then single-token steps of form R,
    equals one full form-R pass (page 'memra-engine tests/kda_fixture_gpu.rs',
    gate 2 lengths)."""
    rng = np.random.default_rng(11)
    T = t0 + steps
    q, k, v, g, b = rand_inputs(rng, T, 2, 4, 3)
    o, S = oracle.recurrent(q, k, v, g, b, lower_bound=-1.0)
    op, Sp = oracle.chunkwise(q[:t0], k[:t0], v[:t0], g[:t0], b[:t0], lower_bound=-1.0,
                              chunk_size=64)
    outs = [op]
    for t in range(t0, T):
        ot, Sp = oracle.recurrent(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1],
                                  b[t:t + 1], initial_state=Sp, lower_bound=-1.0)
        outs.append(ot)
    np.testing.assert_allclose(np.concatenate(outs), o, atol=1e-12)
    np.testing.assert_allclose(Sp, S, atol=1e-12)


@pytest.mark.parametrize("form", FORMS)
def test_beta_zero_is_half_not_skip(form):
    """beta logit 0 means sigmoid 0.5: the state is written (page
    'atlas_core/kimi_k3/kda.rs', test beta_zero_is_sigmoid_half_not_zero), and
    the result differs from a saturated beta."""
    q = np.array([[[1.0, 0.0]]]); k = np.array([[[1.0, 0.0]]]); v = np.array([[[1.0, 0.5]]])
    g = np.full((1, 1, 2), -1.0)
    o0, S0 = run(form, q, k, v, g, np.array([[0.0]]))
    o1, S1 = run(form, q, k, v, g, np.array([[20.0]]))
    assert np.abs(o0).max() > 1e-6
    assert np.abs(o0 - o1).max() > 1e-3
    np.testing.assert_allclose(S0[0, 0], 0.5 * np.outer([1, 0], [1, 0.5]) / math.sqrt(1 + 1e-6),
                               atol=1e-12)


def test_lower_bound_clamps_gate():
    """lower_bound clamps g from below before the decay: a gate below the bound
    behaves exactly like the bound itself, a gate above it is untouched."""
    rng = np.random.default_rng(12)
    q, k, v, _, b = rand_inputs(rng, 6, 1, 3, 2)
    g = np.full((6, 1, 3), -9.0)
    g[::2] = -0.5
    o1, S1 = oracle.recurrent(q, k, v, g, b, lower_bound=-5.0)
    g2 = np.where(g < -5.0, -5.0, g)
    o2, S2 = oracle.recurrent(q, k, v, g2, b)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    o3, _ = oracle.recurrent(q, k, v, g, b)
    assert np.abs(o3 - o1).max() > 1e-6


def test_l2_norm_eps_inside_root():
    """q^ = q / sqrt(sum q^2 + 1e-6) (page 'atlas_core/kimi_k3/kda.rs',
    l2norm_rows): a zero key gives a zero write, and a tiny key is not
    blown up to unit length."""
    q = np.array([[[1.0, 0.0]]]); v = np.array([[[1.0, 1.0]]])
    g = np.zeros((1, 1, 2)); b = np.array([[50.0]])
    _, S = oracle.recurrent(q, np.zeros((1, 1, 2)), v, g, b)
    assert np.all(S == 0)
    _, S = oracle.recurrent(q, np.array([[[1e-4, 0.0]]]), v, g, b)
    want = 1e-4 / math.sqrt(1e-8 + 1e-6)
    np.testing.assert_allclose(S[0, 0, 0], [want, want], rtol=1e-12)


# --- the two forms against each other ---------------------------------------

@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 130])
@pytest.mark.parametrize("C", [1, 2, 3, 16, 64])
@pytest.mark.parametrize("d", [(2, 2), (4, 3), (32, 32)])
def test_forms_agree(T, C, d):
    rng = np.random.default_rng(100 + T * 7 + C)
    Dk, Dv = d
    H = 2
    q, k, v, g, b = rand_inputs(rng, T, H, Dk, Dv, gmin=-3.0)
    S0 = rng.standard_normal((1, H, Dk, Dv))
    for lb in (None, -1.0):
        o1, S1 = oracle.recurrent(q, k, v, g, b, initial_state=S0, lower_bound=lb)
        o2, S2 = oracle.chunkwise(q, k, v, g, b, initial_state=S0, lower_bound=lb, chunk_size=C)
        np.testing.assert_allclose(o2, o1, atol=1e-11, rtol=1e-11)
        np.testing.assert_allclose(S2, S1, atol=1e-11, rtol=1e-11)


def test_forms_agree_varlen_and_steep_gates():
    """Varlen packing with ragged lengths and gates down to -8 per step
    (spans of hundreds in a 64-token chunk): form C exponentiates only
    non-positive gate differences, so it stays finite and equal to form R."""
    rng = np.random.default_rng(13)
    lens = [64, 1, 130, 0, 77]
    T = sum(lens)
    q, k, v, g, b = rand_inputs(rng, T, 2, 5, 4, gmin=-8.0)
    S0 = rng.standard_normal((5, 2, 5, 4))
    cu = np.cumsum([0] + lens)
    o1, S1 = oracle.recurrent(q, k, v, g, b, initial_state=S0, cu_seqlens=cu)
    o2, S2 = oracle.chunkwise(q, k, v, g, b, initial_state=S0, cu_seqlens=cu, chunk_size=64)
    assert np.all(np.isfinite(o2)) and np.all(np.isfinite(S2))
    np.testing.assert_allclose(o2, o1, atol=1e-11, rtol=1e-11)
    np.testing.assert_allclose(S2, S1, atol=1e-11, rtol=1e-11)


def test_batched_layout_equals_packed():
    rng = np.random.default_rng(14)
    B, T, H, Dk, Dv = 3, 10, 2, 4, 3
    q = rng.standard_normal((B, T, H, Dk)); k = rng.standard_normal((B, T, H, Dk))
    v = rng.standard_normal((B, T, H, Dv)); g = rng.uniform(-1, 0, (B, T, H, Dk))
    b = rng.standard_normal((B, T, H))
    o, S = oracle.recurrent(q, k, v, g, b)
    for n in range(B):
        on, Sn = oracle.recurrent(q[n], k[n], v[n], g[n], b[n])
        np.testing.assert_allclose(o[n * T:(n + 1) * T], on, atol=1e-14)
        np.testing.assert_allclose(S[n], Sn[0], atol=1e-14)


# --- in-kernel gate -----------------------------------------------------------

def test_gate_printed_example():
    """tests/golden/gate_rs_test.json: the values kda.rs's own gate test fixes."""
    fx = json.load(open(os.path.join(GOLDEN, "gate_rs_test.json")))
    z = np.array([fx["z"]]); dt = np.array([fx["dt_bias"]]); a = np.array(fx["A_log"])
    g = oracle.gate(z, a, dt)[0]
    sp = lambda x: math.log1p(math.exp(x))  # plain softplus, fine at these arguments
    assert abs(g[0] - (-sp(0.6))) < 1e-6 and abs(g[1] - (-sp(-0.25))) < 1e-6
    g5 = oracle.gate(z, a, dt, lower_bound=fx["safe_lower_bound"])[0]
    assert abs(g5[0] - g[0]) > fx["safe_differs_from_unbounded_by_more_than"]


def test_gate_closed_forms():
    """Safe form: lb * sigmoid(0) = lb / 2 at x = 0, range (lb, 0), monotone in x;
    unbounded form: -rate * x for large x, -rate * e^x for very negative x, never positive."""
    a = np.log(np.array([0.5, 2.0]))            # rates 0.5 and 2
    x = np.zeros((2, 3))
    np.testing.assert_allclose(oracle.gate(x, a, lower_bound=-5.0), -2.5)
    xs = np.linspace(-10, 10, 41)[None, :].repeat(2, 0)
    gs = oracle.gate(xs, a, lower_bound=-5.0)
    assert np.all(gs < 0) and np.all(gs > -5.0) and np.all(np.diff(gs, axis=1) < 0)
    ends = oracle.gate(np.array([[-40.0], [40.0]]), np.zeros(2), lower_bound=-5.0)
    assert -1e-15 < ends[0, 0] <= 0.0 and -5.0 <= ends[1, 0] < -5.0 + 1e-15
    big = oracle.gate(np.full((2, 1), 50.0), a)
    np.testing.assert_allclose(big[:, 0], -np.exp(a) * 50.0, rtol=1e-12)
    tiny = oracle.gate(np.full((2, 1), -40.0), a)
    np.testing.assert_allclose(tiny[:, 0], -np.exp(a) * math.exp(-40.0), rtol=1e-9)
    assert np.all(oracle.gate(np.random.default_rng(0).normal(size=(2, 50)) * 10, a) <= 0)


def test_gate_dt_bias_is_per_head_channel():
    a = np.array([0.0, np.log(3.0)])
    dt = np.array([[0.2, -0.1], [0.0, 0.5]])
    x = np.zeros((4, 2, 2))
    g = oracle.gate(x, a, dt)
    np.testing.assert_allclose(g[1, 0], -oracle.softplus(dt[0]))
    np.testing.assert_allclose(g[3, 1], -3.0 * oracle.softplus(dt[1]))


def test_beta_probability_matches_logit_form():
    """beta given as a probability p (api.py, use_beta_sigmoid_in_kernel=False) is the
    same recurrence as the logit log(p / (1 - p)); forms R and C agree on it."""
    rng = np.random.default_rng(7)
    T, H, D = 37, 2, 4
    q, k, v = (rng.normal(size=(T, H, D)) for _ in range(3))
    g = -np.abs(rng.normal(size=(T, H, D))) * 0.3
    p = rng.uniform(0.05, 0.95, size=(T, H))
    o1, s1 = oracle.recurrent(q, k, v, g, p, beta_is_logit=False)
    o2, s2 = oracle.recurrent(q, k, v, g, np.log(p / (1 - p)))
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s1, s2, rtol=1e-12, atol=1e-13)
    o3, s3 = oracle.chunkwise(q, k, v, g, p, beta_is_logit=False, chunk_size=16)
    np.testing.assert_allclose(o3, o1, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(s3, s1, rtol=1e-10, atol=1e-11)


def test_beta_probability_special_values():
    """p = 0 writes nothing (the state only decays); p = 1 from a zero state with a unit
    key stores exactly k v^T (the write replaces the key's read-out by v)."""
    rng = np.random.default_rng(8)
    H, D = 1, 3
    q, k, v = (rng.normal(size=(1, H, D)) for _ in range(3))
    g = np.full((1, H, D), -0.5)
    S0 = rng.normal(size=(1, H, D, D))
    _, s = oracle.recurrent(q, k, v, g, np.zeros((1, H)), beta_is_logit=False, initial_state=S0)
    np.testing.assert_allclose(s, S0 * math.exp(-0.5), rtol=1e-14)
    kh = k / np.sqrt((k ** 2).sum(-1, keepdims=True) + 1e-6)
    _, s = oracle.recurrent(q, k, v, np.zeros((1, H, D)), np.ones((1, H)), beta_is_logit=False)
    np.testing.assert_allclose(s[0, 0], np.outer(kh[0, 0], v[0, 0]), rtol=1e-13)


def test_in_kernel_gate_forms_agree_and_safe_bound_holds():
    """With gate_form the g input is the gate's argument: forms R and C agree, and the
    safe form keeps every per-token decay above e^lb (state norm shrinks at most by it)."""
    rng = np.random.default_rng(9)
    T, H, D = 70, 3, 8
    q, k, v = (rng.normal(size=(T, H, D)) for _ in range(3))
    z = rng.normal(size=(T, H, D)) * 2
    beta = rng.normal(size=(T, H))
    A_log = rng.uniform(-1, 1, size=H)
    dt = rng.normal(size=(H, D)) * 0.5
    for form, lb in (("softplus", None), ("safe", -5.0)):
        oR, sR = oracle.recurrent(q, k, v, z, beta, gate_form=form, A_log=A_log, dt_bias=dt,
                                  lower_bound=lb)
        oC, sC = oracle.chunkwise(q, k, v, z, beta, gate_form=form, A_log=A_log, dt_bias=dt,
                                  lower_bound=lb, chunk_size=32)
        np.testing.assert_allclose(oC, oR, rtol=1e-9, atol=1e-10)
        np.testing.assert_allclose(sC, sR, rtol=1e-9, atol=1e-10)
    # a single token with zero beta: the state is the decayed initial state, decay = e^gate
    S0 = rng.normal(size=(1, H, D, D))
    _, s = oracle.recurrent(q[:1], k[:1], v[:1], z[:1], np.full((1, H), -np.inf),
                            gate_form="safe", A_log=A_log, dt_bias=dt, lower_bound=-5.0,
                            initial_state=S0)
    gg = -5.0 / (1 + np.exp(-np.exp(A_log)[:, None] * (z[0] + dt)))
    np.testing.assert_allclose(s[0], S0[0] * np.exp(gg)[:, :, None], rtol=1e-12)
    assert np.all(np.exp(gg) > math.exp(-5.0))


def test_gate_form_argument_rules():
    z = np.zeros((2, 1, 2))
    with pytest.raises(ValueError):
        oracle.recurrent(z, z, z, z, np.zeros((2, 1)), gate_form="softplus")   # no A_log
    with pytest.raises(ValueError):
        oracle.recurrent(z, z, z, z, np.zeros((2, 1)), gate_form="safe", A_log=[0.0])  # no lb
