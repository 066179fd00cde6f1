"""Pins of the backward oracle (`oracle.backward`).

The pages give no backward formulas; the gradients are the derivatives of the
token recurrence of page "atlas_core/kimi_k3/kda.rs". The oracle takes them by
reverse-mode differentiation of an fp64 torch restatement of that recurrence. It
is pinned here against an independent route: central finite differences of the
C form R (`oracle.recurrent`, itself pinned in test_oracle_pins.py) for every
input element of small cases, plus a single-token closed form and invariants.
"""
import numpy as np
import pytest

import oracle


def loss_r(q, k, v, g, beta, S0, do, dSf, cu, **kw):
    o, S = oracle.recurrent(q, k, v, g, beta, initial_state=S0, cu_seqlens=cu, **kw)
    L = float(np.sum(o * do))
    if dSf is not None:
        L += float(np.sum(S * dSf))
    return L


def fd_grads(q, k, v, g, beta, S0, do, dSf, cu, h=1e-6, **kw):
    args = [q, k, v, g, beta, S0]
    out = []
    for i, a in enumerate(args):
        gr = np.zeros_like(a)
        it = np.nditer(a, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            ap, am = [x.copy() for x in args], [x.copy() for x in args]
            ap[i][idx] += h
            am[i][idx] -= h
            gr[idx] = (loss_r(*ap, do, dSf, cu, **kw) - loss_r(*am, do, dSf, cu, **kw)) / (2 * h)
        out.append(gr)
    return out


def draw(lens, H, Dk, Dv, seed, lb=None):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q, k = rng.normal(size=(T, H, Dk)), rng.normal(size=(T, H, Dk))
    v = rng.normal(size=(T, H, Dv))
    g = -np.abs(rng.normal(size=(T, H, Dk)))
    if lb is not None:  # keep every gate 0.05 away from the clamp's kink
        g = np.where(np.abs(g - lb) < 0.05, g + 0.1, g)
    beta = rng.normal(size=(T, H))
    S0 = rng.normal(size=(len(lens), H, Dk, Dv)) * 0.3
    do = rng.normal(size=(T, H, Dv))
    dSf = rng.normal(size=(len(lens), H, Dk, Dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, g, beta, S0, do, dSf, cu


CASES = [
    dict(lens=(1,), H=1, Dk=2, Dv=2),
    dict(lens=(4,), H=2, Dk=3, Dv=2),
    dict(lens=(3, 5), H=1, Dk=2, Dv=3),
    dict(lens=(6,), H=1, Dk=2, Dv=2, lb=-0.7),
    dict(lens=(5,), H=1, Dk=3, Dv=2, l2=False),
    dict(lens=(4,), H=1, Dk=2, Dv=2, prob=True, final=False),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_backward_matches_finite_differences(case):
    lb = case.get("lb")
    q, k, v, g, beta, S0, do, dSf, cu = draw(case["lens"], case["H"], case["Dk"], case["Dv"],
                                             seed=len(case["lens"]) * 7 + case["Dk"], lb=lb)
    kw = dict(use_qk_l2norm=case.get("l2", True), lower_bound=lb)
    if case.get("prob"):
        beta = 1.0 / (1.0 + np.exp(-beta))
        kw["beta_is_logit"] = False
    if not case.get("final", True):
        dSf = None
    if not case.get("l2", True):  # unnormalised keys: keep the rule contractive
        k = k * 0.4
    got = oracle.backward(q, k, v, g, beta, do, dS_final=dSf, initial_state=S0, cu_seqlens=cu, **kw)
    want = fd_grads(q, k, v, g, beta, S0, do, dSf, cu, **kw)
    for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), got, want):
        assert np.allclose(a, b, rtol=1e-6, atol=1e-7), (name, np.max(np.abs(a - b)))


def test_single_token_closed_form():
    """One token from a zero state without the L2 norm: o = scale b (q.k) v, so
    dv = scale b (q.k) do, dq = scale b (v.do) k, dk = scale b (v.do) q,
    dbeta (logit) = scale (q.k)(v.do) b (1 - b), and the decay has no effect: dg = 0."""
    rng = np.random.default_rng(11)
    q, k, v, do = (rng.normal(size=(1, 1, 3)) for _ in range(4))
    g = -np.abs(rng.normal(size=(1, 1, 3)))
    beta = np.array([[0.3]])
    scale = 0.5
    b = 1.0 / (1.0 + np.exp(-0.3))
    dq, dk, dv, dg, db, _ = oracle.backward(q, k, v, g, beta, do, scale=scale, use_qk_l2norm=False)
    qk, vd = float(np.sum(q * k)), float(np.sum(v * do))
    assert np.allclose(dv, scale * b * qk * do, atol=1e-14)
    assert np.allclose(dq, scale * b * vd * k, atol=1e-14)
    assert np.allclose(dk, scale * b * vd * q, atol=1e-14)
    assert np.allclose(db, scale * qk * vd * b * (1 - b), atol=1e-14)
    assert np.array_equal(dg, np.zeros_like(dg))


def test_dv_does_not_depend_on_v():
    """The outputs and the final state are affine in v (for fixed q, k, g, beta and
    initial state), so dv is the same for any v."""
    q, k, v, g, beta, S0, do, dSf, cu = draw((7,), 2, 3, 3, seed=12)
    a = oracle.backward(q, k, v, g, beta, do, dS_final=dSf, initial_state=S0, cu_seqlens=cu)[2]
    b = oracle.backward(q, k, 3.0 * v + 1.0, g, beta, do, dS_final=dSf, initial_state=S0, cu_seqlens=cu)[2]
    assert np.allclose(a, b, rtol=0, atol=1e-13)


def test_noop_token_has_no_key_or_value_gradient():
    """beta logit -inf writes nothing (sigmoid = 0): that token's k, v and beta get no
    gradient, and with g = 0 it does not decay either."""
    q, k, v, g, beta, S0, do, dSf, cu = draw((5,), 1, 2, 2, seed=13)
    beta[2] = -np.inf
    g[2] = 0.0
    dq, dk, dv, dg, db, _ = oracle.backward(q, k, v, g, beta, do, dS_final=dSf, initial_state=S0, cu_seqlens=cu)
    assert np.array_equal(dk[2], np.zeros_like(dk[2])) and np.array_equal(dv[2], np.zeros_like(dv[2]))
    assert db[2, 0] == 0.0
    assert np.any(dq[2] != 0.0)
