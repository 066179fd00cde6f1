"""Pins of the decode-token oracle (conv update + SiLU, recurrent step, output gate).

Page "atlas_core/kimi_k3/kda.rs" defines the three pieces (`conv_update`,
`kda_decode_token`, `full_rank_output_gate`) and states two facts about them in
its tests: after four tokens the window of a width-4 convolution holds them
oldest to newest with the current sample in the last slot, and restoring the
state saved after the right token reproduces the sequential decode while the
state of an earlier token does not. Those facts, a hand-worked example
(tests/golden/decode_token_hand.json), closed forms and invariants pin the
oracle; planted mistakes check that the pins would catch an error.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GOLD = json.load(open(os.path.join(HERE, "golden", "decode_token_hand.json")))


# --- pins, each taking the functions under test so that mutants can be fed in --------

def pin_window_advances(conv_update):
    """kda.rs `conv_kernel_4_state_advances`: 6 channels, K = 4, all-ones weights,
    tokens 1, 2, 3, 4: the last slot is the current sample after every token and
    the window ends as 1, 2, 3, 4."""
    state = np.zeros((6, 4))
    w = np.ones((6, 4))
    for t in range(4):
        x = np.full(6, t + 1.0)
        _, state = conv_update(state, x, w)
        assert np.array_equal(state[:, -1], x)
    assert np.array_equal(state, np.tile([1.0, 2.0, 3.0, 4.0], (6, 1)))


def pin_conv_hand(conv_update):
    c = GOLD["conv"]
    y, st = conv_update(np.array([c["state"]]), np.array([c["x"]]), np.array([c["w"]]))
    assert np.array_equal(st[0], c["window"])
    assert abs(y[0] - c["y"]) < 1e-12


def pin_newest_tap_is_silu(conv_update):
    """Weight only on the newest tap: y = silu(x) whatever the history; silu(0) = 0,
    silu(x) - silu(-x) = x, silu(x) -> x for large x and -> 0 for very negative x."""
    rng = np.random.default_rng(3)
    state = rng.normal(size=(5, 4))
    w = np.zeros((5, 4))
    w[:, -1] = 1.0
    x = np.array([0.0, 1.5, -1.5, 40.0, -40.0])
    y, _ = conv_update(state, x, w)
    assert y[0] == 0.0
    assert abs((y[1] - y[2]) - 1.5) < 1e-14
    assert abs(y[3] - 40.0) < 1e-12 and abs(y[4]) < 1e-12


def pin_output_gate_hand(output_gate):
    g = GOLD["output_gate"]
    out = output_gate(np.array(g["core"]), np.array(g["g"]), 2, g["eps"])
    assert np.allclose(out, g["out"], rtol=0, atol=1e-15)


def pin_output_gate_invariants(output_gate):
    """With eps = 0: invariant to a positive scale of a head's core, odd in the core,
    sigmoid(+inf) = 1 leaves RMS(out) = 1, heads independent."""
    rng = np.random.default_rng(4)
    core = rng.normal(size=(3, 8))   # two heads of 4
    g = rng.normal(size=(3, 8))
    base = output_gate(core, g, 4, 0.0)
    scaled = core.copy()
    scaled[:, :4] *= 7.5
    assert np.allclose(output_gate(scaled, g, 4, 0.0), base, rtol=1e-13, atol=0)
    assert np.allclose(output_gate(-core, g, 4, 0.0), -base, rtol=0, atol=1e-15)
    full = output_gate(core, np.full_like(g, np.inf), 4, 0.0)
    assert np.allclose(np.sqrt(np.mean(full.reshape(3, 2, 4) ** 2, axis=-1)), 1.0, atol=1e-14)


def pin_prefix_hit(decode_token):
    """kda.rs `prefix_hit_wrong_slot_diverges`: heads 1, head_dim 2, conv kernel 4,
    lower bound -5, conv weights 0.25, gate = bounded_gate([0.1, -0.2], 0, A_log -1),
    beta logit 0.5, tokens x_t = (t + 1) * 0.1. Decoding token 3 from the state saved
    after token 2 equals the sequential decode; from the state after token 1 it moves."""
    H, D, K = 1, 2, 4
    C = 3 * H * D
    w = np.full((C, K), 0.25)
    g = oracle.gate(np.array([[0.1, -0.2]]), np.array([-1.0]), None, -5.0).reshape(1, H, D)
    beta = np.array([[0.5]])
    conv = np.zeros((1, C, K))
    rec = np.zeros((1, H, D, D))
    snaps = []
    for t in range(2):
        _, conv, rec = decode_token(np.full((1, C), (t + 1) * 0.1), w, conv, g, beta, rec, H=H, Dk=D, Dv=D)
        snaps.append((conv.copy(), rec.copy()))
    x3 = np.full((1, C), 0.4)
    y_seq, conv_seq, _ = decode_token(x3, w, conv, g, beta, rec, H=H, Dk=D, Dv=D)
    y_hit, conv_hit, _ = decode_token(x3, w, snaps[1][0], g, beta, snaps[1][1], H=H, Dk=D, Dv=D)
    assert np.array_equal(y_hit, y_seq) and np.array_equal(conv_hit, conv_seq)
    y_wrong, _, _ = decode_token(x3, w, snaps[0][0], g, beta, snaps[0][1], H=H, Dk=D, Dv=D)
    assert np.max(np.abs(y_wrong - y_hit)) > 1e-4


def pin_token_is_step_of_conv_output(decode_token):
    """The token is the recurrent step (form R, pinned on its own) applied to the
    conv output (conv_update, pinned above), q | k | v in that order, and hands back
    the advanced conv state; weights on every tap and a history in the window make
    a token that skips or misplaces the convolution differ."""
    rng = np.random.default_rng(5)
    N, H, Dk, Dv, K = 3, 2, 4, 3, 4
    C = H * (2 * Dk + Dv)
    x = rng.normal(size=(N, C))
    w = rng.normal(size=(C, K)) * 0.7
    conv = rng.normal(size=(N, C, K))
    g = -np.abs(rng.normal(size=(N, H, Dk)))
    beta = rng.normal(size=(N, H))
    S0 = rng.normal(size=(N, H, Dk, Dv)) * 0.1
    o, conv_new, S = decode_token(x, w, conv, g, beta, S0, H=H, Dk=Dk, Dv=Dv)
    y, conv_want = oracle.conv_update(conv, x, w)
    q = y[:, :H * Dk].reshape(N, H, Dk)
    k = y[:, H * Dk:2 * H * Dk].reshape(N, H, Dk)
    v = y[:, 2 * H * Dk:].reshape(N, H, Dv)
    o_r, S_r = oracle.recurrent(q, k, v, g, beta, initial_state=S0, cu_seqlens=np.arange(N + 1))
    assert np.array_equal(conv_new, conv_want)
    assert np.allclose(o, o_r, rtol=0, atol=1e-15) and np.allclose(S, S_r, rtol=0, atol=1e-15)


# --- the oracle against its pins -------------------------------------------------------

@pytest.mark.parametrize("pin", [pin_window_advances, pin_conv_hand, pin_newest_tap_is_silu])
def test_conv_update_pins(pin):
    pin(oracle.conv_update)


@pytest.mark.parametrize("pin", [pin_output_gate_hand, pin_output_gate_invariants])
def test_output_gate_pins(pin):
    pin(oracle.output_gate)


@pytest.mark.parametrize("pin", [pin_prefix_hit, pin_token_is_step_of_conv_output])
def test_decode_token_pins(pin):
    pin(oracle.decode_token)


def test_decode_token_output_gate_applied():
    """With g_out the token output is the output gate of the core output."""
    rng = np.random.default_rng(6)
    N, H, D, K = 2, 3, 4, 2
    C = 3 * H * D
    args = (rng.normal(size=(N, C)), rng.normal(size=(C, K)) * 0.5, rng.normal(size=(N, C, K)),
            -np.abs(rng.normal(size=(N, H, D))), rng.normal(size=(N, H)), rng.normal(size=(N, H, D, D)))
    g_out = rng.normal(size=(N, H * D))
    core, _, _ = oracle.decode_token(*args, H=H, Dk=D, Dv=D)
    gated, _, _ = oracle.decode_token(*args, H=H, Dk=D, Dv=D, g_out=g_out, norm_eps=1e-5)
    want = oracle.output_gate(core.reshape(N, H * D), g_out, D, 1e-5).reshape(N, H, D)
    assert np.array_equal(gated, want)


# --- planted mistakes: each must fail a pin --------------------------------------------

def _conv_shift_wrong_way(state, x, w):
    st = np.array(state, dtype=np.float64).copy()
    st[..., 1:] = st[..., :-1].copy()
    st[..., -1] = x
    return oracle.silu(np.sum(w * st, axis=-1)), st


def _conv_x_first_slot(state, x, w):
    st = np.array(state, dtype=np.float64).copy()
    st[..., :-1] = st[..., 1:]
    st[..., 0] = x
    return oracle.silu(np.sum(w * st, axis=-1)), st


def _conv_relu(state, x, w):
    st = np.array(state, dtype=np.float64).copy()
    st[..., :-1] = st[..., 1:]
    st[..., -1] = x
    return np.maximum(np.sum(w * st, axis=-1), 0.0), st


def _gate_sum_not_mean(core, g, head_dim, eps):
    c = np.asarray(core, dtype=np.float64).reshape(*np.shape(core)[:-1], -1, head_dim)
    gg = np.asarray(g, dtype=np.float64).reshape(c.shape)
    out = c / np.sqrt(np.sum(c * c, axis=-1, keepdims=True) + eps) / (1.0 + np.exp(-gg))
    return out.reshape(np.shape(core))


def _gate_sigmoid_minus(core, g, head_dim, eps):
    return oracle.output_gate(core, -np.asarray(g, dtype=np.float64), head_dim, eps)


def _token_no_conv(x, w, conv, g, beta, state, **kw):
    y = oracle.silu(np.asarray(x, dtype=np.float64))
    H, Dk, Dv = kw["H"], kw["Dk"], kw["Dv"]
    N = y.shape[0]
    q = y[:, :H * Dk].reshape(N, H, Dk)
    k = y[:, H * Dk:2 * H * Dk].reshape(N, H, Dk)
    v = y[:, 2 * H * Dk:].reshape(N, H, Dv)
    o, S = oracle.recurrent(q, k, v, np.reshape(g, (N, H, Dk)), np.reshape(beta, (N, H)),
                            initial_state=state, cu_seqlens=np.arange(N + 1))
    return o, np.array(conv, dtype=np.float64), S


CONV_PINS = [pin_window_advances, pin_conv_hand, pin_newest_tap_is_silu]
GATE_PINS = [pin_output_gate_hand, pin_output_gate_invariants]
TOKEN_PINS = [pin_prefix_hit, pin_token_is_step_of_conv_output]


def _fails(pins, impl):
    for pin in pins:
        try:
            pin(impl)
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("mutant", [_conv_shift_wrong_way, _conv_x_first_slot, _conv_relu])
def test_conv_mutants_are_caught(mutant):
    assert _fails(CONV_PINS, mutant)


@pytest.mark.parametrize("mutant", [_gate_sum_not_mean, _gate_sigmoid_minus])
def test_output_gate_mutants_are_caught(mutant):
    assert _fails(GATE_PINS, mutant)


def test_token_without_conv_is_caught():
    assert _fails(TOKEN_PINS, _token_no_conv)
