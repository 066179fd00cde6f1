"""The oracle's pins must be strong enough to catch plausible mistakes.

Each case plants one mistake (a dropped term, a wrong sign, a wrong index or
operand, an inclusive/exclusive slip) in a temporary copy of the oracle's C
source, compiles the copy on the CPU, swaps it in for the oracle's library
and runs the pins of test_oracle_pins.py against it: at least one pin must
fail. The committed oracle source is never modified.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

ORACLE_DIR = os.path.dirname(os.path.abspath(oracle.__file__))

MUTANTS = {
    # form R
    "R: no decay": ("kda_recurrent.c", "S[(size_t)c * Dv + j] *= a;", "S[(size_t)c * Dv + j] *= 1.0;"),
    "R: delta sign": ("kda_recurrent.c", "delta[j] = b * (vt[j] - kv);", "delta[j] = b * (vt[j] + kv);"),
    "R: beta not squashed": ("kda_recurrent.c", "if (J->beta_logit) b = rec_sigmoid(b);", ""),
    "R: beta always squashed": ("kda_recurrent.c", "if (J->beta_logit) b = rec_sigmoid(b);",
                                "b = rec_sigmoid(b);"),
    "C: beta always squashed": ("kda_chunkwise.c",
                                "B->b[r] = J->beta_logit ? 1.0 / (1.0 + exp(-J->beta[row])) : J->beta[row];",
                                "B->b[r] = 1.0 / (1.0 + exp(-J->beta[row]));"),
    "R: output reads k": ("kda_recurrent.c", "acc += S[(size_t)c * Dv + j] * qh[c];",
                          "acc += S[(size_t)c * Dv + j] * kh[c];"),
    "R: eps outside root": ("kda_recurrent.c", "double inv = 1.0 / sqrt(ss + 1e-6);",
                            "double inv = 1.0 / (sqrt(ss) + 1e-6);"),
    "R: bound flipped": ("kda_recurrent.c", "if (J->has_lb && gc < J->lb) gc = J->lb;",
                         "if (J->has_lb && gc > J->lb) gc = J->lb;"),
    "R: scale dropped": ("kda_recurrent.c", "ot[j] = J->scale * acc;", "ot[j] = acc;"),
    "R: write uses q": ("kda_recurrent.c", "S[(size_t)c * Dv + j] += kh[c] * delta[j];",
                        "S[(size_t)c * Dv + j] += qh[c] * delta[j];"),
    # form C
    "C: exclusive cumsum": ("kda_chunkwise.c",
                            "(r ? B->G[(size_t)(r - 1) * Dk + c] : 0.0) + gc;",
                            "(r ? B->G[(size_t)(r - 1) * Dk + c] + gc : 0.0);"),
    "C: Aqk drops diagonal": ("kda_chunkwise.c", "B->Aqk[(size_t)r * L + s] = (s <= r) ? aqk : 0.0;",
                              "B->Aqk[(size_t)r * L + s] = (s < r) ? aqk : 0.0;"),
    "C: inverse sign": ("kda_chunkwise.c", "B->T[(size_t)r * L + j] = -B->b[r] * acc;",
                        "B->T[(size_t)r * L + j] = B->b[r] * acc;"),
    "C: W ungated": ("kda_chunkwise.c",
                     "acc += B->T[(size_t)r * L + s] * B->b[s] * B->kh[(size_t)s * Dk + c] *\n"
                     "                       exp(B->G[(size_t)s * Dk + c]);",
                     "acc += B->T[(size_t)r * L + s] * B->b[s] * B->kh[(size_t)s * Dk + c];"),
    "C: state not decayed": ("kda_chunkwise.c", "double acc = exp(Gl[c]) * B->S[(size_t)c * Dv + j];",
                             "double acc = B->S[(size_t)c * Dv + j];"),
    "C: Delta sign": ("kda_chunkwise.c", "B->D[(size_t)r * Dv + j] = B->U[(size_t)r * Dv + j] - acc;",
                      "B->D[(size_t)r * Dv + j] = B->U[(size_t)r * Dv + j] + acc;"),
    "C: Khat reference": ("kda_chunkwise.c", "exp(Gl[c] - B->G[(size_t)s * Dk + c])",
                          "exp(B->G[(size_t)s * Dk + c])"),
    "C: Aqk gate sign": ("kda_chunkwise.c",
                         "double e = exp(B->G[(size_t)r * Dk + c] - B->G[(size_t)s * Dk + c]);",
                         "double e = exp(B->G[(size_t)s * Dk + c] - B->G[(size_t)r * Dk + c]);"),
}

# pins that exercise both forms, plus the form-R-only ones and the cross-check
PIN_CALLS = [
    lambda: pins.test_three_token_hand_example("recurrent", 1),
    lambda: pins.test_three_token_hand_example("chunkwise", 2),
    lambda: pins.test_three_token_hand_example("chunkwise", 64),
    lambda: pins.test_single_token_from_zero_state("recurrent"),
    lambda: pins.test_single_token_from_zero_state("chunkwise"),
    lambda: pins.test_basis_keys_are_gated_causal_linear_attention("recurrent"),
    lambda: pins.test_basis_keys_are_gated_causal_linear_attention("chunkwise"),
    lambda: pins.test_transition_matrix_form("recurrent"),
    lambda: pins.test_transition_matrix_form("chunkwise"),
    lambda: pins.test_pure_decay("chunkwise"),
    lambda: pins.test_lower_bound_clamps_gate(),
    lambda: pins.test_l2_norm_eps_inside_root(),
    lambda: pins.test_beta_zero_is_half_not_skip("recurrent"),
    lambda: pins.test_forms_agree(65, 16, (4, 3)),
    lambda: pins.test_forms_agree_varlen_and_steep_gates(),
    lambda: pins.test_beta_probability_matches_logit_form(),
    lambda: pins.test_beta_probability_special_values(),
]


def _build_mutant(tmp_path, fname, old, new):
    for f in ("kda_recurrent.c", "kda_chunkwise.c"):
        shutil.copy(os.path.join(ORACLE_DIR, f), tmp_path / f)
    src = (tmp_path / fname).read_text()
    assert src.count(old) == 1, f"mutation anchor not found exactly once in {fname}: {old!r}"
    (tmp_path / fname).write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so),
                    str(tmp_path / "kda_recurrent.c"), str(tmp_path / "kda_chunkwise.c"),
                    "-lm", "-lpthread"], check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_kill_mutant(name, tmp_path, monkeypatch):
    fname, old, new = MUTANTS[name]
    path = _build_mutant(tmp_path, fname, old, new)
    good = oracle._load()
    lib = ctypes.CDLL(path)
    for fn in ("kda_oracle_recurrent", "kda_oracle_chunkwise"):
        getattr(lib, fn).argtypes = getattr(good, fn).argtypes
        getattr(lib, fn).restype = ctypes.c_int
    monkeypatch.setattr(oracle, "_lib", lib)
    killed = []
    with np.errstate(all="ignore"):
        for i, call in enumerate(PIN_CALLS):
            try:
                call()
            except AssertionError:
                killed.append(i)
    assert killed, f"no pin caught the planted mistake '{name}'"


def test_unmutated_copy_passes_every_pin(tmp_path, monkeypatch):
    """Control: the same harness on an unmodified copy kills nothing."""
    for f in ("kda_recurrent.c", "kda_chunkwise.c"):
        shutil.copy(os.path.join(ORACLE_DIR, f), tmp_path / f)
    so = tmp_path / "libcopy.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so),
                    str(tmp_path / "kda_recurrent.c"), str(tmp_path / "kda_chunkwise.c"),
                    "-lm", "-lpthread"], check=True)
    good = oracle._load()
    lib = ctypes.CDLL(str(so))
    for fn in ("kda_oracle_recurrent", "kda_oracle_chunkwise"):
        getattr(lib, fn).argtypes = getattr(good, fn).argtypes
        getattr(lib, fn).restype = ctypes.c_int
    monkeypatch.setattr(oracle, "_lib", lib)
    for call in PIN_CALLS:
        call()


# Mistakes planted in the in-kernel gate (numpy side of the oracle): each must
# fail one of the gate pins.
def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _x(g, dt):
    return np.asarray(g, float) + (0.0 if dt is None else np.asarray(dt, float))


def _rate(a):
    return np.exp(np.asarray(a, float)).reshape(-1, 1)


GATE_MUTANTS = {
    "dt_bias dropped": lambda g, a, dt=None, lb=None: (
        -_rate(a) * oracle.softplus(np.asarray(g, float)) if lb is None
        else lb * _sig(_rate(a) * np.asarray(g, float))),
    "rate not exponentiated": lambda g, a, dt=None, lb=None: (
        -np.asarray(a, float).reshape(-1, 1) * oracle.softplus(_x(g, dt)) if lb is None
        else lb * _sig(np.asarray(a, float).reshape(-1, 1) * _x(g, dt))),
    "softplus sign": lambda g, a, dt=None, lb=None: (
        _rate(a) * oracle.softplus(_x(g, dt)) if lb is None else lb * _sig(_rate(a) * _x(g, dt))),
    "safe rate outside": lambda g, a, dt=None, lb=None: (
        -_rate(a) * oracle.softplus(_x(g, dt)) if lb is None else _rate(a) * lb * _sig(_x(g, dt))),
    "safe sigmoid of -x": lambda g, a, dt=None, lb=None: (
        -_rate(a) * oracle.softplus(_x(g, dt)) if lb is None else lb * _sig(-_rate(a) * _x(g, dt))),
    "softplus as relu": lambda g, a, dt=None, lb=None: (
        -_rate(a) * np.maximum(_x(g, dt), 0) if lb is None else lb * _sig(_rate(a) * _x(g, dt))),
}

GATE_PINS = [
    lambda: pins.test_gate_printed_example(),
    lambda: pins.test_gate_closed_forms(),
    lambda: pins.test_gate_dt_bias_is_per_head_channel(),
    lambda: pins.test_in_kernel_gate_forms_agree_and_safe_bound_holds(),
]


@pytest.mark.parametrize("name", sorted(GATE_MUTANTS))
def test_gate_pins_kill_mutant(name, monkeypatch):
    mut = GATE_MUTANTS[name]
    monkeypatch.setattr(oracle, "gate", lambda g, a, dt=None, lower_bound=None: mut(g, a, dt, lower_bound))
    killed = []
    with np.errstate(all="ignore"):
        for i, call in enumerate(GATE_PINS):
            try:
                call()
            except AssertionError:
                killed.append(i)
    assert killed, f"no gate pin caught the planted mistake '{name}'"
