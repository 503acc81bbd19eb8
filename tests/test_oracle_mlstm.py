"""Pins of the oracle's mLSTM cell (``oracle.mlstm_forward``, "Exponential gates and matrix
memory: xLSTM and RWKV-7", section 13.4 and the solution to Exercise 13.6).

* the stabilized and the naive recurrence agree in the safe regime (the page prints 3.1e-15);
* the naive memory is gated linear attention with scalar decay sigmoid(f~) and written value
  exp(i~) v, and its normalizer the same recurrence on the value 1: both against the pinned
  matrix-memory oracle (GLA form);
* the recovery property printed on the page: one write of v = [0.3, -0.7, 1.1] on a unit key
  at input log-gate 800, read at q = k, returns v exactly, where the naive recurrence overflows;
* at log-gate 700 the naive memory is still finite and agrees; at 760 it is not, the
  stabilized one stays bounded.
Copies of the oracle with a planted mistake in the cell must fail one of the pins.
"""
import json
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.library_path()), "gdr_oracle.c")
GOLD = os.path.join(os.path.dirname(__file__), "golden", "mlstm_recovery_ch13_4.json")


def _draw(rng, B=2, T=40, H=2, dk=5, dv=3, i_mu=0.0, i_sd=1.5):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk)) / np.sqrt(dk)
    v = rng.standard_normal((B, T, H, dv))
    f = rng.normal(2.0, 1.5, (B, T, H))
    i = rng.normal(i_mu, i_sd, (B, T, H))
    return q, k, v, f, i


def pin_mlstm_stabilized_equals_naive(cell, seed=0):
    rng = np.random.default_rng(seed)
    q, k, v, f, i = _draw(rng)
    hs = cell(q, k, v, f, i)[0]
    hn = cell(q, k, v, f, i, naive=True)[0]
    err = float(np.max(np.abs(hs - hn)) / np.max(np.abs(hn)))
    assert err < 1e-12, f"stabilized vs naive {err:.3e}"
    return err


def pin_mlstm_naive_is_gated_linear_attention(cell, seed=1):
    """C_t q_t = GLA(q, k, exp(i~) v, log w = log sigmoid(f~)) and n_t^T q_t = the same with
    the value 1; h = C q / max(|n q|, 1)."""
    rng = np.random.default_rng(seed)
    q, k, v, f, i = _draw(rng, T=25)
    B, T, H, dk = q.shape
    logf = -np.logaddexp(0.0, -f)
    lw = np.repeat(logf[..., None], dk, axis=-1)
    num, _ = oracle.forward("gla", q, k, np.exp(i)[..., None] * v, lw)
    den, _ = oracle.forward("gla", q, k, np.exp(i)[..., None], lw)
    ref = num / np.maximum(np.abs(den), 1.0)
    hn = cell(q, k, v, f, i, naive=True)[0]
    err = float(np.max(np.abs(hn - ref)) / np.max(np.abs(ref)))
    assert err < 1e-12, f"naive mLSTM vs gated linear attention {err:.3e}"
    return err


def pin_mlstm_recovery(cell):
    with open(GOLD) as fh:
        gold = json.load(fh)
    v = np.array(gold["v"])
    key = np.array([0.6, 0.0, -0.8])         # unit key
    shp = lambda a: a.reshape(1, 1, 1, -1)
    h = cell(shp(key), shp(key), shp(v), np.zeros((1, 1, 1)),
             np.full((1, 1, 1), gold["input_log_gate"]))[0]
    err = float(np.max(np.abs(h.ravel() - v)))
    assert err < 1e-15, f"recovery at i~ = 800: {h.ravel()} vs {v}"
    return err


def pin_mlstm_overflow_regime(cell, seed=2):
    with open(GOLD) as fh:
        gold = json.load(fh)
    rng = np.random.default_rng(seed)
    q, k, v, f, i = _draw(rng, B=1, T=12, H=1, dk=4, dv=3)
    i_fin = i.copy()
    i_fin[0, 5, 0] = gold["naive_finite_log_gate"]
    hs, hn = cell(q, k, v, f, i_fin)[0], cell(q, k, v, f, i_fin, naive=True)[0]
    assert np.isfinite(hn).all()
    err = float(np.max(np.abs(hs - hn)) / np.max(np.abs(hn)))
    assert err < 1e-12, f"agreement at i~ = 700: {err:.3e}"
    i_ovf = i.copy()
    i_ovf[0, 5, 0] = gold["naive_overflow_log_gate"]
    hs, hn = cell(q, k, v, f, i_ovf)[0], cell(q, k, v, f, i_ovf, naive=True)[0]
    assert not np.isfinite(hn).all(), "the naive memory should overflow at i~ = 760"
    assert np.isfinite(hs).all() and np.max(np.abs(hs)) < 1e3
    return err


MLSTM_PINS = [pin_mlstm_stabilized_equals_naive, pin_mlstm_naive_is_gated_linear_attention,
              pin_mlstm_recovery, pin_mlstm_overflow_regime]


def _cell(lib=None):
    def f(*args, **kw):
        return oracle.mlstm_forward(*args, lib=lib, **kw)
    return f


@pytest.mark.parametrize("pin", MLSTM_PINS, ids=lambda f: f.__name__)
def test_mlstm_pin(pin):
    pin(_cell())


def test_mlstm_state_continues():
    """Running T tokens at once equals running the first half, then the second from the
    first's (C, n, m)."""
    rng = np.random.default_rng(5)
    q, k, v, f, i = _draw(rng, T=30)
    h, C, n, m = oracle.mlstm_forward(q, k, v, f, i)
    h1, C1, n1, m1 = oracle.mlstm_forward(q[:, :13], k[:, :13], v[:, :13], f[:, :13], i[:, :13])
    h2, C2, n2, m2 = oracle.mlstm_forward(q[:, 13:], k[:, 13:], v[:, 13:], f[:, 13:], i[:, 13:],
                                          C1, n1, m1)
    assert np.allclose(np.concatenate([h1, h2], 1), h, rtol=1e-13, atol=1e-13)
    assert np.allclose(C2, C, rtol=1e-13, atol=1e-13) and np.allclose(m2, m, rtol=0, atol=1e-13)


MLSTM_MUTANTS = {
    "floor_not_scaled": ("const double floor_ = naive ? 1.0 : exp(-m);", "const double floor_ = 1.0;"),
    "forget_without_previous_max": ("fs = exp(lf + m - mn);", "fs = exp(lf - mn);"),
    "max_without_forget_path": ("const double mn = fmax(lf + m, li);", "const double mn = li;"),
    "normalizer_sign_kept": ("fmax(fabs(den), floor_)", "fmax(den, floor_)"),
    "naive_input_gate_linear": ("is = exp(li);\n", "is = li;\n"),
    "log_sigmoid_sign": ("return x >= 0.0 ? -log1p(exp(-x)) : x - log1p(exp(x));",
                         "return x >= 0.0 ? log1p(exp(-x)) : x - log1p(exp(x));"),
    "write_transposed": ("is * v[tv + c] * k[tk + j];", "is * v[tv + c] * q[tk + j];"),
}


@pytest.mark.parametrize("name", sorted(MLSTM_MUTANTS))
def test_mlstm_mutant_is_caught(tmp_path, name):
    old, new = MLSTM_MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib_path = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-o", str(lib_path),
                           str(path), "-lm"])
    lib = oracle.load_library(str(lib_path))
    caught = []
    for pin in MLSTM_PINS:
        try:
            pin(_cell(lib))
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin detects mLSTM mutant {name}"
