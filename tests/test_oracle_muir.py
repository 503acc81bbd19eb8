"""Pins of the oracle's Muir token mixer (``oracle.muir_forward``): the gates, the
l2-normalised keys and queries, and the RMSNorm (.) SiLU(g) readout around the GDN-2
recurrence ("Muir: Linear Attention with Sensitivity-Allocated Gating and Matched-Filter
Readout", section 2.1 and section 4.1, eqs. (8)-(9)).

Each pin is a closed form of a special case, written from those definitions: a repeated
unit key with erase gate 1 and no decay erases the first write completely (delta rule with
step 1); no write and no erase leave Diag(alpha) S0 with alpha from the softplus / exp(a_log)
parameterisation; a two-entry initial state gives the readout in closed form; g = 0 silences
the output.  Copies of the oracle with a planted mistake in the mixer must fail one of them.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.library_path()), "gdr_oracle.c")
BIG = 40.0   # |logit| at which sigmoid is 0 or 1 to double precision (e^-40 ~ 4e-18)


def silu(x):
    return x / (1.0 + np.exp(-x))


def sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _unit_silu_key(rng, d):
    """A pre-activation whose SiLU, l2-normalised, is a known unit key."""
    x = rng.uniform(0.5, 2.0, d)
    s = silu(x)
    return x, s / np.linalg.norm(s)


def pin_muir_repeated_key_erases(muir, seed=0):
    """Two writes on the same unit key, erase gate b = 2 sigmoid(0) = 1, alpha = 1:
    S_2 = (I - k k^T) k (w1 v1)^T + k (w2 v2)^T = k (w2 v2)^T."""
    rng = np.random.default_rng(seed)
    dk, dv, H = 6, 5, 1
    kp, k = _unit_silu_key(rng, dk)
    vp = rng.standard_normal((2, dv))
    zw = rng.standard_normal((2, dv))
    tok = lambda a: a.reshape(1, 2, 1, -1)
    shape_k = (1, 2, 1, dk)
    y, S_T = muir(tok(np.stack([kp, kp])), tok(np.stack([kp, kp])), tok(vp),
                  np.full(shape_k, 0.3), np.zeros(shape_k), tok(zw), np.zeros(shape_k),
                  tok(rng.standard_normal((2, dv))), np.full(H, -60.0))
    w2v2 = sig(zw[1]) * silu(vp[1])
    err = float(np.max(np.abs(S_T[0, 0] - np.outer(k, w2v2))))
    assert err < 1e-12, f"repeated key not erased: {err:.3e}"
    return err


def pin_muir_decay_only(muir, seed=1):
    """No write (w = 0) and no erase (b = 0): S_1 = Diag(alpha) S0, log alpha =
    -exp(a_log) softplus(z_f)."""
    rng = np.random.default_rng(seed)
    dk, dv, H = 5, 4, 2
    S0 = rng.standard_normal((1, H, dk, dv))
    zf = rng.standard_normal((1, 1, H, dk)) * 2
    a_log = np.array([0.4, -1.3])
    z = lambda d, v=0.0: np.full((1, 1, H, d), v)
    _, S_T = muir(rng.standard_normal((1, 1, H, dk)), rng.standard_normal((1, 1, H, dk)),
                  rng.standard_normal((1, 1, H, dv)), zf, z(dk, -BIG), z(dv, -BIG), z(dk),
                  z(dv, 1.0), a_log, S0=S0)
    alpha = np.exp(-np.exp(a_log)[None, None, :, None] * np.log1p(np.exp(zf)))[0, 0]
    err = float(np.max(np.abs(S_T[0] - alpha[:, :, None] * S0[0])))
    assert err < 1e-13, f"decay parameterisation mismatch {err:.3e}"
    return err


def pin_muir_readout_closed_form(muir, seed=2):
    """alpha = 1, no write, no erase, S0 with two entries (j1, c1) = 1 and (j2, c2) = -2:
    o_{c1} = gamma_{j1} q_{j1}, o_{c2} = -2 gamma_{j2} q_{j2} (q = l2norm(silu(q_pre)),
    gamma = gamma_stat 2 sigmoid(z_q)), and y = rho (.) o / sqrt(mean(o^2) + eps) (.) silu(g)
    with eps = 1 so that every scale factor shows."""
    rng = np.random.default_rng(seed)
    dk, dv, H = 6, 5, 1
    j1, c1, j2, c2 = 1, 3, 4, 0
    S0 = np.zeros((1, H, dk, dv))
    S0[0, 0, j1, c1], S0[0, 0, j2, c2] = 1.0, -2.0
    qp = rng.standard_normal(dk)
    zq = rng.standard_normal(dk)
    gs = rng.uniform(0.5, 1.5, (H, dk))
    rho = rng.uniform(0.5, 2.0, dv)
    zg = rng.standard_normal(dv)
    z = lambda d, v=0.0: np.full((1, 1, H, d), v)
    y, _ = muir(qp.reshape(1, 1, 1, dk), rng.standard_normal((1, 1, H, dk)),
                rng.standard_normal((1, 1, H, dv)), z(dk), z(dk, -BIG), z(dv, -BIG),
                zq.reshape(1, 1, 1, dk), zg.reshape(1, 1, 1, dv), np.array([-60.0]),
                gamma_stat=gs, rho=rho, eps=1.0, S0=S0)
    q = silu(qp) / np.linalg.norm(silu(qp))
    gam = gs[0] * 2 * sig(zq)
    o = np.zeros(dv)
    o[c1], o[c2] = gam[j1] * q[j1], -2 * gam[j2] * q[j2]
    ref = rho * o / np.sqrt(np.mean(o ** 2) + 1.0) * silu(zg)
    err = float(np.max(np.abs(y[0, 0, 0] - ref)))
    assert err < 1e-13, f"readout closed form mismatch {err:.3e}"
    return err


def pin_muir_output_gate(muir, seed=3):
    """g = 0 gives y = silu(0) (...) = 0 for any state and inputs."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 7, 2, 4, 3
    r = lambda d: rng.standard_normal((B, T, H, d))
    y, _ = muir(r(dk), r(dk), r(dv), r(dk), r(dk), r(dv), r(dk), np.zeros((B, T, H, dv)),
                np.array([0.1, 0.2]), S0=rng.standard_normal((B, H, dk, dv)))
    assert np.all(y == 0.0)
    return 0.0


MUIR_PINS = [pin_muir_repeated_key_erases, pin_muir_decay_only, pin_muir_readout_closed_form,
             pin_muir_output_gate]


def _muir(lib=None):
    def f(*args, **kw):
        return oracle.muir_forward(*args, lib=lib, **kw)
    return f


@pytest.mark.parametrize("pin", MUIR_PINS, ids=lambda f: f.__name__)
def test_muir_pin(pin):
    pin(_muir())


MUIR_MUTANTS = {
    "key_not_normalised": ("      k[ok + j] /= nk2;\n", "\n"),
    "erase_gate_sigmoid": ("bg[ok + j] = 2.0 * sigm(zb[ok + j]);", "bg[ok + j] = sigm(zb[ok + j]);"),
    "decay_rate_not_exponentiated": ("const double rate = exp(a_log[h]);", "const double rate = a_log[h];"),
    "softplus_as_exp": ("lw[ok + j] = -rate * softplus(zf[ok + j]);", "lw[ok + j] = -rate * exp(zf[ok + j]);"),
    "value_without_silu": ("v[ov + c] = silu(v_pre[ov + c]);", "v[ov + c] = v_pre[ov + c];"),
    "gain_without_factor_two": ("* 2.0 * sigm(zq[ok + j]);", "* sigm(zq[ok + j]);"),
    "rms_sum_not_mean": ("sqrt(ms / dv + eps)", "sqrt(ms + eps)"),
    "output_gate_sigmoid": ("* inv * silu(zg[ov + c]);", "* inv * sigm(zg[ov + c]);"),
}


@pytest.mark.parametrize("name", sorted(MUIR_MUTANTS))
def test_muir_mutant_is_caught(tmp_path, name):
    old, new = MUIR_MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib_path = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-o", str(lib_path),
                           str(path), "-lm"])
    lib = oracle.load_library(str(lib_path))
    caught = []
    for pin in MUIR_PINS:
        try:
            pin(_muir(lib))
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin detects Muir mutant {name}"
