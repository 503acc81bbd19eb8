"""Pins of the oracle's reverse mode (``oracle.backward``).

The backward is checked against statements that do not reuse its code:
  * central finite differences of the forward oracle (itself pinned by
    test_oracle_pins.py) along random directions, for every input of every form;
  * the textbook gradients of causal linear attention (GLA with w = 1), written
    out as O(T^2) / O(T^3) sums, including the gradient of the log-decays;
and copies of the oracle with a planted mistake in the reverse code must fail at
least one of those pins.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.library_path()), "gdr_oracle.c")


def _inputs(form, rng, B=1, T=70, H=2, dk=4, dv=3, with_wg=True):
    """Random inputs; T = 70 crosses the backward's 64-token checkpoint segment, and
    d_k != d_v catches transposed state indices."""
    q = rng.standard_normal((B, T, H, dk))
    k = 0.5 * rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    log_w = -np.exp(rng.normal(-1.5, 0.5, (B, T, H, dk)))
    e1 = e2 = None
    if form == "general":
        e1 = 0.4 * rng.standard_normal((B, T, H, dk))
        e2 = 0.4 * rng.standard_normal((B, T, H, dk))
    elif form == "gdn2":
        e1 = rng.uniform(0.0, 1.0, (B, T, H, dk))
        e2 = rng.uniform(0.0, 1.0, (B, T, H, dv)) if with_wg else None
    elif form == "rwkv7":
        e1 = rng.standard_normal((B, T, H, dk))
        e1 /= np.linalg.norm(e1, axis=-1, keepdims=True)
        e2 = rng.uniform(0.0, 2.0, (B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv))
    return dict(q=q, k=k, v=v, log_w=log_w, e1=e1, e2=e2, S0=S0)


def pin_bwd_finite_differences(fwd, bwd, seed=0):
    """<grad, d> against (L(x + eps d) - L(x - eps d)) / (2 eps), L = <dO, o> + <dS_T, S_T>."""
    rng = np.random.default_rng(seed)
    worst = 0.0
    for form, with_wg in (("general", True), ("gdn2", True), ("gdn2", False), ("rwkv7", True),
                          ("gla", True)):
        x = _inputs(form, rng, with_wg=with_wg)
        B, T, H, dk = x["q"].shape
        dv = x["v"].shape[-1]
        dO = rng.standard_normal((B, T, H, dv))
        dST = rng.standard_normal((B, H, dk, dv))
        g = bwd(form, dO=dO, dS_T=dST, **x)

        def loss(y):
            o, S_T = fwd(form, **y)
            return float(np.sum(o * dO) + np.sum(S_T * dST))

        for name, val in x.items():
            if val is None:
                continue
            d = rng.standard_normal(val.shape)
            eps = 1e-6
            fd = (loss({**x, name: val + eps * d}) - loss({**x, name: val - eps * d})) / (2 * eps)
            an = float(np.sum(g[name] * d))
            rel = abs(fd - an) / max(abs(fd), 1e-12)
            assert rel < 1e-6, f"{form} d{name}: analytic {an!r} vs finite difference {fd!r}"
            worst = max(worst, rel)
    return worst


def pin_bwd_linear_attention(bwd, seed=1):
    """GLA with w = 1 and S0 = 0 is causal linear attention o_t = sum_{s<=t} v_s (k_s . q_t).
    Its gradients: dq_t = sum_{s<=t} k_s (v_s . do_t), dk_s = sum_{t>=s} q_t (v_s . do_t),
    dv_s = sum_{t>=s} do_t (k_s . q_t), dS0 = sum_t q_t do_t^T (key x value), and for the
    log-decay r (entering every pair s < r <= t): d log w_r = sum_{t>=r} sum_{s<r}
    (do_t . v_s) k_s (.) q_t."""
    rng = np.random.default_rng(seed)
    T, dk, dv = 12, 3, 4
    q, k = rng.standard_normal((T, dk)), rng.standard_normal((T, dk))
    v, do = rng.standard_normal((T, dv)), rng.standard_normal((T, dv))
    g = bwd("gla", q[None, :, None], k[None, :, None], v[None, :, None],
            np.zeros((1, T, 1, dk)), None, None, np.zeros((1, 1, dk, dv)), dO=do[None, :, None])
    dq = np.array([sum(k[s] * (v[s] @ do[t]) for s in range(t + 1)) for t in range(T)])
    dk_ = np.array([sum(q[t] * (v[s] @ do[t]) for t in range(s, T)) for s in range(T)])
    dv_ = np.array([sum(do[t] * (k[s] @ q[t]) for t in range(s, T)) for s in range(T)])
    dS0 = sum(np.outer(q[t], do[t]) for t in range(T))
    dlw = np.array([sum((do[t] @ v[s]) * k[s] * q[t] for t in range(r, T) for s in range(r))
                    if r > 0 else np.zeros(dk) for r in range(T)])
    worst = 0.0
    for name, ref in (("q", dq), ("k", dk_), ("v", dv_), ("log_w", dlw)):
        err = float(np.max(np.abs(g[name][0, :, 0] - ref)))
        assert err < 1e-12, f"linear-attention d{name} mismatch {err:.3e}"
        worst = max(worst, err)
    err = float(np.max(np.abs(g["S0"][0, 0] - dS0)))
    assert err < 1e-12, f"linear-attention dS0 mismatch {err:.3e}"
    return max(worst, err)


BWD_PINS = [pin_bwd_finite_differences, pin_bwd_linear_attention]


def _fwd(lib=None):
    def f(form, q, k, v, log_w, e1, e2, S0):
        return oracle.forward(form, q, k, v, log_w, e1, e2, S0, lib=lib)
    return f


def _bwd(lib=None):
    def f(form, q, k, v, log_w, e1, e2, S0, dO=None, dS_T=None):
        return oracle.backward(form, q, k, v, log_w, e1, e2, S0, dO, dS_T, lib=lib)
    return f


def _run_pin(pin, lib=None):
    if pin is pin_bwd_finite_differences:
        return pin(_fwd(lib), _bwd(lib))
    return pin(_bwd(lib))


@pytest.mark.parametrize("pin", BWD_PINS, ids=lambda f: f.__name__)
def test_backward_pin(pin):
    _run_pin(pin)


def test_backward_empty_sequence():
    z = np.zeros((1, 0, 2, 3))
    S0 = np.ones((1, 2, 3, 3))
    dST = np.arange(18, dtype=np.float64).reshape(1, 2, 3, 3)
    g = oracle.backward("gla", z, z, z, z, None, None, S0, np.zeros((1, 0, 2, 3)), dST)
    assert g["q"].shape == (1, 0, 2, 3) and np.array_equal(g["S0"], dST)


BWD_MUTANTS = {
    "adjoint_without_decay": ("dS[(size_t)c * dk + j] = dS[(size_t)c * dk + j] * w[j] + de[c] * u[j];",
                              "dS[(size_t)c * dk + j] = dS[(size_t)c * dk + j] + de[c] * u[j];"),
    "adjoint_without_erase": ("dS[(size_t)c * dk + j] = dS[(size_t)c * dk + j] * w[j] + de[c] * u[j];",
                              "dS[(size_t)c * dk + j] = dS[(size_t)c * dk + j] * w[j];"),
    "readout_from_old_state": ("acc += S_cur[(size_t)c * dk + j] * dO[tv + c];",
                               "acc += S_prev[(size_t)c * dk + j] * dO[tv + c];"),
    "erase_key_sign": ("zz -= g * e[c];", "zz += g * e[c];"),
    "gdn2_logw_direct_term": ("dlw += uu * u[j];", ""),
    "rwkv7_da_without_dz": ("de1[tk + j] = uu * e2[ts] + zz;", "de1[tk + j] = uu * e2[ts];"),
    "write_gate_grad_uses_gate": ("de2[tv + c] = dvv[c] * v[tv + c];", "de2[tv + c] = dvv[c] * e2[tv + c];"),
    "state_grad_transposed": ("dS0[so + j * (size_t)dv + c] = dS[(size_t)c * dk + j];",
                              "dS0[so + c * (size_t)dk + j] = dS[(size_t)c * dk + j];"),
}


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_mutant_is_caught(tmp_path, name):
    old, new = BWD_MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib_path = tmp_path / f"lib{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-o", str(lib_path),
                           str(path), "-lm"])
    lib = oracle.load_library(str(lib_path))
    caught = []
    for pin in BWD_PINS:
        try:
            _run_pin(pin, lib)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin detects backward mutant {name}"
