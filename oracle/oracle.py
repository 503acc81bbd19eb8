"""ctypes front end of the fp64 oracle in ``gdr_oracle.c``.

TEST INFRASTRUCTURE (see the package docstring).  Everything here is argument
marshalling: the recurrence itself is the C loop in ``gdr_oracle.c``, which
follows "Exponential gates and matrix memory: xLSTM and RWKV-7", section 13.3,
and "Muir: Linear Attention with Sensitivity-Allocated Gating and
Matched-Filter Readout", section 2.1 eq. (1) / section 4.2 eq. (8).

Inputs are float64 numpy arrays holding the values the GPU receives (bf16 or
fp32 values widened exactly to float64); ``log_w`` likewise (fp32 widened).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

FORMS = {"general": 0, "gdn2": 1, "rwkv7": 2, "gla": 3}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compiles ``gdr_oracle.c`` with gcc and OpenMP into ``liboracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Opens a compiled oracle (the real one, or a test's planted-mistake copy)."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_forward.restype = ctypes.c_int
    lib.oracle_forward.argtypes = [ctypes.c_int] * 6 + [dp] * 9 + [ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_muir_forward.restype = ctypes.c_int
    lib.oracle_muir_forward.argtypes = ([ctypes.c_int] * 5 + [dp] * 11 + [ctypes.c_double] +
                                        [dp] * 3 + [ctypes.c_int])
    lib.oracle_mlstm_forward.restype = ctypes.c_int
    lib.oracle_mlstm_forward.argtypes = [ctypes.c_int] * 6 + [dp] * 12 + [ctypes.c_int]
    lib.oracle_backward.restype = ctypes.c_int
    lib.oracle_backward.argtypes = [ctypes.c_int] * 6 + [dp] * 16 + [ctypes.c_int]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load_library(_LIB)
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def forward(form: str, q, k, v, log_w, e1=None, e2=None, S0=None, n_threads: int = 0,
            lib=None):
    """Token-by-token recurrence over [B, T, H, d] inputs.

    Returns ``(o, S_T)``: o is [B, T, H, dv]; S_T is [B, H, dk, dv] (key channel
    first, the library's storage layout).  ``lib`` selects another compiled copy
    (tests only); default is the oracle built from ``gdr_oracle.c``.
    """
    lib = _load() if lib is None else lib
    q, k, v, log_w, e1, e2, S0 = map(_f64, (q, k, v, log_w, e1, e2, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, H, dk) and log_w.shape == (B, T, H, dk)
    assert v.shape == (B, T, H, dv)
    if S0 is not None:
        assert S0.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    S_T = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = lib.oracle_forward(FORMS[form], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                            _ptr(log_w), _ptr(e1), _ptr(e2), _ptr(S0), _ptr(o), _ptr(S_T),
                            int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_forward failed with code {rc}")
    return o, S_T


def backward(form: str, q, k, v, log_w, e1=None, e2=None, S0=None, dO=None, dS_T=None,
             n_threads: int = 0, lib=None):
    """Gradients of L = <dO, o> + <dS_T, S_T> through the token-by-token recurrence.

    Same inputs as ``forward`` plus ``dO`` [B, T, H, dv] and ``dS_T`` [B, H, dk, dv]
    (None = 0).  Returns a dict with ``q, k, v, log_w`` (shaped like the inputs),
    ``e1`` / ``e2`` (None where the form has no such input) and ``S0`` [B, H, dk, dv].
    """
    lib = _load() if lib is None else lib
    q, k, v, log_w, e1, e2, S0, dO, dS_T = map(_f64, (q, k, v, log_w, e1, e2, S0, dO, dS_T))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, H, dk) and log_w.shape == (B, T, H, dk)
    assert v.shape == (B, T, H, dv) and dO is not None and dO.shape == (B, T, H, dv)
    if dS_T is not None:
        assert dS_T.shape == (B, H, dk, dv)
    g = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("log_w", log_w))}
    g["e1"] = None if e1 is None else np.zeros_like(e1)
    g["e2"] = None if e2 is None else np.zeros_like(e2)
    g["S0"] = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = lib.oracle_backward(FORMS[form], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                             _ptr(log_w), _ptr(e1), _ptr(e2), _ptr(S0), _ptr(dO), _ptr(dS_T),
                             _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["log_w"]),
                             _ptr(g["e1"]), _ptr(g["e2"]), _ptr(g["S0"]), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_backward failed with code {rc}")
    return g


def muir_forward(q_pre, k_pre, v_pre, zf, zb, zw, zq, zg, a_log, gamma_stat=None, rho=None,
                 eps=1e-6, S0=None, n_threads: int = 0, lib=None):
    """The Muir token mixer around the GDN-2 recurrence (``oracle_muir_forward``):
    pre-activations and gate logits [B, T, H, .], a_log [H], gamma_stat [H, dk] or None,
    rho [dv] or None.  Returns ``(y [B, T, H, dv], S_T [B, H, dk, dv])``."""
    lib = _load() if lib is None else lib
    arrs = map(_f64, (q_pre, k_pre, v_pre, zf, zb, zw, zq, zg, a_log, gamma_stat, rho, S0))
    q_pre, k_pre, v_pre, zf, zb, zw, zq, zg, a_log, gamma_stat, rho, S0 = arrs
    B, T, H, dk = q_pre.shape
    dv = v_pre.shape[-1]
    for a, d in ((k_pre, dk), (zf, dk), (zb, dk), (zq, dk), (v_pre, dv), (zw, dv), (zg, dv)):
        assert a.shape == (B, T, H, d)
    assert a_log.shape == (H,)
    y = np.zeros((B, T, H, dv), dtype=np.float64)
    S_T = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = lib.oracle_muir_forward(B, T, H, dk, dv, _ptr(q_pre), _ptr(k_pre), _ptr(v_pre), _ptr(zf),
                                 _ptr(zb), _ptr(zw), _ptr(zq), _ptr(zg), _ptr(a_log),
                                 _ptr(gamma_stat), _ptr(rho), float(eps), _ptr(S0), _ptr(y),
                                 _ptr(S_T), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_muir_forward failed with code {rc}")
    return y, S_T


def mlstm_forward(q, k, v, f_pre, i_pre, C0=None, n0=None, m0=None, naive=False,
                  n_threads: int = 0, lib=None):
    """xLSTM's mLSTM cell (``oracle_mlstm_forward``), stabilized unless ``naive``:
    q, k [B, T, H, dk], v [B, T, H, dv], f_pre, i_pre [B, T, H]; optional initial
    C0 [B, H, dk, dv], n0 [B, H, dk], m0 [B, H].  Returns (h, C_T, n_T, m_T)."""
    lib = _load() if lib is None else lib
    q, k, v, f_pre, i_pre, C0, n0, m0 = map(_f64, (q, k, v, f_pre, i_pre, C0, n0, m0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, H, dk) and v.shape == (B, T, H, dv)
    assert f_pre.shape == (B, T, H) and i_pre.shape == (B, T, H)
    h = np.zeros((B, T, H, dv))
    C_T = np.zeros((B, H, dk, dv))
    n_T = np.zeros((B, H, dk))
    m_T = np.zeros((B, H))
    rc = lib.oracle_mlstm_forward(B, T, H, dk, dv, int(bool(naive)), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(f_pre), _ptr(i_pre), _ptr(C0), _ptr(n0), _ptr(m0), _ptr(h),
                                  _ptr(C_T), _ptr(n_T), _ptr(m_T), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_mlstm_forward failed with code {rc}")
    return h, C_T, n_T, m_T


def decode_step(form: str, q, k, v, log_w, e1, e2, S, n_threads: int = 0):
    """One token per (b, h): inputs [B, H, d], state [B, H, dk, dv].  Returns (o, S_new)."""
    def tok(a):
        return None if a is None else _f64(a)[:, None]
    o, S_new = forward(form, tok(q), tok(k), tok(v), tok(log_w), tok(e1), tok(e2), S,
                       n_threads=n_threads)
    return o[:, 0], S_new
