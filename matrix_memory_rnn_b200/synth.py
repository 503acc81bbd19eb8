"""Seeded synthetic inputs shaped like the pages' workloads.

This module draws random numbers and rounds them to the storage dtype; it holds
none of the recurrence's arithmetic.  Both the CUDA path (tests, bench) and the
fp64 oracle (tests) take their inputs from here, and from nowhere else.

Recipe (all draws with ``numpy.random.default_rng(seed)`` in float64, C order,
token-major [B, T, H, d]; draw order q, k, v, decay, then the form's erase
arguments, then the write gate):

* ``N(m, s)`` is a normal draw, ``sigmoid``/``SiLU``/``L2norm`` are applied in
  float64 to the draw (L2norm over the head's channel axis, no epsilon);
* values are then rounded to the storage dtype: bf16 with round-to-nearest-even
  (via fp32, also round-to-nearest-even), or fp32;
* the decay is passed as fp32 ``log w`` (<= 0), computed in float64 from the
  decay distribution and rounded once to fp32 (bf16 cannot hold decays near 1).

Returned arrays are float32 numpy arrays whose values are exactly the stored
values (bf16 values are exactly representable in fp32).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

__all__ = ["Workload", "PRESETS", "round_bf16", "round_f32", "forward_inputs",
           "decode_state", "decode_step_inputs", "muir_inputs", "mlstm_inputs"]


def round_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def round_bf16(x) -> np.ndarray:
    """float64 -> bf16 values (returned as float32), round to nearest even."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    bits = f.view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    out = ((bits + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return out.view(np.float32)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _silu(x):
    return x * _sigmoid(x)


def _l2norm(x):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


@dataclass(frozen=True)
class Workload:
    name: str
    form: str          # "gdn2" | "rwkv7" | "general" | "gla"
    dtype: str         # "bf16" | "f32"
    B: int
    H: int
    T: int             # tokens per sequence (1 for the decode workload)
    dk: int
    dv: int
    chunk: int
    seed: int
    # distribution parameters
    decay: str = "sigmoid_normal"   # see _log_decay
    decay_mu: float = 3.0
    decay_sigma: float = 1.0
    key: str = "l2_silu"            # "l2_silu" | "l2"
    s0_std: float = 0.0             # std of the initial state (0 = zero state)
    steps: int = 1                  # decode steps

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five workloads of the pages' hot path (sizes as given; chunk 64 where
# unstated, seeds 0..4).
PRESETS = {
    # RWKV-7 form, fp32: a unit, c = 2 sigmoid(N), w = exp(-exp(N(-1, 0.5))), S0 = 0
    "rwkv7_f32": Workload("rwkv7_f32", "rwkv7", "f32", B=1, H=2, T=256, dk=64, dv=64,
                          chunk=64, seed=0, decay="exp_normal", decay_mu=-1.0,
                          decay_sigma=0.5, key="l2"),
    # GDN-2 / Muir form, bf16: k = L2norm(SiLU(N)), alpha = sigmoid(N(3, 1)), b, w = sigmoid(N)
    "gdn2_bf16": Workload("gdn2_bf16", "gdn2", "bf16", B=4, H=16, T=4096, dk=128, dv=128,
                          chunk=64, seed=1),
    # RWKV-7 generalized delta rule, bf16, decay exp(-exp(N(-0.5, 0.5)))
    "rwkv7_bf16": Workload("rwkv7_bf16", "rwkv7", "bf16", B=8, H=32, T=2048, dk=64, dv=64,
                           chunk=64, seed=2, decay="exp_normal", decay_mu=-0.5,
                           decay_sigma=0.5, key="l2"),
    # long context: GDN-2, alpha ~ U[0.99, 0.9999] per channel, chunk 128
    "gdn2_long": Workload("gdn2_long", "gdn2", "bf16", B=1, H=16, T=65536, dk=128, dv=128,
                          chunk=128, seed=3, decay="uniform", decay_mu=0.99,
                          decay_sigma=0.9999),
    # decode: B=256, H=32, state ~ N(0, 0.1), GDN-2 inputs as gdn2_bf16, 1000 steps
    "decode": Workload("decode", "gdn2", "bf16", B=256, H=32, T=1, dk=128, dv=128,
                       chunk=64, seed=4, s0_std=0.1, steps=1000),
}


def _round(x, dtype):
    return round_bf16(x) if dtype == "bf16" else round_f32(x)


def _log_decay(rng, shape, w: Workload):
    if w.decay == "sigmoid_normal":        # alpha = sigmoid(N(mu, sigma)): log alpha = -log(1+e^-x)
        x = rng.normal(w.decay_mu, w.decay_sigma, size=shape)
        return -np.logaddexp(0.0, -x)
    if w.decay == "exp_normal":            # w = exp(-exp(N(mu, sigma)))
        return -np.exp(rng.normal(w.decay_mu, w.decay_sigma, size=shape))
    if w.decay == "uniform":               # alpha ~ U[lo, hi]
        return np.log(rng.uniform(w.decay_mu, w.decay_sigma, size=shape))
    raise ValueError(w.decay)


def _draw(rng, w: Workload, lead: tuple):
    """Draws one batch of token inputs with leading shape ``lead`` (+ channel axis)."""
    sk = lead + (w.dk,)
    sv = lead + (w.dv,)
    q = rng.standard_normal(sk)
    kraw = rng.standard_normal(sk)
    k = _l2norm(_silu(kraw)) if w.key == "l2_silu" else _l2norm(kraw)
    v = rng.standard_normal(sv)
    log_w = _log_decay(rng, sk, w)
    e1 = e2 = None
    if w.form == "gdn2":
        e1 = _sigmoid(rng.standard_normal(sk))            # erase gate b
        e2 = _sigmoid(rng.standard_normal(sv))            # write gate
    elif w.form == "rwkv7":
        e1 = _l2norm(rng.standard_normal(sk))             # unit removal direction a
        e2 = 2.0 * _sigmoid(rng.standard_normal(lead))    # removal coefficient c in (0, 2)
    elif w.form == "general":
        e1 = 0.5 * _l2norm(rng.standard_normal(sk))       # erase vector u
        e2 = _l2norm(rng.standard_normal(sk))             # erase key z
    out = {
        "q": _round(q, w.dtype), "k": _round(k, w.dtype), "v": _round(v, w.dtype),
        "log_w": round_f32(log_w),
        "e1": None if e1 is None else _round(e1, w.dtype),
        "e2": None if e2 is None else _round(e2, w.dtype),
    }
    return out


def forward_inputs(w: Workload, seed: int | None = None) -> dict:
    """Inputs of one chunked-forward call: q, k, v, log_w, e1, e2 ([B, T, H, .]) and S0."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    d = _draw(rng, w, (w.B, w.T, w.H))
    if w.s0_std > 0:
        d["S0"] = round_f32(rng.normal(0.0, w.s0_std, size=(w.B, w.H, w.dk, w.dv)))
    else:
        d["S0"] = None
    return d


def decode_state(w: Workload, seed: int | None = None) -> np.ndarray:
    """Initial decode state [B, H, dk, dv] fp32, N(0, s0_std)."""
    rng = np.random.default_rng((w.seed if seed is None else seed, 1 << 20))
    return round_f32(rng.normal(0.0, w.s0_std, size=(w.B, w.H, w.dk, w.dv)))


def decode_step_inputs(w: Workload, step: int, seed: int | None = None) -> dict:
    """Inputs of decode step ``step``: q, k, v, log_w, e1, e2 shaped [B, H, .]."""
    rng = np.random.default_rng((w.seed if seed is None else seed, step))
    return _draw(rng, w, (w.B, w.H))


def muir_inputs(w: Workload, seed: int | None = None, static_gains: bool = True) -> dict:
    """Inputs of one Muir-mixer call (shapes of ``w``; form ignored): the activations
    after the projections and the causal convolution q, k, v ~ N(0, 1), and the gate logits
    z_f ~ N(-4, 1) (softplus ~ 0.02: decays 0.75-0.98 per token with the rates below),
    z_b, z_w, z_q, z_g ~ N(0, 1), all at the storage dtype; a_log ~ U[log 1, log 16] per head,
    gamma_stat ~ U[0.5, 1.5] per (head, key channel) and the RMSNorm weight ~ U[0.5, 1.5]
    per value channel (fp32; ones when ``static_gains`` is False, their initial values)."""
    rng = np.random.default_rng(w.seed + 10 if seed is None else seed)
    sk = (w.B, w.T, w.H, w.dk)
    sv = (w.B, w.T, w.H, w.dv)
    r = lambda shape, m=0.0: _round(rng.normal(m, 1.0, size=shape), w.dtype)
    out = {"q": r(sk), "k": r(sk), "v": r(sv), "zf": r(sk, -4.0), "zb": r(sk), "zw": r(sv),
           "zq": r(sk), "zg": r(sv),
           "a_log": round_f32(rng.uniform(0.0, np.log(16.0), size=w.H))}
    if static_gains:
        out["gamma_stat"] = round_f32(rng.uniform(0.5, 1.5, size=(w.H, w.dk)))
        out["rms_weight"] = round_f32(rng.uniform(0.5, 1.5, size=w.dv))
    else:
        out["gamma_stat"] = out["rms_weight"] = None
    return out


def mlstm_inputs(w: Workload, seed: int | None = None, i_mu: float = 0.0, i_sd: float = 1.0) -> dict:
    """Inputs of one mLSTM call (shapes of ``w``): q, k ~ N(0, 1/d_k) per entry (the scaled
    keys of the cell), v ~ N(0, 1) at the storage dtype, and fp32 gate pre-activations
    f~ ~ N(3, 1) (forget gates near sigmoid(3) = 0.95) and i~ ~ N(i_mu, i_sd)."""
    rng = np.random.default_rng(w.seed + 20 if seed is None else seed)
    sk = (w.B, w.T, w.H, w.dk)
    sv = (w.B, w.T, w.H, w.dv)
    s = 1.0 / np.sqrt(w.dk)
    return {"q": _round(rng.normal(0.0, s, sk), w.dtype), "k": _round(rng.normal(0.0, s, sk), w.dtype),
            "v": _round(rng.standard_normal(sv), w.dtype),
            "f_pre": round_f32(rng.normal(3.0, 1.0, (w.B, w.T, w.H))),
            "i_pre": round_f32(rng.normal(i_mu, i_sd, (w.B, w.T, w.H)))}
