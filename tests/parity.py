"""Shared helpers of the GPU parity tests: run libgdr and the oracle on the same
seeded inputs and measure the per-head relative error.

Error norms, per (b, h) head, max over heads, with X the head's T x dv output block (and
separately its final d_k x d_v state, or a gradient's block):
  - relative Frobenius error ||X_gpu - X_ref||_F / max(||X_ref||_F, 1e-30), the bar of record;
  - elementwise error max |X_gpu - X_ref| / max(RMS(X_ref), 1e-30).  The Frobenius norm of a
    T = 4096 head dilutes one wrong token (its 128 outputs) by 1/sqrt(4096) = 1.6 %, under the
    2e-2 bar; the elementwise norm does not dilute it, so the full-size tests assert both.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth

# Bars: fp32 inputs 1e-4, bf16 inputs 2e-2 (fp32 state and accumulation).  The fp32
# kernel is held to 1e-4 on either input dtype (it computes every product in fp32).
TOL = {"f32": 1e-4, "bf16": 2e-2}
TOL_FP32_KERNEL = 1e-4
# Elementwise bars: five times the Frobenius bar.  Rounding errors of a correct kernel are
# spread over the block, so their largest element sits a few standard deviations above
# the Frobenius average; a wrong or missing token sits near 1 or above.
ELEM_FACTOR = 5.0
ELEM_TOL = {k: ELEM_FACTOR * v for k, v in TOL.items()}


def head_rel_err(x, ref, head_axes):
    """Max over heads of the Frobenius relative error; `head_axes` index the head in x."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    other = tuple(i for i in range(x.ndim) if i not in head_axes)
    num = np.sqrt(np.sum((x - ref) ** 2, axis=other))
    den = np.maximum(np.sqrt(np.sum(ref ** 2, axis=other)), 1e-30)
    return float(np.max(num / den)) if num.size else 0.0


def head_max_err(x, ref, head_axes):
    """Max over heads of max |x - ref| / RMS(ref) within the head; `head_axes` as above."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    other = tuple(i for i in range(x.ndim) if i not in head_axes)
    num = np.max(np.abs(x - ref), axis=other) if x.size else np.zeros(0)
    den = np.maximum(np.sqrt(np.mean(ref ** 2, axis=other)), 1e-30) if x.size else np.ones(0)
    return float(np.max(num / den)) if num.size else 0.0


def check_parity(x, ref, head_axes, tol, label="", elem_tol=None):
    """Asserts both bars (Frobenius `tol`, elementwise `elem_tol`, by default ELEM_FACTOR *
    tol); returns both errors."""
    elem_tol = ELEM_FACTOR * tol if elem_tol is None else elem_tol
    rel, mx = head_rel_err(x, ref, head_axes), head_max_err(x, ref, head_axes)
    print(f"{label}: max head rel err {rel:.3e}, max elementwise err / RMS {mx:.3e}")
    assert rel < tol, f"{label}: Frobenius {rel:.3e} >= {tol:.1e}"
    assert mx < elem_tol, f"{label}: elementwise {mx:.3e} >= {elem_tol:.1e}"
    return rel, mx


def oracle_forward(w, inp, S0=None, heads=None):
    """Oracle on the synth inputs; `heads` = optional list of (b, h) to restrict to."""
    S0 = inp.get("S0") if S0 is None else S0
    args = [inp["q"], inp["k"], inp["v"], inp["log_w"], inp["e1"], inp["e2"], S0]
    if heads is None:
        return oracle.forward(w.form, *args)
    outs = []
    for b, h in heads:
        sub = [None if a is None else (a[b:b + 1, h:h + 1] if a.ndim == 4 and a is S0 else
                                       (a[b:b + 1, :, h:h + 1] if a.ndim >= 3 else a))
               for a in args]
        outs.append(oracle.forward(w.form, *sub))
    return outs


def gpu_forward(w, inp, algo="auto", chunk=None, S0=None, device="cuda", workspace_bytes=None):
    """``workspace_bytes`` = None sizes the workspace with gdr_forward_workspace_size (the
    fastest path); a small value (e.g. 256) selects the single-kernel tensor-core path."""
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, w.dtype,
                      device)
    s0 = inp.get("S0") if S0 is None else S0
    s0 = None if s0 is None else torch.from_numpy(np.ascontiguousarray(s0, np.float32)).to(device)
    ws = None if workspace_bytes is None else gdr.new_workspace(workspace_bytes, device)
    o, S_T = gdr.gdr_forward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                     d["e2"], s0, chunk=chunk or w.chunk, algo=algo,
                                     workspace=ws)
    torch.cuda.synchronize()
    return o.cpu().numpy(), S_T.cpu().numpy()


def small(form, dtype, dk=64, dv=64, T=100, B=2, H=3, chunk=32, seed=11, **kw):
    base = dict(gdn2=synth.PRESETS["gdn2_bf16"], rwkv7=synth.PRESETS["rwkv7_bf16"],
                general=synth.PRESETS["rwkv7_bf16"], gla=synth.PRESETS["gdn2_bf16"])[form]
    return base.with_(name=f"{form}_{dtype}_small", form=form, dtype=dtype, B=B, H=H, T=T,
                      dk=dk, dv=dv, chunk=chunk, seed=seed, **kw)
