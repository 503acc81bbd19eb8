"""GPU parity of gdr_backward_chunked against the fp64 oracle's reverse mode.

Every gradient (q, k, v, log_w, e1, e2, S0) is compared per head with the same
relative Frobenius norm and bars as the forward (1e-4 for fp32 inputs, 2e-2 for
bf16 inputs), on seeded synthetic inputs with a random initial state, a random
output gradient dO and a random final-state gradient dS_T.
"""
import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth
from parity import ELEM_TOL, TOL, head_max_err, head_rel_err, small

pytestmark = pytest.mark.gpu

FORMS = ["gdn2", "rwkv7", "general", "gla"]
# per-head axes of each gradient: token-major [B, T, H, .] or RWKV-7's c [B, T, H]
HEAD_AXES = {"q": (0, 2), "k": (0, 2), "v": (0, 2), "log_w": (0, 2), "e1": (0, 2), "e2": (0, 2),
             "S0": (0, 1)}


def _case(w, seed=5, with_state=True, with_dST=True, log_w=None, e2_none=False):
    inp = synth.forward_inputs(w)
    if log_w is not None:
        inp["log_w"] = log_w(inp["log_w"]).astype(np.float32)
    if e2_none:
        inp["e2"] = None
    rng = np.random.default_rng(seed)
    S0 = synth.round_f32(rng.normal(0, 0.5, (w.B, w.H, w.dk, w.dv))) if with_state else None
    dO = synth.round_f32(rng.standard_normal((w.B, w.T, w.H, w.dv)))
    dST = synth.round_f32(rng.standard_normal((w.B, w.H, w.dk, w.dv))) if with_dST else None
    return inp, S0, dO, dST


def _gpu_backward(w, inp, S0, dO, dST):
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, w.dtype)
    f32 = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    g = gdr.gdr_backward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"],
                                 f32(S0), f32(dO), f32(dST))
    torch.cuda.synchronize()
    return {k: None if x is None else x.cpu().numpy() for k, x in g.items()}


def _compare(w, inp, S0, dO, dST, tol, label):
    g = _gpu_backward(w, inp, S0, dO, dST)
    ref = oracle.backward(w.form, inp["q"], inp["k"], inp["v"], inp["log_w"], inp["e1"],
                          inp["e2"], S0, dO, dST)
    errs = {}
    for name, r in ref.items():
        if r is None:
            assert g[name] is None, name
            continue
        assert g[name] is not None and g[name].shape == r.shape, name
        assert np.isfinite(g[name]).all(), f"{label}: non-finite d{name}"
        errs[name] = head_rel_err(g[name], r, HEAD_AXES[name])
    print(label, " ".join(f"{k}:{v:.1e}" for k, v in errs.items()))
    bad = {k: v for k, v in errs.items() if not v < tol}
    assert not bad, f"{label}: {bad}"
    return errs


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv,T", [(64, 64, 100), (128, 128, 77), (64, 128, 33), (128, 64, 1),
                                     (64, 64, 32)])
def test_backward_parity(form, dtype, dk, dv, T):
    w = small(form, dtype, dk=dk, dv=dv, T=T, B=2, H=2, chunk=64)
    inp, S0, dO, dST = _case(w)
    _compare(w, inp, S0, dO, dST, TOL[dtype], f"bwd {form} {dtype} {dk}x{dv} T={T}")


@pytest.mark.parametrize("form", ["gdn2", "rwkv7"])
def test_backward_without_state_gradients(form):
    """S0 = 0 and dS_T = 0 (the training case), over many chunks."""
    w = small(form, "bf16", dk=64, dv=64, T=300, B=1, H=3, chunk=64)
    inp, S0, dO, dST = _case(w, with_state=False, with_dST=False)
    _compare(w, inp, S0, dO, dST, TOL["bf16"], f"bwd {form} no state")


def test_backward_gdn2_without_write_gate():
    w = small("gdn2", "bf16", dk=128, dv=128, T=90, B=1, H=2, chunk=64)
    inp, S0, dO, dST = _case(w, e2_none=True)
    _compare(w, inp, S0, dO, dST, TOL["bf16"], "bwd gdn2 no wg")


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_strong_decay_uses_exact_path(form, dtype):
    """Chunks where a channel decays by more than 80 nats form their decayed products
    from pairwise exponentials; both paths in one call."""
    w = small(form, dtype, dk=64, dv=64, T=130, B=1, H=2, chunk=64)

    def strong(lw):
        lw = lw.copy()
        lw[:, :, :, ::5] = -3.5           # 32 tokens x 3.5 nats = 112 nats per chunk
        lw[:, 40:44, 1, 7] = -60.0
        return lw
    inp, S0, dO, dST = _case(w, log_w=strong)
    _compare(w, inp, S0, dO, dST, TOL[dtype], f"bwd strong decay {form} {dtype}")


def test_backward_zero_length_and_empty():
    w = small("gdn2", "bf16", dk=64, dv=64, T=0, B=2, H=2, chunk=64)
    inp, S0, dO, dST = _case(w)
    g = _gpu_backward(w, inp, S0, dO, dST)
    assert np.array_equal(g["S0"], dST) and g["q"].shape == (2, 0, 2, 64)


def test_backward_rejects_unsupported_dims():
    w = small("gla", "bf16", dk=32, dv=64, T=10, B=1, H=1, chunk=64)
    inp, S0, dO, dST = _case(w)
    with pytest.raises(gdr.GdrError) as ei:
        _gpu_backward(w, inp, S0, dO, dST)
    assert ei.value.code == 2


@pytest.mark.parametrize("preset", ["gdn2_bf16", "rwkv7_bf16"])
def test_backward_full_size_sampled_heads(preset):
    """The full workloads in one call; the oracle checks two sampled heads (every
    (b, h) is an independent sequence, so its inputs are a slice)."""
    w = synth.PRESETS[preset]
    inp, S0, dO, dST = _case(w, with_state=False)
    g = _gpu_backward(w, inp, S0, dO, dST)
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sl = lambda a: None if a is None else a[b:b + 1, :, h:h + 1]
        ref = oracle.backward(w.form, sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_w"]),
                              sl(inp["e1"]), sl(inp["e2"]), None, sl(dO),
                              dST[b:b + 1, h:h + 1])
        for name, r in ref.items():
            if r is None:
                continue
            x = g[name][b:b + 1, h:h + 1] if name == "S0" else g[name][b:b + 1, :, h:h + 1]
            err = head_rel_err(x, r, HEAD_AXES[name])
            el = head_max_err(x, r, HEAD_AXES[name])
            print(f"bwd {preset} head ({b},{h}) d{name}: {err:.2e} elementwise {el:.2e}")
            assert err < TOL["bf16"], (name, err)
            assert el < ELEM_TOL["bf16"], (name, el)
