"""GPU parity of gdr_mlstm_forward (xLSTM's mLSTM cell with the log-domain stabilizer)
against the fp64 oracle: readouts h per head (relative Frobenius norm, the forward's bars),
the final stabilized state (C, n per head; m within fp32 rounding of its sums)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth
from parity import TOL, check_parity, head_rel_err, small

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(__file__), "golden", "mlstm_recovery_ch13_4.json")


def _state(w, seed):
    """A stabilized state as a previous call leaves it (from the oracle on a short prefix)."""
    inp = synth.mlstm_inputs(w.with_(T=9), seed=seed)
    _, C, n, m = oracle.mlstm_forward(inp["q"], inp["k"], inp["v"], inp["f_pre"], inp["i_pre"])
    return C.astype(np.float32), n.astype(np.float32), m.astype(np.float32)


def _gpu(w, inp, state=None):
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to("cuda", tdt) for k in ("q", "k", "v")}
    g = {k: torch.from_numpy(np.ascontiguousarray(inp[k], np.float32)).cuda() for k in ("f_pre", "i_pre")}
    st = [None] * 3 if state is None else [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in state]
    out = gdr.gdr_mlstm_forward(d["q"], d["k"], d["v"], g["f_pre"], g["i_pre"], *st)
    torch.cuda.synchronize()
    return [x.cpu().numpy() for x in out]


def _check(w, inp, state, tol, label):
    h, C, n, m = _gpu(w, inp, state)
    st = [None] * 3 if state is None else state
    hr, Cr, nr, mr = oracle.mlstm_forward(inp["q"], inp["k"], inp["v"], inp["f_pre"], inp["i_pre"], *st)
    eh = head_rel_err(h, hr, (0, 2))
    eC = head_rel_err(C, Cr, (0, 1))
    en = head_rel_err(n, nr, (0, 1))
    em = float(np.max(np.abs(m - mr) / (1.0 + np.abs(mr))))
    print(f"{label}: h {eh:.2e} C {eC:.2e} n {en:.2e} m {em:.2e}")
    assert np.isfinite(h).all()
    assert eh < tol and eC < tol and en < tol and em < 1e-5


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 64, 100, 257])
@pytest.mark.parametrize("with_state", [False, True])
def test_mlstm_parity(dtype, dk, dv, T, with_state):
    w = small("gdn2", dtype, dk=dk, dv=dv, T=T, B=2, H=3, chunk=64)
    inp = synth.mlstm_inputs(w)
    state = _state(w, 77) if with_state else None
    _check(w, inp, state, TOL[dtype], f"mlstm {dtype} {dk}x{dv} T={T} S0={with_state}")


def _readout_condition(inp):
    """kappa_t per (b, t, h): the condition number of the readout's quotient,
    (|q_t| . n~_t) / max(|q_t . n_t|, e^{-m_t}), with n~_t the normalizer built from |k| (the same
    gates, so the oracle forms it when given |k| for k).  A kernel whose sums carry a relative
    rounding u returns h_t with an error of order u kappa_t |h_t|, whatever its order of
    summation: where q_t . n_t nearly cancels, kappa_t is large."""
    B, T, H, _ = inp["q"].shape
    q = np.asarray(inp["q"], np.float64)
    kap = np.ones((B, T, H))
    for t in range(T):
        sl = {k: x[:, :t + 1] for k, x in inp.items()}
        _, _, n, m = oracle.mlstm_forward(sl["q"], sl["k"], sl["v"], sl["f_pre"], sl["i_pre"])
        _, _, na, _ = oracle.mlstm_forward(sl["q"], np.abs(sl["k"]), sl["v"], sl["f_pre"], sl["i_pre"])
        qt = q[:, t]
        kap[:, t] = (np.abs(qt) * na).sum(-1) / np.maximum(np.abs((qt * n).sum(-1)), np.exp(-m))
    return kap


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk", [64, 128])
def test_mlstm_large_input_gates(dtype, dk):
    """Input log-gates up to 800 (the naive memory would overflow): the stabilized cell stays
    finite and matches.  After a dominant gate, q_t . n_t is small against |q_t| |n_t| for some
    tokens, so h_t there is a quotient of two nearly cancelling sums, and any fixed-precision
    kernel errs there in proportion to the quotient's condition number kappa_t.  The bar is
    the forward's, applied to each token's error divided by max(1, kappa_t); bf16 inputs must
    also meet it unweighted.  That holds only with the state operand of Q C and Q n carried
    past bf16."""
    w = small("gdn2", dtype, dk=dk, dv=dk, T=200, B=1, H=2, chunk=64)
    inp = synth.mlstm_inputs(w, i_mu=5.0, i_sd=4.0)
    i = inp["i_pre"].copy()
    i[0, 17, 0], i[0, 130, 1], i[0, 131, 1] = 800.0, 760.0, 790.0
    inp["i_pre"] = i
    h, C, n, m = _gpu(w, inp)
    hr, Cr, nr, mr = oracle.mlstm_forward(inp["q"], inp["k"], inp["v"], inp["f_pre"], inp["i_pre"])
    assert np.isfinite(h).all()
    kap = _readout_condition(inp)
    dh = np.linalg.norm(h - hr, axis=-1) / np.maximum(1.0, kap)     # [B, T, H]
    ew = max(np.sqrt((dh[..., j] ** 2).sum() / (hr[..., j, :] ** 2).sum()) for j in range(w.H))
    eh = head_rel_err(h, hr, (0, 2))
    eC, en = head_rel_err(C, Cr, (0, 1)), head_rel_err(n, nr, (0, 1))
    print(f"mlstm large gates {dtype} d={dk}: h {eh:.2e} (kappa-weighted {ew:.2e}, max kappa "
          f"{kap.max():.1e}) C {eC:.2e} n {en:.2e}")
    assert ew < TOL[dtype] and eC < TOL[dtype] and en < TOL[dtype]
    assert np.max(np.abs(m - mr) / (1.0 + np.abs(mr))) < 1e-5
    if dtype == "bf16":
        assert eh < TOL[dtype]


def test_mlstm_recovery_on_the_gpu():
    with open(GOLD) as fh:
        gold = json.load(fh)
    dk = dv = 64
    key = np.zeros(dk, np.float32)
    key[3], key[40] = 0.6, -0.8
    v = np.zeros(dv, np.float32)
    v[:3] = gold["v"]
    w = small("gdn2", "f32", dk=dk, dv=dv, T=1, B=1, H=1, chunk=64)
    inp = {"q": key.reshape(1, 1, 1, dk), "k": key.reshape(1, 1, 1, dk), "v": v.reshape(1, 1, 1, dv),
           "f_pre": np.zeros((1, 1, 1), np.float32),
           "i_pre": np.full((1, 1, 1), gold["input_log_gate"], np.float32)}
    h = _gpu(w, inp)[0]
    assert np.max(np.abs(h.ravel() - v)) < 1e-6


def test_mlstm_state_continues():
    """Two calls with the state passed between them equal one call up to rounding (the
    split at token 130 moves the chunk boundaries; tf32 products on bf16 inputs)."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=300, B=2, H=2, chunk=64)
    inp = synth.mlstm_inputs(w)
    h, C, n, m = _gpu(w, inp)
    a = {k: x[:, :130] for k, x in inp.items()}
    b = {k: x[:, 130:] for k, x in inp.items()}
    h1, C1, n1, m1 = _gpu(w.with_(T=130), a)
    h2, C2, n2, m2 = _gpu(w.with_(T=170), b, (C1, n1, m1))
    assert head_rel_err(np.concatenate([h1, h2], 1), h, (0, 2)) < 2e-3
    assert head_rel_err(C2, C, (0, 1)) < 2e-3 and np.max(np.abs(m2 - m)) < 1e-4


def test_mlstm_zero_length():
    w = small("gdn2", "bf16", dk=64, dv=64, T=0, B=1, H=2, chunk=64)
    inp = synth.mlstm_inputs(w)
    h, C, n, m = _gpu(w, inp)
    assert h.shape == (1, 0, 2, 64) and not C.any() and not n.any() and np.all(np.isneginf(m))


@pytest.mark.parametrize("preset", ["gdn2_bf16", "rwkv7_bf16"])
def test_mlstm_full_size_sampled_heads(preset):
    w = synth.PRESETS[preset]
    inp = synth.mlstm_inputs(w)
    h, C, n, m = _gpu(w, inp)
    for b, hh in ((0, 0), (w.B - 1, w.H - 1)):
        sl = {k: x[b:b + 1, :, hh:hh + 1] for k, x in inp.items()}
        hr, Cr, _, _ = oracle.mlstm_forward(sl["q"], sl["k"], sl["v"], sl["f_pre"], sl["i_pre"])
        check_parity(h[b:b + 1, :, hh:hh + 1], hr, (0, 2), TOL["bf16"], f"mlstm full size ({b},{hh}) h")
        check_parity(C[b:b + 1, hh:hh + 1], Cr, (0, 1), TOL["bf16"], f"mlstm full size ({b},{hh}) C")


def _bf16_case(T=257, B=1, H=2, d=128):
    w = small("gdn2", "bf16", dk=d, dv=d, T=T, B=B, H=H, chunk=64)
    inp = synth.mlstm_inputs(w)
    d = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to("cuda", torch.bfloat16) for k in ("q", "k", "v")}
    g = {k: torch.from_numpy(np.ascontiguousarray(inp[k], np.float32)).cuda() for k in ("f_pre", "i_pre")}
    return w, inp, d, g


@pytest.mark.parametrize("dk", [64, 128])
def test_mlstm_status_word_stays_ok_and_changes_nothing(dk):
    """The tensor-core kernel (bf16, d_k = d_v = dk) leaves a given status word at GDR_OK, and
    the outputs are bit-identical with and without it."""
    w, inp, d, g = _bf16_case(d=dk)
    status = torch.zeros(64, dtype=torch.uint8, device="cuda")
    h1, C1, n1, m1 = gdr.gdr_mlstm_forward(d["q"], d["k"], d["v"], g["f_pre"], g["i_pre"], status=status)
    assert gdr.gdr_read_status(status) == "GDR_OK"
    h0, C0, n0, m0 = gdr.gdr_mlstm_forward(d["q"], d["k"], d["v"], g["f_pre"], g["i_pre"])
    torch.cuda.synchronize()
    for x, y in ((h1, h0), (C1, C0), (n1, n0), (m1, m0)):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dk", [64, 128])
def test_mlstm_bounded_wait_reports_timeout_and_context_survives(monkeypatch, dk):
    """Fault injection on the host: the kernel withholds the commit of [P~ V | P~ 1], the
    bounded wait for it runs out (about 2 s), GDR_ERR_TIMEOUT lands in the status word, and
    the next call on the same context matches the oracle."""
    w, inp, d, g = _bf16_case(T=130, d=dk)
    status = torch.zeros(4, dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("GDR_DEBUG_FAULT", "skip_handoff")
    gdr.gdr_mlstm_forward(d["q"], d["k"], d["v"], g["f_pre"], g["i_pre"], status=status)
    assert gdr.gdr_read_status(status) == "GDR_ERR_TIMEOUT"
    monkeypatch.delenv("GDR_DEBUG_FAULT")
    h, C, n, m = gdr.gdr_mlstm_forward(d["q"], d["k"], d["v"], g["f_pre"], g["i_pre"], status=status)
    assert gdr.gdr_read_status(status) == "GDR_OK"
    hr, Cr, nr, mr = oracle.mlstm_forward(inp["q"], inp["k"], inp["v"], inp["f_pre"], inp["i_pre"])
    check_parity(h.cpu().numpy(), hr, (0, 2), TOL["bf16"], "mlstm after a timeout: h")
    check_parity(C.cpu().numpy(), Cr, (0, 1), TOL["bf16"], "mlstm after a timeout: C")
