"""Seeded sweep of small random configurations against the fp64 oracle: forward (every
form, both input dtypes, head dimensions 16..128, ragged lengths, every chunk size, the
automatic path and the fp32 kernel, with and without an initial state), decode, the
reverse mode and the mLSTM cell.  The configurations are drawn once from a fixed seed, so
the cases are the same on every run; each stays small enough for the oracle."""
import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth
from parity import TOL, TOL_FP32_KERNEL, gpu_forward, head_rel_err, oracle_forward, small

pytestmark = pytest.mark.gpu

FORMS = ["gdn2", "rwkv7", "general", "gla"]
DIMS = [16, 32, 64, 128]
_rng = np.random.default_rng(20261202)


def _draw_forward(n):
    cases = []
    for i in range(n):
        cases.append(dict(form=FORMS[_rng.integers(4)], dtype=["bf16", "f32"][_rng.integers(2)],
                          dk=int(_rng.choice(DIMS)), dv=int(_rng.choice(DIMS)),
                          T=int(_rng.integers(1, 261)), B=int(_rng.integers(1, 3)),
                          H=int(_rng.integers(1, 4)), chunk=int(_rng.choice([16, 32, 64, 128])),
                          algo=["auto", "fp32"][_rng.integers(2)], state=bool(_rng.integers(2)),
                          seed=1000 + i))
    return cases


def _draw(n, dims, tmax, seed0):
    return [dict(form=FORMS[_rng.integers(4)], dtype=["bf16", "f32"][_rng.integers(2)],
                 dk=int(_rng.choice(dims)), dv=int(_rng.choice(dims)), T=int(_rng.integers(1, tmax)),
                 B=int(_rng.integers(1, 3)), H=int(_rng.integers(1, 4)), state=bool(_rng.integers(2)),
                 seed=seed0 + i) for i in range(n)]


FWD = _draw_forward(48)
DEC = _draw(16, DIMS, 2, 2000)
BWD = _draw(16, [64, 128], 141, 3000)
MLSTM = _draw(12, [64, 128], 201, 4000)


def _id(c):
    return "-".join(f"{k}{v}" for k, v in c.items() if k != "seed")


def _state(rng, B, H, dk, dv, std=0.5):
    return synth.round_f32(rng.normal(0.0, std, (B, H, dk, dv)))


@pytest.mark.parametrize("c", FWD, ids=_id)
def test_sweep_forward(c):
    w = small(c["form"], c["dtype"], dk=c["dk"], dv=c["dv"], T=c["T"], B=c["B"], H=c["H"],
              chunk=c["chunk"], seed=c["seed"])
    inp = synth.forward_inputs(w)
    if c["state"]:
        inp["S0"] = _state(np.random.default_rng(c["seed"]), w.B, w.H, w.dk, w.dv)
    o, S = gpu_forward(w, inp, algo=c["algo"])
    o_ref, S_ref = oracle_forward(w, inp)
    tol = TOL_FP32_KERNEL if (c["algo"] == "fp32" or c["dtype"] == "f32") else TOL["bf16"]
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    assert np.isfinite(o).all() and np.isfinite(S).all()
    assert eo < tol and es < tol, (eo, es)


@pytest.mark.parametrize("c", DEC, ids=_id)
def test_sweep_decode(c):
    w = small(c["form"], c["dtype"], dk=c["dk"], dv=c["dv"], T=1, B=c["B"], H=c["H"],
              seed=c["seed"]).with_(s0_std=0.3)
    S0 = synth.decode_state(w)
    S = torch.from_numpy(S0).cuda()
    S_ref = S0.astype(np.float64)
    for step in range(3):
        inp = synth.decode_step_inputs(w, step)
        d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, c["dtype"])
        o = gdr.gdr_decode_step(c["form"], d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"], S)
        o_ref, S_ref = oracle.decode_step(c["form"], inp["q"], inp["k"], inp["v"], inp["log_w"],
                                          inp["e1"], inp["e2"], S_ref)
        torch.cuda.synchronize()
        assert head_rel_err(o.cpu().numpy()[:, :, None], o_ref[:, :, None], (0, 1)) < 1e-5
        assert head_rel_err(S.cpu().numpy(), S_ref, (0, 1)) < 1e-5


@pytest.mark.parametrize("c", BWD, ids=_id)
def test_sweep_backward(c):
    w = small(c["form"], c["dtype"], dk=c["dk"], dv=c["dv"], T=c["T"], B=c["B"], H=c["H"],
              chunk=64, seed=c["seed"])
    inp = synth.forward_inputs(w)
    rng = np.random.default_rng(c["seed"])
    S0 = _state(rng, w.B, w.H, w.dk, w.dv) if c["state"] else None
    dO = synth.round_f32(rng.standard_normal((w.B, w.T, w.H, w.dv)))
    dST = synth.round_f32(rng.standard_normal((w.B, w.H, w.dk, w.dv)))
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, w.dtype)
    f32 = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    g = gdr.gdr_backward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"],
                                 f32(S0), f32(dO), f32(dST))
    torch.cuda.synchronize()
    ref = oracle.backward(w.form, inp["q"], inp["k"], inp["v"], inp["log_w"], inp["e1"], inp["e2"],
                          S0, dO, dST)
    axes = {"S0": (0, 1)}
    for name, r in ref.items():
        if r is None:
            assert g[name] is None, name
            continue
        x = g[name].cpu().numpy()
        assert np.isfinite(x).all(), name
        err = head_rel_err(x, r, axes.get(name, (0, 2)))
        assert err < TOL[c["dtype"]], (name, err)


@pytest.mark.parametrize("c", MLSTM, ids=_id)
def test_sweep_mlstm(c):
    w = small("gdn2", c["dtype"], dk=c["dk"], dv=c["dv"], T=c["T"], B=c["B"], H=c["H"], chunk=64,
              seed=c["seed"])
    inp = synth.mlstm_inputs(w)
    state = None
    if c["state"]:
        pre = synth.mlstm_inputs(w.with_(T=7), seed=c["seed"] + 1)
        _, C, n, m = oracle.mlstm_forward(pre["q"], pre["k"], pre["v"], pre["f_pre"], pre["i_pre"])
        state = (C.astype(np.float32), n.astype(np.float32), m.astype(np.float32))
    tdt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
    d = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to("cuda", tdt) for k in ("q", "k", "v")}
    gt = {k: torch.from_numpy(np.ascontiguousarray(inp[k], np.float32)).cuda() for k in ("f_pre", "i_pre")}
    st = [None] * 3 if state is None else [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in state]
    h, C, n, m = (x.cpu().numpy() for x in
                  gdr.gdr_mlstm_forward(d["q"], d["k"], d["v"], gt["f_pre"], gt["i_pre"], *st))
    torch.cuda.synchronize()
    hr, Cr, nr, mr = oracle.mlstm_forward(inp["q"], inp["k"], inp["v"], inp["f_pre"], inp["i_pre"],
                                          *([None] * 3 if state is None else state))
    tol = TOL[c["dtype"]]
    assert head_rel_err(h, hr, (0, 2)) < tol
    assert head_rel_err(C, Cr, (0, 1)) < tol and head_rel_err(n, nr, (0, 1)) < tol
    assert np.max(np.abs(m - mr) / (1.0 + np.abs(mr))) < 1e-5
