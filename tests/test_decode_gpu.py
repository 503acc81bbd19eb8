"""GPU parity of gdr_decode_step against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth
from parity import ELEM_TOL, TOL, head_max_err, head_rel_err, small

pytestmark = pytest.mark.gpu


def _dev(inp, dtype):
    return gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, dtype)


@pytest.mark.parametrize("form", ["gdn2", "rwkv7", "general", "gla"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (16, 128), (128, 32), (32, 16)])
def test_decode_small(form, dtype, dk, dv):
    w = small(form, dtype, dk=dk, dv=dv, T=1, B=3, H=5).with_(s0_std=0.3)
    S0 = synth.decode_state(w)
    S = torch.from_numpy(S0).cuda()
    S_ref = S0.astype(np.float64)
    for step in range(4):
        inp = synth.decode_step_inputs(w, step)
        d = _dev(inp, dtype)
        o = gdr.gdr_decode_step(form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"], S)
        o_ref, S_ref = oracle.decode_step(form, inp["q"], inp["k"], inp["v"], inp["log_w"],
                                          inp["e1"], inp["e2"], S_ref)
        torch.cuda.synchronize()
        assert head_rel_err(o.cpu().numpy()[:, :, None], o_ref[:, :, None], (0, 1)) < 1e-5
        assert head_rel_err(S.cpu().numpy(), S_ref, (0, 1)) < 1e-5


def test_decode_full_size():
    """B=256, H=32, d=128, state N(0, 0.1): every head over 10 steps, then 1000
    consecutive steps (inputs cycled from a pool of 16 seeded steps) checked on a
    subset of heads at steps 1, 10, 100, 1000."""
    w = synth.PRESETS["decode"]
    S0 = synth.decode_state(w)
    S = torch.from_numpy(S0).cuda()
    pool = [synth.decode_step_inputs(w, s) for s in range(16)]
    dpool = [_dev(p, "bf16") for p in pool]
    heads = [(b, h) for b in (0, 77, 255) for h in (0, 13, 31)]
    bsel = sorted({b for b, _ in heads})
    S_sub = S0[bsel].astype(np.float64)
    S_all = S0.astype(np.float64)
    worst = worst_el = 0.0
    for step in range(1, 1001):
        p, d = pool[(step - 1) % 16], dpool[(step - 1) % 16]
        o = gdr.gdr_decode_step("gdn2", d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"], S)
        sub = {k: None if p[k] is None else p[k][bsel] for k in p}
        o_sub, S_sub = oracle.decode_step("gdn2", sub["q"], sub["k"], sub["v"], sub["log_w"],
                                          sub["e1"], sub["e2"], S_sub)
        if step <= 10:
            o_all, S_all = oracle.decode_step("gdn2", p["q"], p["k"], p["v"], p["log_w"],
                                              p["e1"], p["e2"], S_all)
            torch.cuda.synchronize()
            og, Sg = o.cpu().numpy()[:, :, None], S.cpu().numpy()
            worst = max(worst, head_rel_err(og, o_all[:, :, None], (0, 1)),
                        head_rel_err(Sg, S_all, (0, 1)))
            worst_el = max(worst_el, head_max_err(og, o_all[:, :, None], (0, 1)),
                           head_max_err(Sg, S_all, (0, 1)))
        if step in (1, 10, 100, 1000):
            torch.cuda.synchronize()
            Sg = S.cpu().numpy()[bsel]
            og = o.cpu().numpy()[bsel]
            worst = max(worst, head_rel_err(Sg, S_sub, (0, 1)),
                        head_rel_err(og[:, :, None], o_sub[:, :, None], (0, 1)))
            worst_el = max(worst_el, head_max_err(Sg, S_sub, (0, 1)),
                           head_max_err(og[:, :, None], o_sub[:, :, None], (0, 1)))
    print(f"decode 1000 steps: max head rel err {worst:.3e}, max elementwise err / RMS {worst_el:.3e}")
    assert worst < TOL["bf16"] and worst_el < ELEM_TOL["bf16"]
