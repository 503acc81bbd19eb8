"""The autograd entry point: loss.backward() through gdr_chunked against the oracle's
reverse mode (same bars as the backward's parity tests)."""
import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth
from matrix_memory_rnn_b200.autograd import gdr_chunked
from parity import TOL, head_rel_err, small

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("form,dtype,d", [("gdn2", "bf16", 128), ("rwkv7", "bf16", 64),
                                          ("general", "f32", 64), ("gla", "bf16", 128)])
def test_autograd_matches_the_oracle(form, dtype, d):
    w = small(form, dtype, dk=d, dv=d, T=150, B=2, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    rng = np.random.default_rng(21)
    S0 = synth.round_f32(rng.normal(0, 0.5, (w.B, w.H, d, d)))
    dO = synth.round_f32(rng.standard_normal((w.B, w.T, w.H, d)))
    dST = synth.round_f32(rng.standard_normal((w.B, w.H, d, d)))
    dev = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, dtype)
    leaves = {k: (None if t is None else t.clone().requires_grad_(True)) for k, t in dev.items()}
    S0_t = torch.from_numpy(S0).cuda().requires_grad_(True)
    o, S_T = gdr_chunked(form, *(leaves[k] for k in ("q", "k", "v", "log_w", "e1", "e2")), S0_t)
    loss = (o * torch.from_numpy(dO).cuda()).sum() + (S_T * torch.from_numpy(dST).cuda()).sum()
    loss.backward()
    torch.cuda.synchronize()
    ref = oracle.backward(form, inp["q"], inp["k"], inp["v"], inp["log_w"], inp["e1"], inp["e2"],
                          S0, dO, dST)
    tol = TOL[dtype]   # bf16 inputs get their gradients back in bf16 (one more rounding)
    for name, leaf in leaves.items():
        if leaf is None:
            continue
        assert leaf.grad is not None and leaf.grad.dtype == leaf.dtype, name
        axes = (0, 2)
        err = head_rel_err(leaf.grad.float().cpu().numpy(), ref[name], axes)
        assert err < tol, (name, err)
    assert head_rel_err(S0_t.grad.cpu().numpy(), ref["S0"], (0, 1)) < TOL[dtype]
