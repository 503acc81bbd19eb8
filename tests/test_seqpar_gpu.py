"""Sequence parallelism's data path on one GPU: gdr_state_compose against fp64 products,
and the segment-map algorithm (maps of every segment, entry states by composition, each
segment's pass) against the oracle over the whole sequence."""
import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, seqpar, synth
from parity import TOL, head_rel_err, oracle_forward, small

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (16, 16), (32, 64)])
@pytest.mark.parametrize("with_in", [True, False])
def test_state_compose(dk, dv, with_in):
    rng = np.random.default_rng(dk + dv)
    B, H = 2, 3
    M = rng.standard_normal((B, H, dk, dk)).astype(np.float32)
    S = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    Q = rng.standard_normal((B, H, dk, dv)).astype(np.float32)
    c = lambda a: torch.from_numpy(a).cuda()
    out = gdr.gdr_state_compose(c(M), c(S) if with_in else None, c(Q)).cpu().numpy()
    ref = (M.astype(np.float64) @ S.astype(np.float64) if with_in else 0.0) + Q
    assert np.max(np.abs(out - ref)) < 2e-5 * max(np.max(np.abs(ref)), 1.0)


@pytest.mark.parametrize("form,dk,dtype", [("gdn2", 128, "bf16"), ("rwkv7", 64, "bf16"),
                                           ("general", 64, "f32"), ("gla", 128, "bf16")])
@pytest.mark.parametrize("n_seg", [2, 3, 4])
def test_segments_compose_to_the_whole_sequence(form, dk, dtype, n_seg):
    w = small(form, dtype, dk=dk, dv=dk, T=301, B=2, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    inp["S0"] = synth.round_f32(np.random.default_rng(4).normal(0, 0.5, (w.B, w.H, dk, dk)))
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, dtype)
    S0 = torch.from_numpy(inp["S0"]).cuda()
    o, S = seqpar.emulate_segments(form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"], S0,
                                   n_seg=n_seg, chunk=w.chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_forward(w, inp)
    eo = head_rel_err(o.cpu().numpy(), o_ref, (0, 2))
    es = head_rel_err(S.cpu().numpy(), S_ref, (0, 1))
    print(f"seqpar {form} {dtype} d={dk} segments={n_seg}: o {eo:.2e} S {es:.2e}")
    assert eo < TOL[dtype] and es < TOL[dtype]


def test_single_process_is_the_plain_forward():
    w = small("gdn2", "bf16", dk=128, dv=128, T=200, B=1, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    o, S_T, S_in = seqpar.sequence_parallel_forward("gdn2", d["q"], d["k"], d["v"], d["log_w"],
                                                    d["e1"], d["e2"])
    o2, S2 = gdr.gdr_forward_chunked("gdn2", d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"])
    assert S_in is None and torch.equal(o, o2) and torch.equal(S_T, S2)
