"""gdr_state_init on the GPU: the zero fill and the copy, bit for bit, and a sequence
resumed through a state that it copied, against the oracle on the whole sequence.

The state is the checkpoint a stream resumes from ("Muir ...", section 4.2: the chunk's
end state is affine in its start state, eq. (10), so a sequence split at any token and
continued from the carried state is the same sequence).
"""
import numpy as np
import pytest
import torch

from matrix_memory_rnn_b200 import gdr, synth
from parity import TOL, check_parity, oracle_forward, small

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,dk,dv", [(2, 3, 128, 128), (1, 1, 16, 32), (3, 2, 64, 16)])
def test_zero_fill_and_copy_are_exact(B, H, dk, dv):
    S = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    gdr.gdr_state_init(S)
    torch.cuda.synchronize()
    got = S.cpu().numpy()
    assert got.view(np.uint32).max() == 0, "zero fill must write +0.0 everywhere"

    src = torch.from_numpy(np.random.default_rng(B * 100 + dk).standard_normal(
        (B, H, dk, dv)).astype(np.float32)).cuda()
    src[0, 0, 0, 0] = float("-inf")        # special values are copied as bits
    src[-1, -1, -1, -1] = -0.0
    S.fill_(float("nan"))
    gdr.gdr_state_init(S, src)
    torch.cuda.synchronize()
    assert np.array_equal(S.cpu().numpy().view(np.uint32), src.cpu().numpy().view(np.uint32))

    # src == S is a no-op
    gdr.gdr_state_init(S, S)
    torch.cuda.synchronize()
    assert np.array_equal(S.cpu().numpy().view(np.uint32), src.cpu().numpy().view(np.uint32))


def test_on_a_side_stream_orders_with_the_forward():
    """The fill is enqueued on the given stream, ahead of a forward on the same stream."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=70, B=1, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    s = torch.cuda.Stream()
    S = torch.full((w.B, w.H, w.dk, w.dv), float("nan"), device="cuda")
    torch.cuda.current_stream().synchronize()
    with torch.cuda.stream(s):
        gdr.gdr_state_init(S, stream=s)
        o, S_T = gdr.gdr_forward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                         d["e2"], S, chunk=64, stream=s)
    s.synchronize()
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o.cpu().numpy(), o_ref, (0, 2), TOL["bf16"], "from a zero-filled state: o")
    check_parity(S_T.cpu().numpy(), S_ref, (0, 1), TOL["bf16"], "from a zero-filled state: S_T")


@pytest.mark.parametrize("form,d,algo", [("gdn2", 128, "auto"), ("rwkv7", 64, "auto"),
                                         ("general", 64, "fp32")])
def test_resume_through_a_copied_state(form, d, algo):
    """[0, T1) from S0, the state copied into a fresh NaN-filled buffer by gdr_state_init,
    then [T1, T) from the copy: o and S_T against the oracle on [0, T)."""
    w = small(form, "bf16", dk=d, dv=d, T=230, B=2, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    inp["S0"] = synth.round_f32(np.random.default_rng(31).normal(0, 0.5, (w.B, w.H, d, d)))
    dev = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    S0 = torch.from_numpy(inp["S0"]).cuda()
    T1 = 100
    part = lambda lo, hi: {k: None if x is None else x[:, lo:hi].contiguous() for k, x in dev.items()}
    p1, p2 = part(0, T1), part(T1, w.T)
    o1, S_mid = gdr.gdr_forward_chunked(form, p1["q"], p1["k"], p1["v"], p1["log_w"], p1["e1"],
                                        p1["e2"], S0, chunk=64, algo=algo)
    S_resume = torch.full_like(S_mid, float("nan"))
    gdr.gdr_state_init(S_resume, S_mid)
    o2, S_T = gdr.gdr_forward_chunked(form, p2["q"], p2["k"], p2["v"], p2["log_w"], p2["e1"],
                                      p2["e2"], S_resume, chunk=64, algo=algo)
    torch.cuda.synchronize()
    assert np.array_equal(S_resume.cpu().numpy(), S_mid.cpu().numpy())
    o = torch.cat([o1, o2], dim=1).cpu().numpy()
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o, o_ref, (0, 2), TOL["bf16"], f"resume {form} {algo}: o")
    check_parity(S_T.cpu().numpy(), S_ref, (0, 1), TOL["bf16"], f"resume {form} {algo}: S_T")
