"""The entry point for callers that cannot allocate device memory.

Some callers (a plugin whose host application owns every device allocation, a
serving loop that forbids allocation once its memory plan is fixed) cannot hand
libgdr a workspace.  gdr_forward_chunked_noalloc takes its scratch from a fixed
array inside the library instead.  This checks, through the C ABI, that two
calls in a row give what the allocating entry point gives on the same kernel, and
what the oracle gives, for each kernel the call can take; and that a case it cannot
serve is refused before anything is enqueued.  The file is named to be collected
last.
"""
import ctypes

import numpy as np
import pytest
import torch

from matrix_memory_rnn_b200 import gdr, synth
from parity import TOL, head_rel_err, oracle_forward, small

pytestmark = pytest.mark.gpu

GDR_ERR_WORKSPACE = 7


def _noalloc():
    fn = gdr.library().gdr_forward_chunked_noalloc
    fn.argtypes = [ctypes.POINTER(gdr.gdr_fwd_args), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _case(form, d, seed=9):
    w = small(form, "bf16", dk=d, dv=d, T=200, B=2, H=3, chunk=64)
    inp = synth.forward_inputs(w)
    inp["S0"] = synth.round_f32(np.random.default_rng(seed).normal(0, 0.5, (w.B, w.H, d, d)))
    dev = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    S0 = torch.from_numpy(inp["S0"]).cuda()
    return w, inp, (w.form, dev["q"], dev["k"], dev["v"], dev["log_w"], dev["e1"], dev["e2"], S0)


# (form, d, algo, the allocating call's workspace that selects the same kernel):
#   GDN-2 d = 128: the single-kernel tensor-core forward (status word only, 256 bytes)
#   RWKV-7 d = 64: the two-stream tensor-core kernel
#   GLA d = 128 with algo auto: the token-recurrent kernel (the tensor-core path needs records)
#   GLA d = 128 with algo fp32: the fp32 chunkwise kernel
CASES = [("gdn2", 128, "tc", 256), ("rwkv7", 64, "auto", 256), ("gla", 128, "auto", 256),
         ("gla", 128, "fp32", 256)]


@pytest.mark.parametrize("form,d,algo,ws", CASES)
def test_noalloc_entry_point_matches_allocating_one(form, d, algo, ws):
    fn = _noalloc()
    w, inp, args = _case(form, d)
    o_ref, S_ref = gdr.gdr_forward_chunked(*args, chunk=64, algo=algo,
                                           workspace=gdr.new_workspace(ws, "cuda"))
    torch.cuda.synchronize()
    o_ref, S_ref = o_ref.cpu().numpy(), S_ref.cpu().numpy()
    o_or, S_or = oracle_forward(w, inp)

    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full((w.B, w.T, w.H, w.dv), float("nan"), device="cuda")
        S_T = torch.full((w.B, w.H, w.dk, w.dv), float("nan"), device="cuda")
        a = gdr._fwd_struct(*args, o, S_T, 64, algo, None)
        assert a.workspace is None
        rc = fn(ctypes.byref(a), stream)
        assert rc == 0, f"call {call}: status {gdr.STATUS.get(rc, rc)}"
        torch.cuda.synchronize()
        o_np, S_np = o.cpu().numpy(), S_T.cpu().numpy()
        assert np.isfinite(o_np).all() and np.isfinite(S_np).all()
        assert head_rel_err(o_np, o_ref, (0, 2)) < TOL["bf16"]
        assert head_rel_err(S_np, S_ref, (0, 1)) < TOL["bf16"]
        assert head_rel_err(o_np, o_or, (0, 2)) < TOL["bf16"]
        assert head_rel_err(S_np, S_or, (0, 1)) < TOL["bf16"]


def test_noalloc_refuses_what_needs_records():
    """GLA at d = 128 on the tensor cores needs per-chunk records the array cannot hold:
    GDR_ERR_WORKSPACE, and the outputs are left untouched (nothing was enqueued)."""
    fn = _noalloc()
    w, inp, args = _case("gla", 128)
    o = torch.full((w.B, w.T, w.H, w.dv), float("nan"), device="cuda")
    S_T = torch.full((w.B, w.H, w.dk, w.dv), float("nan"), device="cuda")
    a = gdr._fwd_struct(*args, o, S_T, 64, "tc", None)
    rc = fn(ctypes.byref(a), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == GDR_ERR_WORKSPACE
    assert torch.isnan(o).all() and torch.isnan(S_T).all()


def test_noalloc_reports_a_timeout_through_its_status_reader(monkeypatch):
    """Fault injection on the host: the single-kernel forward withholds the commit of its
    first product, its bounded wait runs out, and gdr_noalloc_read_status returns
    GDR_ERR_TIMEOUT from the library's array (then GDR_OK: it clears the word).  The next
    call on the same context matches the oracle."""
    w, inp, args = _case("gdn2", 128)
    o = torch.empty((w.B, w.T, w.H, w.dv), device="cuda")
    S_T = torch.empty((w.B, w.H, w.dk, w.dv), device="cuda")
    assert gdr.gdr_noalloc_read_status() == "GDR_OK"
    monkeypatch.setenv("GDR_DEBUG_FAULT", "skip_handoff")
    gdr.gdr_forward_chunked_noalloc(*args, algo="tc", o=o, S_T=S_T)
    assert gdr.gdr_noalloc_read_status() == "GDR_ERR_TIMEOUT"
    assert gdr.gdr_noalloc_read_status() == "GDR_OK"
    monkeypatch.delenv("GDR_DEBUG_FAULT")
    gdr.gdr_forward_chunked_noalloc(*args, algo="tc", o=o, S_T=S_T)
    assert gdr.gdr_noalloc_read_status() == "GDR_OK"
    o_or, S_or = oracle_forward(w, inp)
    assert head_rel_err(o.cpu().numpy(), o_or, (0, 2)) < TOL["bf16"]
    assert head_rel_err(S_T.cpu().numpy(), S_or, (0, 1)) < TOL["bf16"]
