"""The entry point for callers that cannot allocate device memory.

Some callers (a plugin whose host application owns every device allocation, a
serving loop that forbids allocation once its memory plan is fixed) cannot hand
libgdr a workspace.  gdr_forward_chunked_noalloc takes its scratch from a fixed
array inside the library instead.  This checks, through the C ABI, that two
calls in a row give what the allocating entry point gives.  The file is named to
be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from matrix_memory_rnn_b200 import gdr, synth
from parity import TOL, head_rel_err, small

pytestmark = pytest.mark.gpu


def test_noalloc_entry_point_matches_allocating_one():
    lib = gdr.library()
    fn = lib.gdr_forward_chunked_noalloc
    fn.argtypes = [ctypes.POINTER(gdr.gdr_fwd_args), ctypes.c_void_p]
    fn.restype = ctypes.c_int

    w = small("gdn2", "bf16", dk=128, dv=128, T=200, B=2, H=3, chunk=64)
    inp = synth.forward_inputs(w)
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    S0 = torch.from_numpy(synth.round_f32(
        np.random.default_rng(9).normal(0, 0.5, (w.B, w.H, w.dk, w.dv)))).cuda()
    args = (w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"], S0)

    o_ref, S_ref = gdr.gdr_forward_chunked(*args, chunk=64, algo="tc")
    torch.cuda.synchronize()
    o_ref, S_ref = o_ref.cpu().numpy(), S_ref.cpu().numpy()

    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full((w.B, w.T, w.H, w.dv), float("nan"), device="cuda")
        S_T = torch.full((w.B, w.H, w.dk, w.dv), float("nan"), device="cuda")
        a = gdr._fwd_struct(*args, o, S_T, 64, "tc", None)
        assert a.workspace is None
        rc = fn(ctypes.byref(a), stream)
        assert rc == 0, f"call {call}: status {gdr.STATUS.get(rc, rc)}"
        torch.cuda.synchronize()
        o_np, S_np = o.cpu().numpy(), S_T.cpu().numpy()
        assert np.isfinite(o_np).all() and np.isfinite(S_np).all()
        assert head_rel_err(o_np, o_ref, (0, 2)) < TOL["bf16"]
        assert head_rel_err(S_np, S_ref, (0, 1)) < TOL["bf16"]
