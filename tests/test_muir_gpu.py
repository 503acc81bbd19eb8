"""GPU parity of gdr_muir_forward (the Muir token mixer around the GDN-2 recurrence)
against the fp64 oracle's mixer on the same seeded pre-activations and gate logits.
Error norm and bars as the forward: per head, y over its T x d_v block and S_T."""
import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth
from parity import TOL, check_parity, head_rel_err, small

pytestmark = pytest.mark.gpu

TOKEN = ("q", "k", "v", "zf", "zb", "zw", "zq", "zg")
# Elementwise bar of the mixer's outputs.  (1) The readout y_t = rho (.) o_t / RMS(o_t) (.)
# SiLU(z_g) normalizes each token: an error of o_t that scales with the head's output level R
# (the bf16 rounding of the state's contribution) becomes an error of y_t scaled by
# R / RMS(o_t), large for the few tokens whose output nearly cancels.  (2) The mixer's erase
# gate b = 2 sigmoid(z_b) reaches 2, so the transition (I - k (b (.) k)^T) Diag(alpha) has an
# eigenvalue near -1 along the current key: rounding errors along such directions are hardly
# damped and gather in a few state entries over long sequences (about 0.12 elementwise on S_T
# after 2300 tokens, with 3e-3 to 5e-3 Frobenius, for the fused path and for the separate
# prologue with accurate activations alike).  A token or state entry that is wrong is off by
# about 1 RMS, so 0.5 still separates it from these.
Y_ELEM_TOL = 0.5


def _run(w, inp, S0=None, algo="auto", workspace_bytes=None, unfused=False):
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    d = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to("cuda", tdt) for k in TOKEN}
    f32 = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    ws = None if workspace_bytes is None else gdr.new_workspace(workspace_bytes, "cuda")
    y, S_T = gdr.gdr_muir_forward(*(d[k] for k in TOKEN), f32(inp["a_log"]), f32(inp["gamma_stat"]),
                                  f32(inp["rms_weight"]), 1e-6, f32(S0), chunk=w.chunk, algo=algo,
                                  unfused=unfused, workspace=ws)
    torch.cuda.synchronize()
    return y.cpu().numpy(), S_T.cpu().numpy()


def _ref(inp, S0=None, sl=None):
    pick = (lambda a: a) if sl is None else sl
    return oracle.muir_forward(*(pick(inp[k]) for k in TOKEN), inp["a_log"], inp["gamma_stat"],
                               inp["rms_weight"], 1e-6, S0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 100, 257])
@pytest.mark.parametrize("with_state", [False, True])
def test_muir_parity(dtype, dk, dv, T, with_state):
    w = small("gdn2", dtype, dk=dk, dv=dv, T=T, B=2, H=3, chunk=64)
    inp = synth.muir_inputs(w, static_gains=with_state)
    S0 = (synth.round_f32(np.random.default_rng(12).normal(0, 0.5, (w.B, w.H, dk, dv)))
          if with_state else None)
    y, S = _run(w, inp, S0)
    y_ref, S_ref = _ref(inp, S0)
    ey, es = head_rel_err(y, y_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"muir {dtype} {dk}x{dv} T={T} S0={with_state}: y {ey:.2e} S {es:.2e}")
    assert np.isfinite(y).all()
    assert ey < TOL[dtype] and es < TOL[dtype]


def test_muir_full_size_sampled_heads():
    w = synth.PRESETS["gdn2_bf16"]
    inp = synth.muir_inputs(w)
    y, S = _run(w, inp)
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sl = lambda a: a[b:b + 1, :, h:h + 1]
        sub = dict(inp, a_log=inp["a_log"][h:h + 1], gamma_stat=inp["gamma_stat"][h:h + 1])
        y_ref, S_ref = _ref(sub, None, sl)
        check_parity(y[b:b + 1, :, h:h + 1], y_ref, (0, 2), TOL["bf16"], f"muir full size ({b},{h}) y",
                     elem_tol=Y_ELEM_TOL)
        check_parity(S[b:b + 1, h:h + 1], S_ref, (0, 1), TOL["bf16"], f"muir full size ({b},{h}) S_T",
                     elem_tol=Y_ELEM_TOL)


def test_muir_zero_length():
    w = small("gdn2", "bf16", dk=64, dv=64, T=0, B=1, H=2, chunk=64)
    inp = synth.muir_inputs(w)
    S0 = np.random.default_rng(1).standard_normal((1, 2, 64, 64)).astype(np.float32)
    y, S = _run(w, inp, S0)
    assert y.shape == (1, 0, 2, 64) and np.array_equal(S, S0)


def test_muir_fused_strong_decay_uses_exact_path():
    """bf16, d = 128 runs the mixer inside the tensor-core forward; decay logits that make
    some channels decay by more than 80 nats per chunk take its exact pairwise path."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=150, B=1, H=2, chunk=64)
    inp = synth.muir_inputs(w)
    zf = inp["zf"].copy()
    zf[:, :, :, ::9] = 6.0          # softplus ~ 6: log alpha ~ -6 exp(a_log) per token
    inp["zf"] = synth.round_bf16(zf)
    inp["a_log"] = np.full(w.H, np.log(4.0), np.float32)
    y, S = _run(w, inp)
    y_ref, S_ref = _ref(inp)
    ey, es = head_rel_err(y, y_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"muir fused strong decay: y {ey:.2e} S {es:.2e}")
    assert np.isfinite(y).all() and ey < TOL["bf16"] and es < TOL["bf16"]


def test_muir_fused_against_unfused():
    """The fused path (activations inside the forward) and the unfused one (prologue
    kernel, fp32 forward, epilogue) on the same inputs."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=200, B=2, H=2, chunk=64)
    inp = synth.muir_inputs(w)
    y_f, S_f = _run(w, inp, algo="auto")
    y_u, S_u = _run(w, inp, algo="fp32")
    assert head_rel_err(y_f, y_u, (0, 2)) < TOL["bf16"]
    assert head_rel_err(S_f, S_u, (0, 1)) < TOL["bf16"]


@pytest.mark.parametrize("unfused", [False, True])
def test_muir_bf16_d128_both_paths(unfused):
    """bf16, d = 128: the fused path and the separate prologue (both on the tensor-core
    forward) against the oracle, with a ragged tail and an initial state."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=333, B=2, H=3, chunk=64)
    inp = synth.muir_inputs(w)
    S0 = synth.round_f32(np.random.default_rng(13).normal(0, 0.5, (w.B, w.H, 128, 128)))
    y, S = _run(w, inp, S0, unfused=unfused)
    y_ref, S_ref = _ref(inp, S0)
    assert head_rel_err(y, y_ref, (0, 2)) < TOL["bf16"]
    assert head_rel_err(S, S_ref, (0, 1)) < TOL["bf16"]


def test_muir_long_sequence_one_launch():
    """A few long sequences run the fused mixer as one cooperative launch (prep CTAs with
    the activations publish records that chain CTAs consume): against the oracle."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=64 * 36 + 5, B=1, H=2, chunk=64)
    inp = synth.muir_inputs(w)
    S0 = synth.round_f32(np.random.default_rng(14).normal(0, 0.5, (w.B, w.H, 128, 128)))
    y, S = _run(w, inp, S0)
    y_ref, S_ref = _ref(inp, S0)
    check_parity(y, y_ref, (0, 2), TOL["bf16"], "muir one launch y", elem_tol=Y_ELEM_TOL)
    check_parity(S, S_ref, (0, 1), TOL["bf16"], "muir one launch S_T", elem_tol=Y_ELEM_TOL)
    # the separate prologue (accurate activations) on the same sequence
    y_u, S_u = _run(w, inp, S0, unfused=True)
    check_parity(y_u, y_ref, (0, 2), TOL["bf16"], "muir unfused, long y", elem_tol=Y_ELEM_TOL)
    check_parity(S_u, S_ref, (0, 1), TOL["bf16"], "muir unfused, long S_T", elem_tol=Y_ELEM_TOL)
