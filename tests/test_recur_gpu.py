"""GPU parity of the token-recurrent forward kernel (algo "recurrent"; also what algo "auto"
takes when the fp32 chunkwise kernel would leave SMs idle) against the fp64 oracle.  The
kernel computes in fp32 from the inputs as given, so bf16 inputs are held to the fp32 bar
too: the oracle sees the same bf16-rounded values."""
import numpy as np
import pytest

from matrix_memory_rnn_b200 import synth
from parity import TOL_FP32_KERNEL, check_parity, gpu_forward, oracle_forward, small

pytestmark = pytest.mark.gpu

FORMS = ["gdn2", "rwkv7", "general", "gla"]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 64), (128, 128), (128, 32), (64, 16)])
@pytest.mark.parametrize("T", [1, 9, 130])
def test_recurrent_parity(form, dtype, dk, dv, T):
    """Every form, both dtypes, every key width (d_k = 16 leaves half the lanes idle), value
    widths of two to sixteen eight-column CTAs, and token counts below, across and past the
    eight-token staging block, from a nonzero initial state."""
    w = small(form, dtype, dk=dk, dv=dv, T=T, B=2, H=2, chunk=64, seed=31 + T)
    inp = synth.forward_inputs(w)
    inp["S0"] = synth.round_f32(np.random.default_rng(T).normal(0.0, 0.5, (w.B, w.H, dk, dv)))
    o, S = gpu_forward(w, inp, algo="recurrent")
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o, o_ref, (0, 2), TOL_FP32_KERNEL, f"recurrent {form} {dtype} {dk}x{dv} T={T} o")
    check_parity(S, S_ref, (0, 1), TOL_FP32_KERNEL, f"recurrent {form} {dtype} {dk}x{dv} T={T} S")


def test_recurrent_resume():
    """Two calls with the state passed between them equal one call."""
    w = small("rwkv7", "f32", dk=64, dv=64, T=200, B=1, H=2, chunk=64, seed=5)
    inp = synth.forward_inputs(w)
    o_full, S_full = gpu_forward(w, inp, algo="recurrent")
    a = {k: (x[:, :77] if x is not None and x.ndim >= 3 else x) for k, x in inp.items()}
    b = {k: (x[:, 77:] if x is not None and x.ndim >= 3 else x) for k, x in inp.items()}
    o1, S1 = gpu_forward(w.with_(T=77), a, algo="recurrent")
    o2, S2 = gpu_forward(w.with_(T=123), b, algo="recurrent", S0=S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o_full, rtol=0, atol=1e-5)
    np.testing.assert_allclose(S2, S_full, rtol=0, atol=1e-5)


def test_small_rwkv7_fp32_workload_full_size():
    """The five-config suite's small fp32 case (RWKV-7, B=1, H=2, T=256, d=64) at its full
    size through algo auto, which takes the token-recurrent kernel for it."""
    w = synth.PRESETS["rwkv7_f32"]
    inp = synth.forward_inputs(w)
    o, S = gpu_forward(w, inp, algo="auto")
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o, o_ref, (0, 2), TOL_FP32_KERNEL, "rwkv7_f32 auto o")
    check_parity(S, S_ref, (0, 1), TOL_FP32_KERNEL, "rwkv7_f32 auto S")


@pytest.mark.parametrize("form", FORMS)
def test_recurrent_long_d128(form):
    """d_k = d_v = 128 over 1001 tokens (125 staging blocks and a one-token tail), fp32 inputs
    through algo auto, from a nonzero state: the per-step rounding of the fp32 state stays
    at the fp32 bar over the whole sequence."""
    w = small(form, "f32", dk=128, dv=128, T=1001, B=1, H=3, chunk=64, seed=77)
    inp = synth.forward_inputs(w)
    inp["S0"] = synth.round_f32(np.random.default_rng(5).normal(0.0, 0.5, (w.B, w.H, 128, 128)))
    o, S = gpu_forward(w, inp, algo="auto")
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o, o_ref, (0, 2), TOL_FP32_KERNEL, f"recurrent long {form} o")
    check_parity(S, S_ref, (0, 1), TOL_FP32_KERNEL, f"recurrent long {form} S")
