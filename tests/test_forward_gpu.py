"""GPU parity of gdr_forward_chunked against the fp64 oracle, plus internal
consistency (chunk-size invariance, split-sequence resume, decode x T)."""
import numpy as np
import pytest
import torch

import oracle
from matrix_memory_rnn_b200 import gdr, synth
from parity import (TOL, TOL_FP32_KERNEL, check_parity, gpu_forward, head_rel_err, oracle_forward,
                    small)

pytestmark = pytest.mark.gpu

FORMS = ["gdn2", "rwkv7", "general", "gla"]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,chunk,T", [(64, 64, 32, 100), (128, 128, 64, 77),
                                           (32, 128, 16, 50), (128, 16, 128, 300),
                                           (16, 32, 64, 1)])
def test_fp32_kernel_small(form, dtype, dk, dv, chunk, T):
    w = small(form, dtype, dk=dk, dv=dv, T=T, chunk=chunk)
    inp = synth.forward_inputs(w)
    inp["S0"] = synth.round_f32(np.random.default_rng(5).normal(0, 0.3, (w.B, w.H, dk, dv)))
    o, S = gpu_forward(w, inp, algo="fp32")
    o_ref, S_ref = oracle_forward(w, inp)
    assert head_rel_err(o, o_ref, (0, 2)) < TOL_FP32_KERNEL
    assert head_rel_err(S, S_ref, (0, 1)) < TOL_FP32_KERNEL


@pytest.mark.parametrize("name", ["rwkv7_f32", "gdn2_bf16", "rwkv7_bf16", "gdn2_long"])
def test_preset_full_size(name):
    w = synth.PRESETS[name]
    inp = synth.forward_inputs(w)
    o, S = gpu_forward(w, inp, algo="auto")
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o, o_ref, (0, 2), TOL[w.dtype], f"{name} o")
    check_parity(S, S_ref, (0, 1), TOL[w.dtype], f"{name} S_T")


def test_zero_tokens_copies_state():
    w = small("gdn2", "bf16", T=0)
    inp = synth.forward_inputs(w.with_(T=1))
    S0 = np.random.default_rng(3).normal(0, 1, (w.B, w.H, w.dk, w.dv)).astype(np.float32)
    d = gdr.to_device({k: inp[k][:, :0] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    s0 = torch.from_numpy(S0).cuda()
    o, S_T = gdr.gdr_forward_chunked("gdn2", d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                     d["e2"], s0, chunk=64)
    torch.cuda.synchronize()
    assert o.numel() == 0 and np.array_equal(S_T.cpu().numpy(), S0)


@pytest.mark.parametrize("algo", ["fp32", "auto"])
def test_state_alias_and_resume(algo):
    """S_T may alias S0; running [0, T1) then [T1, T) from its state equals [0, T)."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=192, chunk=64)
    inp = synth.forward_inputs(w)
    o_full, S_full = gpu_forward(w, inp, algo=algo)
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    S = torch.zeros((w.B, w.H, w.dk, w.dv), device="cuda")
    outs = []
    for lo, hi in ((0, 70), (70, 192)):
        part = {k: None if d[k] is None else d[k][:, lo:hi].contiguous() for k in d}
        o, _ = gdr.gdr_forward_chunked("gdn2", part["q"], part["k"], part["v"], part["log_w"],
                                       part["e1"], part["e2"], S, S_T=S, chunk=64, algo=algo)
        outs.append(o)
    torch.cuda.synchronize()
    o_split = torch.cat(outs, dim=1).cpu().numpy()
    tol = TOL_FP32_KERNEL if algo == "fp32" else 1e-2
    assert head_rel_err(o_split, o_full, (0, 2)) < tol
    assert head_rel_err(S.cpu().numpy(), S_full, (0, 1)) < tol


@pytest.mark.parametrize("algo", ["fp32", "auto"])
def test_chunk_size_invariance(algo):
    w = small("rwkv7", "bf16", dk=64, dv=64, T=256)
    inp = synth.forward_inputs(w)
    res = [gpu_forward(w, inp, algo=algo, chunk=c) for c in (16, 32, 64, 128)]
    tol = TOL_FP32_KERNEL if algo == "fp32" else 1e-2
    for o, S in res[1:]:
        assert head_rel_err(o, res[0][0], (0, 2)) < tol
        assert head_rel_err(S, res[0][1], (0, 1)) < tol


def test_decode_steps_equal_chunked_forward():
    w = small("rwkv7", "f32", dk=64, dv=64, T=40, chunk=16)
    inp = synth.forward_inputs(w)
    o_ref, S_ref = gpu_forward(w, inp, algo="fp32")
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "f32")
    S = torch.zeros((w.B, w.H, w.dk, w.dv), device="cuda")
    outs = []
    for t in range(w.T):
        tok = {k: d[k][:, t].contiguous() for k in d}
        outs.append(gdr.gdr_decode_step("rwkv7", tok["q"], tok["k"], tok["v"], tok["log_w"],
                                        tok["e1"], tok["e2"], S).clone())
    torch.cuda.synchronize()
    o_dec = torch.stack(outs, dim=1).cpu().numpy()
    assert head_rel_err(o_dec, o_ref, (0, 2)) < 1e-4
    assert head_rel_err(S.cpu().numpy(), S_ref, (0, 1)) < 1e-4


def test_eviction_on_gpu():
    """Targeted removal evicts (k_A, v_A) as (1 - c)^T ("Exponential gates ...", 13.3)."""
    d, T, c = 64, 30, 0.1
    rng = np.random.default_rng(4)
    kA = rng.standard_normal(d); kA /= np.linalg.norm(kA)
    vA = rng.standard_normal(d)
    P = np.eye(d) - np.outer(kA, kA)
    n = T + 1
    q = np.ones((1, n, 1, d)); k = np.zeros((1, n, 1, d)); v = np.zeros((1, n, 1, d))
    a = np.zeros((1, n, 1, d)); cc = np.zeros((1, n, 1))
    k[0, 0, 0], v[0, 0, 0], a[0, 0, 0] = kA, vA, kA
    for t in range(1, n):
        b = P @ rng.standard_normal(d); b /= np.linalg.norm(b)
        k[0, t, 0], v[0, t, 0], a[0, t, 0], cc[0, t, 0] = b, rng.standard_normal(d), kA, c
    f = lambda x: torch.tensor(x, dtype=torch.float32, device="cuda").contiguous()
    _, S_T = gdr.gdr_forward_chunked("rwkv7", f(q), f(k), f(v), f(np.zeros((1, n, 1, d))),
                                     f(a), f(cc), None, chunk=16, algo="fp32")
    torch.cuda.synchronize()
    St = S_T[0, 0].double().cpu().numpy()
    kA32 = np.asarray(f(kA).cpu().numpy(), np.float64)
    vA32 = np.asarray(f(vA).cpu().numpy(), np.float64)
    ratio = np.linalg.norm(St.T @ kA32) / np.linalg.norm(vA32)
    assert abs(ratio - (1 - c) ** T) < 1e-5


# the two tensor-core paths: "split" (prep + chain kernels, full workspace) and
# "fused" (one kernel, the 256-byte minimum workspace)
TC_PATHS = {"split": None, "fused": 256}


@pytest.mark.parametrize("path", sorted(TC_PATHS))
@pytest.mark.parametrize("T", [1, 64, 100, 257])
@pytest.mark.parametrize("with_state", [False, True])
def test_tc_kernel_gdn2(T, with_state, path):
    """Tensor-core kernels (GDN-2, bf16, d = 128, C = 64) against the oracle, with a ragged tail."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=T, B=2, H=3, chunk=64)
    inp = synth.forward_inputs(w)
    if with_state:
        inp["S0"] = synth.round_f32(np.random.default_rng(7).normal(0, 0.5, (w.B, w.H, 128, 128)))
    o, S = gpu_forward(w, inp, algo="tc", workspace_bytes=TC_PATHS[path])
    o_ref, S_ref = oracle_forward(w, inp)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"tc-{path} T={T} S0={with_state}: o {eo:.3e} S {es:.3e}")
    assert eo < TOL["bf16"] and es < TOL["bf16"]


@pytest.mark.parametrize("path", sorted(TC_PATHS))
def test_tc_kernel_serves_chunk_128(path):
    """A requested chunk of 128 runs on the tensor-core kernels as two 64-token chunks."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=300, B=1, H=2, chunk=128)
    inp = synth.forward_inputs(w)
    o, S = gpu_forward(w, inp, algo="tc", workspace_bytes=TC_PATHS[path])
    o_ref, S_ref = oracle_forward(w, inp)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    assert eo < TOL["bf16"] and es < TOL["bf16"]
    o64, S64 = gpu_forward(w.with_(chunk=64), inp, algo="tc", workspace_bytes=TC_PATHS[path])
    assert np.array_equal(o, o64) and np.array_equal(S, S64)


@pytest.mark.parametrize("path", sorted(TC_PATHS))
def test_tc_full_size_gdn2(path):
    w = synth.PRESETS["gdn2_bf16"]
    inp = synth.forward_inputs(w)
    o, S = gpu_forward(w, inp, algo="tc", workspace_bytes=TC_PATHS[path])
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o, o_ref, (0, 2), TOL["bf16"], f"tc-{path} gdn2_bf16 o")
    check_parity(S, S_ref, (0, 1), TOL["bf16"], f"tc-{path} gdn2_bf16 S_T")


@pytest.mark.parametrize("form,H", [("gdn2", 2), ("gla", 2), ("gdn2", 20)])
def test_tc_long_sequences_one_launch(form, H):
    """Few long sequences (here 2 or 20 heads x 41 chunks): prep and chain CTAs share one
    cooperative launch, the chain CTAs fetching each record once a prep CTA has published
    it.  Two heads run 32-column value slices (8 chains), twenty heads 64-column slices
    (40 chains: 32-column ones would take more than half the SMs).  Against the oracle,
    with a ragged tail and an initial state; bit-identical on a second call."""
    w = small(form, "bf16", dk=128, dv=128, T=64 * 40 + 17, B=1, H=H, chunk=64)
    inp = synth.forward_inputs(w)
    inp["S0"] = synth.round_f32(np.random.default_rng(12).normal(0, 0.5, (w.B, w.H, 128, 128)))
    o, S = gpu_forward(w, inp, algo="tc")
    o_ref, S_ref = oracle_forward(w, inp)
    check_parity(o, o_ref, (0, 2), TOL["bf16"], f"one launch {form} o")
    check_parity(S, S_ref, (0, 1), TOL["bf16"], f"one launch {form} S_T")
    o2, S2 = gpu_forward(w, inp, algo="tc")
    assert np.array_equal(o, o2) and np.array_equal(S, S2)


@pytest.mark.parametrize("path", sorted(TC_PATHS))
def test_tc_kernel_strong_decay_uses_exact_path(path):
    """Channels whose decay over a chunk exceeds e^-80 take the exact pairwise path."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=200, B=1, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    lw = inp["log_w"].copy()
    lw[:, :, :, ::7] = -3.0          # 64 tokens x 3 nats = 192 nats per chunk on these channels
    lw[:, 70:80, 1, 5] = -60.0       # a burst of very strong decay on one head
    inp["log_w"] = lw.astype(np.float32)
    o, S = gpu_forward(w, inp, algo="tc", workspace_bytes=TC_PATHS[path])
    o_ref, S_ref = oracle_forward(w, inp)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"tc strong decay: o {eo:.3e} S {es:.3e}")
    assert np.isfinite(o).all() and np.isfinite(S).all()
    assert eo < TOL["bf16"] and es < TOL["bf16"]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("T", [1, 64, 100, 257])
@pytest.mark.parametrize("with_state", [False, True])
def test_tc_general_kernel(form, T, with_state):
    """Two-stream tensor-core kernel (every form, bf16, d = 64, C = 64) against the oracle."""
    w = small(form, "bf16", dk=64, dv=64, T=T, B=2, H=3, chunk=64)
    inp = synth.forward_inputs(w)
    if with_state:
        inp["S0"] = synth.round_f32(np.random.default_rng(8).normal(0, 0.5, (w.B, w.H, 64, 64)))
    o, S = gpu_forward(w, inp, algo="tc")
    o_ref, S_ref = oracle_forward(w, inp)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"tc-general {form} T={T} S0={with_state}: o {eo:.3e} S {es:.3e}")
    assert eo < TOL["bf16"] and es < TOL["bf16"]


def test_tc_general_gdn2_without_write_gate():
    """GDN-2 with no write gate (written value v) on the two-stream kernel."""
    w = small("gdn2", "bf16", dk=64, dv=64, T=150, B=2, H=3, chunk=64)
    inp = synth.forward_inputs(w)
    inp["e2"] = None
    o, S = gpu_forward(w, inp, algo="tc")
    o_ref, S_ref = oracle_forward(w, inp)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    assert eo < TOL["bf16"] and es < TOL["bf16"]


@pytest.mark.parametrize("form", FORMS)
def test_tc_general_strong_decay_uses_exact_path(form):
    """Channels whose decay over a chunk exceeds e^-80 take the exact pairwise path."""
    w = small(form, "bf16", dk=64, dv=64, T=200, B=1, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    lw = inp["log_w"].copy()
    lw[:, :, :, ::7] = -3.0
    lw[:, 70:80, 1, 5] = -60.0
    inp["log_w"] = lw.astype(np.float32)
    o, S = gpu_forward(w, inp, algo="tc")
    o_ref, S_ref = oracle_forward(w, inp)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"tc-general strong decay {form}: o {eo:.3e} S {es:.3e}")
    assert np.isfinite(o).all() and np.isfinite(S).all()
    assert eo < TOL["bf16"] and es < TOL["bf16"]


@pytest.mark.parametrize("T", [1, 100, 257])
@pytest.mark.parametrize("with_state", [False, True])
def test_tc_split_gla(T, with_state):
    """GLA at d = 128 on the prep + chain kernels (GDN-2's chunk algebra with b = 0)."""
    w = small("gla", "bf16", dk=128, dv=128, T=T, B=2, H=3, chunk=64)
    inp = synth.forward_inputs(w)
    if with_state:
        inp["S0"] = synth.round_f32(np.random.default_rng(9).normal(0, 0.5, (w.B, w.H, 128, 128)))
    o, S = gpu_forward(w, inp, algo="tc")
    o_ref, S_ref = oracle_forward(w, inp)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"tc-split gla T={T} S0={with_state}: o {eo:.3e} S {es:.3e}")
    assert eo < TOL["bf16"] and es < TOL["bf16"]


def test_tc_split_gla_strong_decay_and_small_workspace():
    """GLA at d = 128: the exact pairwise path, and without the record workspace algo=tc
    reports GDR_ERR_WORKSPACE while algo=auto takes the fp32 kernel."""
    w = small("gla", "bf16", dk=128, dv=128, T=200, B=1, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    lw = inp["log_w"].copy()
    lw[:, :, :, ::7] = -3.0
    lw[:, 70:80, 1, 5] = -60.0
    inp["log_w"] = lw.astype(np.float32)
    o_ref, S_ref = oracle_forward(w, inp)
    o, S = gpu_forward(w, inp, algo="tc")
    assert head_rel_err(o, o_ref, (0, 2)) < TOL["bf16"]
    assert head_rel_err(S, S_ref, (0, 1)) < TOL["bf16"]
    with pytest.raises(gdr.GdrError) as ei:
        gpu_forward(w, inp, algo="tc", workspace_bytes=256)
    assert ei.value.code == 7
    o, S = gpu_forward(w, inp, algo="auto", workspace_bytes=256)
    assert head_rel_err(o, o_ref, (0, 2)) < TOL["bf16"]
    assert head_rel_err(S, S_ref, (0, 1)) < TOL["bf16"]


@pytest.mark.parametrize("d,algo,ws", [(128, "auto", None), (128, "tc", 256), (64, "tc", None),
                                       (64, "fp32", None)])
def test_deltanet_through_gdn2_form(d, algo, ws):
    """Plain DeltaNet (no decay, u = beta k, z = k, write beta v k^T) is the GDN-2 form with
    log w = 0 and the erase and write gates both set to the per-token strength beta.  The
    oracle runs it in the general form with that mapping written out in fp64."""
    B, T, H = 2, 200, 2
    rng = np.random.default_rng(21)
    q = synth.round_bf16(rng.standard_normal((B, T, H, d)))
    kk = rng.standard_normal((B, T, H, d))
    k = synth.round_bf16(kk / np.linalg.norm(kk, axis=-1, keepdims=True))
    v = synth.round_bf16(rng.standard_normal((B, T, H, d)))
    beta = synth.round_bf16(1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, 1)))))
    gate = np.broadcast_to(beta, (B, T, H, d)).copy()
    log_w = np.zeros((B, T, H, d), np.float32)
    dev = gdr.to_device(dict(q=q, k=k, v=v, log_w=log_w, e1=gate, e2=gate), "bf16")
    o, S_T = gdr.gdr_forward_chunked("gdn2", dev["q"], dev["k"], dev["v"], dev["log_w"],
                                     dev["e1"], dev["e2"], None, chunk=64, algo=algo,
                                     workspace=None if ws is None else gdr.new_workspace(ws, "cuda"))
    torch.cuda.synchronize()
    b64, k64 = beta.astype(np.float64), k.astype(np.float64)
    o_ref, S_ref = oracle.forward("general", q, k, b64 * v, log_w, b64 * k64, k, None)
    eo = head_rel_err(o.cpu().numpy(), o_ref, (0, 2))
    es = head_rel_err(S_T.cpu().numpy(), S_ref, (0, 1))
    print(f"deltanet d={d} {algo}: o {eo:.3e} S {es:.3e}")
    assert eo < TOL["bf16"] and es < TOL["bf16"]


@pytest.mark.parametrize("form,d,algo", [("gdn2", 128, "auto"), ("gdn2", 128, "fp32"),
                                         ("rwkv7", 64, "auto"), ("rwkv7", 64, "fp32")])
def test_zero_erase_reduces_to_gla(form, d, algo):
    """With the erase strength at zero (GDN-2 b = 0, RWKV-7 c = 0) the recurrence is gated
    linear attention: the oracle's GLA form on the same decays, with GDN-2's write gate
    folded into v in fp64."""
    w = small(form, "bf16", dk=d, dv=d, T=150, B=2, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    inp["e1" if form == "gdn2" else "e2"] = np.zeros_like(inp["e1" if form == "gdn2" else "e2"])
    o, S = gpu_forward(w, inp, algo=algo)
    v = inp["v"].astype(np.float64) * (inp["e2"] if form == "gdn2" else 1.0)
    o_ref, S_ref = oracle.forward("gla", inp["q"], inp["k"], v, inp["log_w"], None, None, None)
    eo, es = head_rel_err(o, o_ref, (0, 2)), head_rel_err(S, S_ref, (0, 1))
    print(f"zero erase {form} {algo}: o {eo:.3e} S {es:.3e}")
    assert eo < TOL["bf16"] and es < TOL["bf16"]


def test_tc_rejects_what_it_does_not_cover():
    w = small("rwkv7", "bf16", dk=32, dv=32, T=64, B=1, H=1, chunk=64)
    inp = synth.forward_inputs(w)
    with pytest.raises(gdr.GdrError) as ei:
        gpu_forward(w, inp, algo="tc")
    assert ei.value.code == 2


def test_bounded_wait_reports_timeout_and_context_survives(monkeypatch):
    """Fault injection on the host: the prep kernel's front group withholds its hand-off,
    the back group's bounded wait runs out, the call reports GDR_ERR_TIMEOUT through the
    workspace status word, and the next call on the same context is correct."""
    w = small("gdn2", "bf16", dk=128, dv=128, T=192, B=1, H=2, chunk=64)
    inp = synth.forward_inputs(w)
    d = gdr.to_device({k: inp[k] for k in ("q", "k", "v", "log_w", "e1", "e2")}, "bf16")
    ws = gdr.new_workspace(gdr.gdr_forward_workspace_size(w.form, d["q"], d["k"], d["v"],
                                                          d["log_w"], d["e1"], d["e2"], 64,
                                                          "tc"), "cuda")
    monkeypatch.setenv("GDR_DEBUG_FAULT", "skip_handoff")
    gdr.gdr_forward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"], d["e2"],
                            None, chunk=64, algo="tc", workspace=ws)
    assert gdr.gdr_read_status(ws) == "GDR_ERR_TIMEOUT"
    monkeypatch.delenv("GDR_DEBUG_FAULT")
    o, S = gdr.gdr_forward_chunked(w.form, d["q"], d["k"], d["v"], d["log_w"], d["e1"],
                                   d["e2"], None, chunk=64, algo="tc", workspace=ws)
    assert gdr.gdr_read_status(ws) == "GDR_OK"
    o_ref, S_ref = oracle_forward(w, inp)
    assert head_rel_err(o.cpu().numpy(), o_ref, (0, 2)) < TOL["bf16"]
    assert head_rel_err(S.cpu().numpy(), S_ref, (0, 1)) < TOL["bf16"]
