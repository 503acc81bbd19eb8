"""Host-only checks of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from matrix_memory_rnn_b200 import build as gbuild
from matrix_memory_rnn_b200 import gdr

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "gdr.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_]\w*\s*\*?\s*(gdr_\w+)\s*\(", src,
                                 flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gdr.library()


def test_header_declares_the_path_entry_points():
    names = declared_functions()
    for fn in ("gdr_forward_chunked", "gdr_decode_step", "gdr_state_init",
               "gdr_forward_workspace_size", "gdr_status_string"):
        assert fn in names


def test_every_declared_symbol_is_exported(lib):
    for fn in declared_functions():
        assert hasattr(lib, fn), f"{fn} declared in gdr.h but not exported"


def test_status_strings_and_version(lib):
    for code in range(8):
        s = lib.gdr_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.gdr_status_string(99) == b"unknown status"
    assert lib.gdr_version() >= 100


def _args(**kw):
    a = gdr.gdr_fwd_args()
    a.form, a.dtype, a.B, a.H, a.T, a.dk, a.dv, a.chunk = 1, 1, 1, 1, 8, 64, 64, 64
    fake = 0x10000
    a.q = a.k = a.v = a.log_w = a.e1 = a.o = ctypes.c_void_p(fake)
    for name, val in kw.items():
        setattr(a, name, val)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(chunk=24), 2), (dict(form=9), 1),
    (dict(dtype=5), 1), (dict(B=-1), 1), (dict(T=-3), 1), (dict(algo=7), 1),
    (dict(q=None), 1), (dict(e1=None), 1), (dict(o=None), 1),
    (dict(k=ctypes.c_void_p(0x10004)), 3), (dict(workspace=ctypes.c_void_p(0x10010)), 3),
])
def test_forward_rejects_bad_arguments_on_host(lib, kw, code):
    a = _args(**kw)
    assert lib.gdr_forward_chunked(ctypes.byref(a), None) == code


def _kernel_name(lib, a):
    name = ctypes.c_char_p()
    rc = lib.gdr_forward_kernel_name(ctypes.byref(a), ctypes.byref(name))
    return rc, (name.value.decode() if rc == 0 else None)


def _tc_split_bytes(lib, a):
    n = ctypes.c_size_t(0)
    assert lib.gdr_forward_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    return n.value


def test_forward_kernel_selection(lib):
    """The host-side plan of gdr_forward_chunked, as the name query reports it (no GPU)."""
    ws = ctypes.c_void_p(0x100000)
    # GDN-2 bf16 d = 128: two kernels with the record workspace, one kernel with the status
    # word only; fp32 inputs take the token recurrence under AUTO and the chunkwise fp32
    # kernel under FP32
    big = _args(dk=128, dv=128, T=4096, H=16, B=4)
    need = _tc_split_bytes(lib, big)
    assert need > 4096
    assert _kernel_name(lib, _args(dk=128, dv=128, T=4096, H=16, B=4, workspace=ws,
                                   workspace_bytes=need)) == (0, "tc_split")
    assert _kernel_name(lib, _args(dk=128, dv=128, T=4096, H=16, B=4, workspace=ws,
                                   workspace_bytes=256)) == (0, "tc_single")
    assert _kernel_name(lib, _args(dk=128, dv=128, dtype=0, workspace=ws,
                                   workspace_bytes=256)) == (0, "recurrent")
    assert _kernel_name(lib, _args(dtype=0, algo=1)) == (0, "fp32")
    assert _kernel_name(lib, _args(dtype=0, algo=3)) == (0, "recurrent")
    # every form at bf16, d = 64: the two-stream tensor-core kernel (status word only)
    assert _kernel_name(lib, _args(workspace=ws, workspace_bytes=256)) == (0, "tc_two_stream")
    # bf16 at d = 64 without the status word: GDR_ERR_WORKSPACE, as the forward itself
    assert _kernel_name(lib, _args())[0] == 7
    # no tokens: S_T = S0; no sequences: nothing
    assert _kernel_name(lib, _args(T=0, S_T=ctypes.c_void_p(0x20000))) == (0, "copy_state")
    assert _kernel_name(lib, _args(B=0)) == (0, "none")
    # the same host checks as the forward
    assert _kernel_name(lib, _args(dk=48))[0] == 2
    assert _kernel_name(lib, _args(algo=7))[0] == 1
    name = ctypes.c_char_p()
    assert lib.gdr_forward_kernel_name(ctypes.byref(_args()), None) == 1
    assert lib.gdr_forward_kernel_name(None, ctypes.byref(name)) == 1


def test_forward_zero_batch_is_a_noop(lib):
    a = _args(B=0, q=None, k=None, v=None, log_w=None, e1=None, o=None)
    assert lib.gdr_forward_chunked(ctypes.byref(a), None) == 0


def test_workspace_size(lib):
    a = _args()
    n = ctypes.c_size_t(0)
    assert lib.gdr_forward_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value >= 4 and n.value % 256 == 0
    assert lib.gdr_forward_workspace_size(None, ctypes.byref(n)) == 1


def test_decode_rejects_bad_arguments_on_host(lib):
    a = gdr.gdr_step_args()
    a.form, a.dtype, a.B, a.H, a.dk, a.dv = 1, 1, 2, 2, 64, 64
    fake = ctypes.c_void_p(0x10000)
    a.q = a.k = a.v = a.log_w = a.e1 = a.S = a.o = fake
    b = gdr.gdr_step_args.from_buffer_copy(a)
    b.dk = 40
    assert lib.gdr_decode_step(ctypes.byref(b), None) == 2
    b = gdr.gdr_step_args.from_buffer_copy(a)
    b.S = None
    assert lib.gdr_decode_step(ctypes.byref(b), None) == 1
    b = gdr.gdr_step_args.from_buffer_copy(a)
    b.S = ctypes.c_void_p(0x10008)
    assert lib.gdr_decode_step(ctypes.byref(b), None) == 3
    b = gdr.gdr_step_args.from_buffer_copy(a)
    b.form = 2   # RWKV-7 needs e2 (the removal coefficient)
    assert lib.gdr_decode_step(ctypes.byref(b), None) == 1
    b = gdr.gdr_step_args.from_buffer_copy(a)
    b.B = 0
    assert lib.gdr_decode_step(ctypes.byref(b), None) == 0


def test_state_init_rejects_bad_arguments_on_host(lib):
    assert lib.gdr_state_init(None, 1, 1, 64, 64, None, None) == 1
    assert lib.gdr_state_init(None, 0, 1, 64, 64, None, None) == 0
    assert lib.gdr_state_init(None, 1, 1, 48, 64, None, None) == 1


def _bwd_args(**kw):
    a = gdr.gdr_bwd_args()
    a.form, a.dtype, a.B, a.H, a.T, a.dk, a.dv, a.chunk = 1, 1, 1, 1, 8, 64, 64, 64
    fake = ctypes.c_void_p(0x10000)
    for name in ("q", "k", "v", "log_w", "e1", "dO", "g_q", "g_k", "g_v", "g_log_w", "g_e1"):
        setattr(a, name, fake)
    for name, val in kw.items():
        setattr(a, name, val)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(dk=32), 2), (dict(dv=16), 2), (dict(chunk=24), 2), (dict(form=9), 1), (dict(T=-1), 1),
    (dict(dO=None), 1), (dict(g_q=None), 1), (dict(g_e1=None), 1),
    (dict(g_k=ctypes.c_void_p(0x10004)), 3), (dict(workspace=None), 7),
])
def test_backward_rejects_bad_arguments_on_host(lib, kw, code):
    a = _bwd_args(**kw)
    assert lib.gdr_backward_chunked(ctypes.byref(a), None) == code


def test_backward_workspace_size(lib):
    a = _bwd_args()
    n = ctypes.c_size_t(0)
    assert lib.gdr_backward_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value >= 3 * 64 * 64 * 4 and n.value % 256 == 0   # two states, one adjoint at T = 8
    a = _bwd_args(B=0)
    assert lib.gdr_backward_chunked(ctypes.byref(a), None) == 0


def _muir_args(**kw):
    a = gdr.gdr_muir_args()
    a.dtype, a.B, a.H, a.T, a.dk, a.dv, a.chunk = 1, 1, 1, 8, 64, 64, 64
    fake = ctypes.c_void_p(0x10000)
    for name in ("q", "k", "v", "zf", "zb", "zw", "zq", "zg", "a_log", "y"):
        setattr(a, name, fake)
    a.rms_eps = 1e-6
    for name, val in kw.items():
        setattr(a, name, val)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(dk=48), 2), (dict(chunk=24), 2), (dict(dtype=4), 1), (dict(algo=9), 1),
    (dict(zq=None), 1), (dict(a_log=None), 1), (dict(y=None), 1), (dict(rms_eps=-1.0), 1),
    (dict(zg=ctypes.c_void_p(0x10002)), 3), (dict(workspace=None), 7),
])
def test_muir_rejects_bad_arguments_on_host(lib, kw, code):
    a = _muir_args(**kw)
    assert lib.gdr_muir_forward(ctypes.byref(a), None) == code


def _mlstm_args(**kw):
    a = gdr.gdr_mlstm_args()
    a.dtype, a.B, a.H, a.T, a.dk, a.dv = 1, 1, 1, 8, 64, 64
    fake = ctypes.c_void_p(0x10000)
    for name in ("q", "k", "v", "f_pre", "i_pre", "h"):
        setattr(a, name, fake)
    for name, val in kw.items():
        setattr(a, name, val)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(dk=32), 2), (dict(dv=16), 2), (dict(dtype=3), 1), (dict(T=-2), 1),
    (dict(i_pre=None), 1), (dict(h=None), 1), (dict(C0=ctypes.c_void_p(0x10000)), 1),
    (dict(v=ctypes.c_void_p(0x10008)), 3),
])
def test_mlstm_rejects_bad_arguments_on_host(lib, kw, code):
    a = _mlstm_args(**kw)
    assert lib.gdr_mlstm_forward(ctypes.byref(a), None) == code


def test_state_compose_rejects_bad_arguments_on_host(lib):
    fake = ctypes.c_void_p(0x10000)
    assert lib.gdr_state_compose(None, fake, None, fake, 2, 64, 64, None) == 1
    assert lib.gdr_state_compose(fake, fake, fake, fake, 2, 48, 64, None) == 1
    assert lib.gdr_state_compose(fake, fake, fake, None, 2, 64, 64, None) == 1   # S_in aliases S_out
    assert lib.gdr_state_compose(fake, fake, None, None, 0, 64, 64, None) == 0


def test_binding_rejects_host_memory():
    """Host tensors never reach the library: the binding checks every tensor and every
    caller-supplied workspace for device memory before marshalling a pointer."""
    import torch
    with pytest.raises(ValueError):
        gdr._workspace(torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError):
        gdr._need(torch.zeros(4), "x", torch.float32, (4,))
    x = torch.zeros(1, 8, 1, 64)
    with pytest.raises(ValueError):
        gdr.gdr_forward_chunked("gla", x, x, x, x)
    with pytest.raises(ValueError):
        gdr.gdr_state_compose(torch.zeros(1, 1, 64, 64), None, torch.zeros(1, 1, 64, 64))
