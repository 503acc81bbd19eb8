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
