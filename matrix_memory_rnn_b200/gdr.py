"""Python binding of libgdr (include/gdr.h): argument marshalling only.

Every function here validates tensor dtypes/devices, passes raw device pointers
and the current CUDA stream to the C ABI, and raises ``GdrError`` on a non-OK
status.  All arithmetic runs in libgdr's CUDA kernels; there is no fallback.
If ``libgdr.so`` is missing and cannot be built, importing the library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdr.so")

FORMS = {"general": 0, "gdn2": 1, "rwkv7": 2, "gla": 3}
DTYPES = {"f32": 0, "bf16": 1}
ALGOS = {"auto": 0, "fp32": 1, "tc": 2, "recurrent": 3}
STATUS = {0: "GDR_OK", 1: "GDR_ERR_INVALID_ARG", 2: "GDR_ERR_UNSUPPORTED",
          3: "GDR_ERR_MISALIGNED", 4: "GDR_ERR_CUDA", 5: "GDR_ERR_DEVICE_CHECK",
          6: "GDR_ERR_TIMEOUT", 7: "GDR_ERR_WORKSPACE"}

_c_int, _vp, _fp = ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p


class gdr_fwd_args(ctypes.Structure):
    _fields_ = [("form", _c_int), ("dtype", _c_int), ("B", _c_int), ("H", _c_int),
                ("T", _c_int), ("dk", _c_int), ("dv", _c_int), ("chunk", _c_int),
                ("algo", _c_int), ("q", _vp), ("k", _vp), ("v", _vp), ("log_w", _fp),
                ("e1", _vp), ("e2", _vp), ("S0", _fp), ("o", _fp), ("S_T", _fp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class gdr_step_args(ctypes.Structure):
    _fields_ = [("form", _c_int), ("dtype", _c_int), ("B", _c_int), ("H", _c_int),
                ("dk", _c_int), ("dv", _c_int), ("q", _vp), ("k", _vp), ("v", _vp),
                ("log_w", _fp), ("e1", _vp), ("e2", _vp), ("S", _fp), ("o", _fp)]


class gdr_bwd_args(ctypes.Structure):
    _fields_ = [("form", _c_int), ("dtype", _c_int), ("B", _c_int), ("H", _c_int),
                ("T", _c_int), ("dk", _c_int), ("dv", _c_int), ("chunk", _c_int),
                ("q", _vp), ("k", _vp), ("v", _vp), ("log_w", _fp), ("e1", _vp), ("e2", _vp),
                ("S0", _fp), ("dO", _fp), ("dS_T", _fp), ("g_q", _fp), ("g_k", _fp),
                ("g_v", _fp), ("g_log_w", _fp), ("g_e1", _fp), ("g_e2", _fp), ("g_S0", _fp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class gdr_muir_args(ctypes.Structure):
    _fields_ = [("dtype", _c_int), ("B", _c_int), ("H", _c_int), ("T", _c_int), ("dk", _c_int),
                ("dv", _c_int), ("chunk", _c_int), ("algo", _c_int), ("q", _vp), ("k", _vp),
                ("v", _vp), ("zf", _vp), ("zb", _vp), ("zw", _vp), ("zq", _vp), ("zg", _vp),
                ("a_log", _fp), ("gamma_stat", _fp), ("rms_weight", _fp),
                ("rms_eps", ctypes.c_float), ("unfused", _c_int), ("S0", _fp), ("y", _fp),
                ("S_T", _fp),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class gdr_mlstm_args(ctypes.Structure):
    _fields_ = [("dtype", _c_int), ("B", _c_int), ("H", _c_int), ("T", _c_int), ("dk", _c_int),
                ("dv", _c_int), ("q", _vp), ("k", _vp), ("v", _vp), ("f_pre", _fp), ("i_pre", _fp),
                ("C0", _fp), ("n0", _fp), ("m0", _fp), ("h", _fp), ("C_T", _fp), ("n_T", _fp),
                ("m_T", _fp), ("status", _vp)]


class GdrError(RuntimeError):
    def __init__(self, fn, code):
        self.code = int(code)
        super().__init__(f"{fn} failed: {STATUS.get(self.code, self.code)}")


_lock = threading.Lock()
_lib = None


def _declare(lib):
    """Argument and result types of the C ABI on a loaded libgdr (or its timing build)."""
    lib.gdr_forward_chunked.argtypes = [ctypes.POINTER(gdr_fwd_args), _vp]
    lib.gdr_forward_workspace_size.argtypes = [ctypes.POINTER(gdr_fwd_args),
                                               ctypes.POINTER(ctypes.c_size_t)]
    lib.gdr_forward_kernel_name.argtypes = [ctypes.POINTER(gdr_fwd_args),
                                            ctypes.POINTER(ctypes.c_char_p)]
    lib.gdr_backward_chunked.argtypes = [ctypes.POINTER(gdr_bwd_args), _vp]
    lib.gdr_backward_workspace_size.argtypes = [ctypes.POINTER(gdr_bwd_args),
                                                ctypes.POINTER(ctypes.c_size_t)]
    lib.gdr_muir_forward.argtypes = [ctypes.POINTER(gdr_muir_args), _vp]
    lib.gdr_muir_workspace_size.argtypes = [ctypes.POINTER(gdr_muir_args),
                                            ctypes.POINTER(ctypes.c_size_t)]
    lib.gdr_mlstm_forward.argtypes = [ctypes.POINTER(gdr_mlstm_args), _vp]
    lib.gdr_state_compose.argtypes = [_fp, _fp, _fp, _fp, _c_int, _c_int, _c_int, _vp]
    lib.gdr_decode_step.argtypes = [ctypes.POINTER(gdr_step_args), _vp]
    lib.gdr_state_init.argtypes = [_fp, _c_int, _c_int, _c_int, _c_int, _fp, _vp]
    lib.gdr_read_status.argtypes = [_vp, _vp, ctypes.POINTER(_c_int)]
    lib.gdr_status_string.restype = ctypes.c_char_p
    lib.gdr_status_string.argtypes = [_c_int]
    for fn in ("gdr_forward_chunked", "gdr_forward_workspace_size", "gdr_forward_kernel_name",
               "gdr_backward_chunked", "gdr_backward_workspace_size",
               "gdr_muir_forward", "gdr_muir_workspace_size", "gdr_mlstm_forward",
               "gdr_state_compose",
               "gdr_decode_step",
               "gdr_state_init", "gdr_read_status", "gdr_version"):
        getattr(lib, fn).restype = _c_int


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                from . import build as _build   # nvcc is required; raises if absent
                _build.build()
            lib = ctypes.CDLL(LIB_PATH)
            _declare(lib)
            _lib = lib
    return _lib


def library():
    """The loaded ``ctypes.CDLL`` (loads it on first use)."""
    return _load()


def _check(fn, rc):
    if rc != 0:
        raise GdrError(fn, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, shape):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _workspace(w):
    """A caller-supplied workspace must be device memory: a contiguous CUDA tensor."""
    if w is not None and (not isinstance(w, torch.Tensor) or not w.is_cuda or not w.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return w


def _dtype_of(q):
    if q.dtype == torch.bfloat16:
        return "bf16", torch.bfloat16
    if q.dtype == torch.float32:
        return "f32", torch.float32
    raise ValueError(f"inputs must be bf16 or fp32, got {q.dtype}")


def _e_shapes(form, lead, dk, dv):
    if form == "general":
        return lead + (dk,), lead + (dk,)
    if form == "gdn2":
        return lead + (dk,), lead + (dv,)
    if form == "rwkv7":
        return lead + (dk,), lead
    return None, None


def _fwd_struct(form, q, k, v, log_w, e1, e2, S0, o, S_T, chunk, algo, workspace, o_ptr=None):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dname, tdt = _dtype_of(q)
    _need(q, "q", tdt, (B, T, H, dk))
    _need(k, "k", tdt, (B, T, H, dk))
    _need(v, "v", tdt, (B, T, H, dv))
    _need(log_w, "log_w", torch.float32, (B, T, H, dk))
    s1, s2 = _e_shapes(form, (B, T, H), dk, dv)
    if s1 is not None:
        _need(e1, "e1", tdt, s1)
    if e2 is not None or form in ("general", "rwkv7"):
        _need(e2, "e2", tdt, s2)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv))
    if o_ptr is None:
        _need(o, "o", torch.float32, (B, T, H, dv))
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dk, dv))
    a = gdr_fwd_args()
    a.form, a.dtype, a.algo = FORMS[form], DTYPES[dname], ALGOS[algo]
    a.B, a.H, a.T, a.dk, a.dv, a.chunk = B, H, T, dk, dv, chunk
    a.q, a.k, a.v, a.log_w = _ptr(q), _ptr(k), _ptr(v), _ptr(log_w)
    a.e1, a.e2, a.S0, a.S_T = _ptr(e1), _ptr(e2), _ptr(S0), _ptr(S_T)
    a.o = _ptr(o) if o_ptr is None else o_ptr
    if workspace is not None:
        a.workspace = _ptr(_workspace(workspace))
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    return a


def gdr_forward_workspace_size(form, q, k, v, log_w, e1=None, e2=None, chunk=64, algo="auto"):
    """Bytes of device workspace ``gdr_forward_chunked`` needs for these inputs."""
    B, T, H, dk = q.shape
    a = gdr_fwd_args()
    a.form, a.dtype, a.algo = FORMS[form], DTYPES[_dtype_of(q)[0]], ALGOS[algo]
    a.B, a.H, a.T, a.dk, a.dv, a.chunk = B, H, T, dk, v.shape[-1], chunk
    n = ctypes.c_size_t(0)
    _check("gdr_forward_workspace_size",
           _load().gdr_forward_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return int(n.value)


def gdr_forward_kernel_name(form, q, k, v, log_w, e1=None, e2=None, S0=None, *, chunk=64,
                            algo="auto", workspace_bytes=None):
    """The kernel ``gdr_forward_chunked`` runs for these inputs (a host-only query): with
    ``workspace_bytes`` None, the workspace it allocates by default."""
    B, T, H, dk = q.shape
    if workspace_bytes is None:
        workspace_bytes = gdr_forward_workspace_size(form, q, k, v, log_w, e1, e2, chunk, algo)
    # o and the workspace: the query checks only that they are given and aligned
    a = _fwd_struct(form, q, k, v, log_w, e1, e2, S0, None, None, chunk, algo, None,
                    o_ptr=ctypes.c_void_p(256))
    a.workspace = ctypes.c_void_p(256)
    a.workspace_bytes = int(workspace_bytes)
    name = ctypes.c_char_p()
    _check("gdr_forward_kernel_name", _load().gdr_forward_kernel_name(ctypes.byref(a), ctypes.byref(name)))
    return name.value.decode()


def new_workspace(nbytes, device):
    """A zeroed, 256-byte aligned device workspace of at least ``nbytes`` bytes."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def gdr_forward_chunked(form, q, k, v, log_w, e1=None, e2=None, S0=None, *, chunk=64,
                        algo="auto", o=None, S_T=None, want_state=True, workspace=None,
                        stream=None):
    """Chunkwise forward.  Tensors [B, T, H, d] (q, k, v, e1, e2 bf16 or fp32; log_w fp32).

    Returns ``(o, S_T)`` with o [B, T, H, dv] fp32 and S_T [B, H, dk, dv] fp32
    (None when ``want_state`` is False and no ``S_T`` buffer is given).
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(gdr_forward_workspace_size(form, q, k, v, log_w, e1, e2,
                                                             chunk, algo), q.device)
    a = _fwd_struct(form, q, k, v, log_w, e1, e2, S0, o, S_T, chunk, algo, workspace)
    _check("gdr_forward_chunked", _load().gdr_forward_chunked(ctypes.byref(a), _stream(stream)))
    return o, S_T


def _bwd_struct(form, q, k, v, log_w, e1, e2, S0, dO, dS_T, grads, chunk, workspace):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dname, tdt = _dtype_of(q)
    _need(q, "q", tdt, (B, T, H, dk))
    _need(k, "k", tdt, (B, T, H, dk))
    _need(v, "v", tdt, (B, T, H, dv))
    _need(log_w, "log_w", torch.float32, (B, T, H, dk))
    s1, s2 = _e_shapes(form, (B, T, H), dk, dv)
    if s1 is not None:
        _need(e1, "e1", tdt, s1)
    if e2 is not None or form in ("general", "rwkv7"):
        _need(e2, "e2", tdt, s2)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv))
    _need(dO, "dO", torch.float32, (B, T, H, dv))
    if dS_T is not None:
        _need(dS_T, "dS_T", torch.float32, (B, H, dk, dv))
    a = gdr_bwd_args()
    a.form, a.dtype = FORMS[form], DTYPES[dname]
    a.B, a.H, a.T, a.dk, a.dv, a.chunk = B, H, T, dk, dv, chunk
    a.q, a.k, a.v, a.log_w = _ptr(q), _ptr(k), _ptr(v), _ptr(log_w)
    a.e1, a.e2, a.S0, a.dO, a.dS_T = _ptr(e1), _ptr(e2), _ptr(S0), _ptr(dO), _ptr(dS_T)
    if grads is not None:
        for name in ("q", "k", "v", "log_w", "e1", "e2", "S0"):
            setattr(a, "g_" + name, _ptr(grads.get(name)))
    if workspace is not None:
        a.workspace = _ptr(_workspace(workspace))
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    return a


def gdr_backward_workspace_size(form, q, k, v, log_w, e1=None, e2=None, chunk=64):
    """Bytes of device workspace ``gdr_backward_chunked`` needs for these inputs."""
    B, T, H, dk = q.shape
    a = gdr_bwd_args()
    a.form, a.dtype = FORMS[form], DTYPES[_dtype_of(q)[0]]
    a.B, a.H, a.T, a.dk, a.dv, a.chunk = B, H, T, dk, v.shape[-1], chunk
    n = ctypes.c_size_t(0)
    _check("gdr_backward_workspace_size",
           _load().gdr_backward_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return int(n.value)


def gdr_backward_chunked(form, q, k, v, log_w, e1=None, e2=None, S0=None, dO=None, dS_T=None, *,
                         chunk=64, want_S0=True, grads=None, workspace=None, stream=None):
    """Reverse mode of ``gdr_forward_chunked``: gradients of <dO, o> + <dS_T, S_T>.

    Returns a dict with fp32 tensors ``q, k, v, log_w`` (shaped like the inputs),
    ``e1`` / ``e2`` (None where the form has no such input) and ``S0`` [B, H, dk, dv]
    (None when ``want_S0`` is False).  ``grads`` may hold preallocated outputs.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    g = dict(grads or {})

    def out(name, shape):
        if g.get(name) is None:
            g[name] = torch.empty(shape, dtype=torch.float32, device=dev)
        _need(g[name], "grad " + name, torch.float32, shape)

    out("q", (B, T, H, dk))
    out("k", (B, T, H, dk))
    out("v", (B, T, H, dv))
    out("log_w", (B, T, H, dk))
    s1, s2 = _e_shapes(form, (B, T, H), dk, dv)
    if s1 is not None:
        out("e1", s1)
    else:
        g["e1"] = None
    if s2 is not None and (e2 is not None or form in ("general", "rwkv7")):
        out("e2", s2)
    else:
        g["e2"] = None
    if want_S0:
        out("S0", (B, H, dk, dv))
    else:
        g["S0"] = None
    if workspace is None:
        workspace = new_workspace(gdr_backward_workspace_size(form, q, k, v, log_w, e1, e2, chunk),
                                  dev)
    a = _bwd_struct(form, q, k, v, log_w, e1, e2, S0, dO, dS_T, g, chunk, workspace)
    _check("gdr_backward_chunked", _load().gdr_backward_chunked(ctypes.byref(a), _stream(stream)))
    return g


def _muir_struct(q, k, v, zf, zb, zw, zq, zg, a_log, gamma_stat, rms_weight, rms_eps, S0, y,
                 S_T, chunk, algo, workspace, unfused=False):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dname, tdt = _dtype_of(q)
    for t, name, d in ((q, "q", dk), (k, "k", dk), (zf, "zf", dk), (zb, "zb", dk), (zq, "zq", dk),
                       (v, "v", dv), (zw, "zw", dv), (zg, "zg", dv)):
        _need(t, name, tdt, (B, T, H, d))
    _need(a_log, "a_log", torch.float32, (H,))
    if gamma_stat is not None:
        _need(gamma_stat, "gamma_stat", torch.float32, (H, dk))
    if rms_weight is not None:
        _need(rms_weight, "rms_weight", torch.float32, (dv,))
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv))
    if y is not None:
        _need(y, "y", torch.float32, (B, T, H, dv))
    if S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dk, dv))
    a = gdr_muir_args()
    a.dtype, a.algo = DTYPES[dname], ALGOS[algo]
    a.B, a.H, a.T, a.dk, a.dv, a.chunk = B, H, T, dk, dv, chunk
    for name, t in (("q", q), ("k", k), ("v", v), ("zf", zf), ("zb", zb), ("zw", zw), ("zq", zq),
                    ("zg", zg), ("a_log", a_log), ("gamma_stat", gamma_stat),
                    ("rms_weight", rms_weight), ("S0", S0), ("y", y), ("S_T", S_T)):
        setattr(a, name, _ptr(t))
    a.rms_eps = float(rms_eps)
    a.unfused = int(bool(unfused))
    if workspace is not None:
        a.workspace = _ptr(_workspace(workspace))
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    return a


def gdr_muir_workspace_size(q, k, v, chunk=64, algo="auto", unfused=False):
    """Bytes of device workspace ``gdr_muir_forward`` needs for inputs of these shapes."""
    B, T, H, dk = q.shape
    a = gdr_muir_args()
    a.dtype, a.algo = DTYPES[_dtype_of(q)[0]], ALGOS[algo]
    a.unfused = int(bool(unfused))
    a.B, a.H, a.T, a.dk, a.dv, a.chunk = B, H, T, dk, v.shape[-1], chunk
    n = ctypes.c_size_t(0)
    _check("gdr_muir_workspace_size",
           _load().gdr_muir_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return int(n.value)


def gdr_muir_forward(q, k, v, zf, zb, zw, zq, zg, a_log, gamma_stat=None, rms_weight=None,
                     rms_eps=1e-6, S0=None, *, chunk=64, algo="auto", unfused=False, y=None,
                     S_T=None, want_state=True, workspace=None, stream=None):
    """The Muir token mixer around the GDN-2 recurrence (include/gdr.h, gdr_muir_forward):
    pre-activations q, k, v and gate logits zf, zb, zw, zq, zg [B, T, H, .] (bf16 or fp32),
    a_log [H], optional gamma_stat [H, dk] and rms_weight [dv] (fp32).  Returns (y, S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if y is None:
        y = torch.empty((B, T, H, dv), dtype=torch.float32, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(gdr_muir_workspace_size(q, k, v, chunk, algo, unfused), q.device)
    a = _muir_struct(q, k, v, zf, zb, zw, zq, zg, a_log, gamma_stat, rms_weight, rms_eps, S0, y,
                     S_T, chunk, algo, workspace, unfused)
    _check("gdr_muir_forward", _load().gdr_muir_forward(ctypes.byref(a), _stream(stream)))
    return y, S_T


def gdr_mlstm_forward(q, k, v, f_pre, i_pre, C0=None, n0=None, m0=None, *, h=None,
                      want_state=True, status=None, stream=None):
    """xLSTM's mLSTM cell (include/gdr.h, gdr_mlstm_forward): q, k [B, T, H, dk], v
    [B, T, H, dv] (bf16 or fp32), gate pre-activations f_pre, i_pre [B, T, H] fp32, optional
    stabilized state C0 [B, H, dk, dv], n0 [B, H, dk], m0 [B, H].  ``status``: optional
    contiguous CUDA tensor whose first 4 bytes receive GDR_ERR_TIMEOUT if a bounded device
    wait runs out (read with ``gdr_read_status``).  Returns (h, C_T, n_T, m_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dname, tdt = _dtype_of(q)
    _need(q, "q", tdt, (B, T, H, dk))
    _need(k, "k", tdt, (B, T, H, dk))
    _need(v, "v", tdt, (B, T, H, dv))
    _need(f_pre, "f_pre", torch.float32, (B, T, H))
    _need(i_pre, "i_pre", torch.float32, (B, T, H))
    if C0 is not None:
        _need(C0, "C0", torch.float32, (B, H, dk, dv))
        _need(n0, "n0", torch.float32, (B, H, dk))
        _need(m0, "m0", torch.float32, (B, H))
    dev = q.device
    if h is None:
        h = torch.empty((B, T, H, dv), dtype=torch.float32, device=dev)
    _need(h, "h", torch.float32, (B, T, H, dv))
    C_T = n_T = m_T = None
    if want_state:
        C_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
        n_T = torch.empty((B, H, dk), dtype=torch.float32, device=dev)
        m_T = torch.empty((B, H), dtype=torch.float32, device=dev)
    a = gdr_mlstm_args()
    a.dtype, a.B, a.H, a.T, a.dk, a.dv = DTYPES[dname], B, H, T, dk, dv
    for name, t in (("q", q), ("k", k), ("v", v), ("f_pre", f_pre), ("i_pre", i_pre), ("C0", C0),
                    ("n0", n0), ("m0", m0), ("h", h), ("C_T", C_T), ("n_T", n_T), ("m_T", m_T)):
        setattr(a, name, _ptr(t))
    if status is not None and _workspace(status).numel() * status.element_size() < 4:
        raise ValueError("status must hold at least 4 bytes")
    a.status = _ptr(status)
    _check("gdr_mlstm_forward", _load().gdr_mlstm_forward(ctypes.byref(a), _stream(stream)))
    return h, C_T, n_T, m_T


def gdr_decode_step(form, q, k, v, log_w, e1, e2, S, *, o=None, stream=None):
    """One token per (b, h): inputs [B, H, d]; S [B, H, dk, dv] fp32 updated in place.  Returns o."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    dname, tdt = _dtype_of(q)
    _need(q, "q", tdt, (B, H, dk))
    _need(k, "k", tdt, (B, H, dk))
    _need(v, "v", tdt, (B, H, dv))
    _need(log_w, "log_w", torch.float32, (B, H, dk))
    s1, s2 = _e_shapes(form, (B, H), dk, dv)
    if s1 is not None:
        _need(e1, "e1", tdt, s1)
    if e2 is not None or form in ("general", "rwkv7"):
        _need(e2, "e2", tdt, s2)
    _need(S, "S", torch.float32, (B, H, dk, dv))
    if o is None:
        o = torch.empty((B, H, dv), dtype=torch.float32, device=q.device)
    _need(o, "o", torch.float32, (B, H, dv))
    a = gdr_step_args()
    a.form, a.dtype = FORMS[form], DTYPES[dname]
    a.B, a.H, a.dk, a.dv = B, H, dk, dv
    a.q, a.k, a.v, a.log_w = _ptr(q), _ptr(k), _ptr(v), _ptr(log_w)
    a.e1, a.e2, a.S, a.o = _ptr(e1), _ptr(e2), _ptr(S), _ptr(o)
    _check("gdr_decode_step", _load().gdr_decode_step(ctypes.byref(a), _stream(stream)))
    return o


def gdr_state_compose(M, S_in, Q, *, out=None, stream=None):
    """M [B, H, dk, dk] S_in [B, H, dk, dv] + Q [B, H, dk, dv] per head (S_in None = 0)."""
    B, H, dk, dv = Q.shape
    _need(M, "M", torch.float32, (B, H, dk, dk))
    _need(Q, "Q", torch.float32, (B, H, dk, dv))
    if S_in is not None:
        _need(S_in, "S_in", torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty_like(Q)
    _need(out, "out", torch.float32, (B, H, dk, dv))
    _check("gdr_state_compose", _load().gdr_state_compose(_ptr(out), _ptr(M), _ptr(S_in), _ptr(Q),
                                                          B * H, dk, dv, _stream(stream)))
    return out


def gdr_state_init(S, src=None, *, stream=None):
    """S [B, H, dk, dv] fp32 = src (same shape) or zeros."""
    B, H, dk, dv = S.shape
    _need(S, "S", torch.float32, (B, H, dk, dv))
    if src is not None:
        _need(src, "src", torch.float32, (B, H, dk, dv))
    _check("gdr_state_init",
           _load().gdr_state_init(_ptr(S), B, H, dk, dv, _ptr(src), _stream(stream)))
    return S


def gdr_read_status(workspace, *, stream=None):
    """Synchronizes and returns (and clears) the device status word of ``workspace``."""
    st = ctypes.c_int(0)
    _check("gdr_read_status", _load().gdr_read_status(_ptr(_workspace(workspace)), _stream(stream),
                                                      ctypes.byref(st)))
    return STATUS.get(st.value, st.value)


def gdr_version():
    return int(_load().gdr_version())


def to_device(arrays: dict, dtype: str, device="cuda") -> dict:
    """Moves the float32 numpy arrays of ``synth`` to the device: ``log_w``/``S0`` stay
    fp32, the token inputs become ``dtype`` ("bf16" or "f32"; exact, the values are
    already rounded to it)."""
    import numpy as np
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for name, a in arrays.items():
        if a is None:
            out[name] = None
            continue
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
        t = t.to(device=device, dtype=torch.float32 if name in ("log_w", "S0") else tdt)
        out[name] = t.contiguous()
    return out


def gdr_forward_chunked_noalloc(form, q, k, v, log_w, e1=None, e2=None, S0=None, *, chunk=64,
                                algo="auto", o=None, S_T=None, stream=None):
    """``gdr_forward_chunked`` through the entry point that allocates nothing.

    For callers that may not allocate device memory: libgdr supplies the scratch
    from a fixed array of its own (see include/gdr.h).  ``o`` and ``S_T`` must be
    given by the caller (this function allocates nothing either).
    """
    lib = _load()
    fn = lib.gdr_forward_chunked_noalloc
    fn.argtypes = [ctypes.POINTER(gdr_fwd_args), _vp]
    fn.restype = _c_int
    if o is None:
        raise ValueError("o is required (the no-alloc path allocates nothing)")
    a = _fwd_struct(form, q, k, v, log_w, e1, e2, S0, o, S_T, chunk, algo, None)
    _check("gdr_forward_chunked_noalloc", fn(ctypes.byref(a), _stream(stream)))
    return o, S_T


def gdr_noalloc_read_status(*, stream=None):
    """Synchronizes ``stream`` and returns (and clears) the device status word of
    ``gdr_forward_chunked_noalloc`` on the current device."""
    lib = _load()
    fn = lib.gdr_noalloc_read_status
    fn.argtypes = [_vp, ctypes.POINTER(_c_int)]
    fn.restype = _c_int
    st = ctypes.c_int(0)
    _check("gdr_noalloc_read_status", fn(_stream(stream), ctypes.byref(st)))
    return STATUS.get(st.value, st.value)
