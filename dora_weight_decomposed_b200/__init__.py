"""DoRA adapter layer for B200 (sm_100a): Python binding of libdora_b200.so.

The functions here only marshal arguments: they check tensor dtypes, devices
and shapes, allocate outputs and the workspace with torch (device memory and
streams are the only things torch provides), and call the C ABI declared in
include/dora.h. Every step of the computation runs in the library's CUDA
kernels; if the library is missing the import of this module still works but
every call raises.

    norm, g, gm1 = dora_norm(W0, A, B, m, s)
    y, su, pre   = dora_forward(x, W0, A, B, gm1, s)
    dm, dA, dB, dx = dora_backward(dy, x, W0, A, B, norm, g, su, pre, s)    # full=True: no detach
    W_merged     = dora_merge(W0, A, B, g, s)
    B_vera       = dora_vera_compose(B_shared, b, d)       # DVoRA: B' for the calls above
    db, dd       = dora_vera_grad(B_shared, b, d, dB)

bf16 tensors use the tcgen05 tensor-core path; fp32 tensors use the SIMT path.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = ["DoraError", "load_library", "library_path", "dora_workspace_size", "dora_norm", "dora_forward",
           "dora_norm_noalloc", "dora_backward", "dora_backward_full", "dora_merge", "dora_vera_compose",
           "dora_selftest_timeout",
           "dora_vera_grad", "dora_device_status", "dora_last_error",
           "dora_version",
           "dora_profile_start",
           "dora_profile_stop", "dora_profile_count", "dora_profile_read", "DORA_OP_NORM",
           "DORA_OP_FORWARD", "DORA_OP_BACKWARD", "DORA_OP_MERGE", "DORA_OP_BACKWARD_FULL", "STATUS_NAMES",
           "EXPORTED_SYMBOLS"]

DORA_BF16, DORA_FP32 = 0, 1
DORA_OP_NORM, DORA_OP_FORWARD, DORA_OP_BACKWARD, DORA_OP_MERGE, DORA_OP_BACKWARD_FULL, DORA_OP_VERA_GRAD = range(6)
STATUS_NAMES = {0: "DORA_OK", 1: "DORA_EINVAL", 2: "DORA_EUNSUPPORTED", 3: "DORA_EWORKSPACE", 4: "DORA_ECUDA",
                5: "DORA_ETIMEOUT"}
EXPORTED_SYMBOLS = ("dora_workspace_size", "dora_norm", "dora_norm_noalloc", "dora_forward", "dora_backward",
                    "dora_backward_full", "dora_merge", "dora_vera_compose", "dora_vera_grad", "dora_device_status",
                    "dora_selftest_timeout",
                    "dora_profile_start", "dora_profile_stop", "dora_profile_count", "dora_profile_read",
                    "dora_last_error", "dora_version")

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libdora_b200.so")


class DoraError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class ProfileRecord(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("ms", ctypes.c_float)]


class DoraDesc(ctypes.Structure):
    _fields_ = [("d_out", ctypes.c_int64), ("d_in", ctypes.c_int64), ("r", ctypes.c_int64),
                ("dtype", ctypes.c_int), ("s", ctypes.c_float)]


_lib = None
_lib_lock = threading.Lock()


def load_library() -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing; build it with `python -m dora_weight_decomposed_b200.build`")
        lib = ctypes.CDLL(path)
        P, I64, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        DP = ctypes.POINTER(DoraDesc)
        lib.dora_workspace_size.argtypes = [DP, I64, ctypes.c_int]
        lib.dora_workspace_size.restype = SZ
        lib.dora_norm.argtypes = [DP, P, P, P, P, P, P, P, P, SZ, P]
        lib.dora_norm.restype = ctypes.c_int
        lib.dora_forward.argtypes = [DP, I64, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.dora_forward.restype = ctypes.c_int
        lib.dora_backward.argtypes = [DP, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.dora_backward.restype = ctypes.c_int
        lib.dora_backward_full.argtypes = lib.dora_backward.argtypes
        lib.dora_backward_full.restype = ctypes.c_int
        lib.dora_merge.argtypes = [DP, P, P, P, P, P, P, SZ, P]
        lib.dora_merge.restype = ctypes.c_int
        lib.dora_vera_compose.argtypes = [DP, P, P, P, P, P]
        lib.dora_vera_compose.restype = ctypes.c_int
        lib.dora_vera_grad.argtypes = [DP, P, P, P, P, P, P, P, SZ, P]
        lib.dora_vera_grad.restype = ctypes.c_int
        lib.dora_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint)]
        lib.dora_device_status.restype = ctypes.c_int
        lib.dora_selftest_timeout.argtypes = [ctypes.c_uint32, P, P]
        lib.dora_selftest_timeout.restype = ctypes.c_int
        lib.dora_profile_start.argtypes = [ctypes.c_int]
        lib.dora_profile_start.restype = ctypes.c_int
        lib.dora_profile_stop.argtypes = []
        lib.dora_profile_stop.restype = ctypes.c_int
        lib.dora_profile_count.argtypes = []
        lib.dora_profile_count.restype = ctypes.c_int
        lib.dora_profile_read.argtypes = [ctypes.POINTER(ProfileRecord), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
        lib.dora_profile_read.restype = ctypes.c_int
        lib.dora_last_error.argtypes = []
        lib.dora_last_error.restype = ctypes.c_char_p
        lib.dora_version.argtypes = []
        lib.dora_version.restype = ctypes.c_int
        _lib = lib
        return lib


def dora_last_error() -> str:
    return load_library().dora_last_error().decode()


def dora_version() -> int:
    return load_library().dora_version()


def _check(status: int) -> None:
    if status != 0:
        raise DoraError(status, dora_last_error())


def _torch():
    import torch
    return torch


def _desc(d_out: int, d_in: int, r: int, dtype, s: float) -> DoraDesc:
    torch = _torch()
    if dtype == torch.bfloat16:
        code = DORA_BF16
    elif dtype == torch.float32:
        code = DORA_FP32
    else:
        raise TypeError(f"DoRA tensors must be bfloat16 or float32, got {dtype}")
    return DoraDesc(int(d_out), int(d_in), int(r), code, float(s))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream_ptr(stream) -> int | None:
    """The CUDA stream handle; the library launches on the current device, so the stream must be on it."""
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    if s.device.index != torch.cuda.current_device():
        raise ValueError(f"stream is on {s.device}, but the current device is cuda:{torch.cuda.current_device()}")
    return s.cuda_stream or None


def _shape(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _args(dtype, device, **spec):
    """Check every given tensor (name=(tensor, shape, kind)); kind "t" = the layer dtype, "f" = float32.

    The C ABI cannot see shapes or dtypes: a wrong one would make a kernel read
    or write past a buffer, so every tensor, inputs and caller-supplied outputs
    alike, is checked here before anything is launched. None entries (optional
    outputs) are skipped.
    """
    torch = _torch()
    # The library launches every kernel on the current device: tensors on another
    # device would hand it pointers that device cannot use.
    if device.type == "cuda" and device.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {device}, but the current device is cuda:{torch.cuda.current_device()}; "
                         f"call under torch.cuda.device({device.index})")
    for name, (t, shape, kind) in spec.items():
        if t is None:
            continue
        _shape(t, shape, name)
        want = dtype if kind == "t" else torch.float32
        if t.dtype != want:
            raise TypeError(f"{name} is {t.dtype}, expected {want}")
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device}")


def dora_workspace_size(d_out: int, d_in: int, r: int, dtype, s: float, T: int, op: int) -> int:
    d = _desc(d_out, d_in, r, dtype, s)
    return int(load_library().dora_workspace_size(ctypes.byref(d), int(T), int(op)))


def _workspace(desc: DoraDesc, T: int, op: int, device, ws):
    torch = _torch()
    need = int(load_library().dora_workspace_size(ctypes.byref(desc), int(T), int(op)))
    if ws is not None:
        return ws, ws.numel() * ws.element_size()
    if need == 0:
        return None, 0
    return torch.empty(need, dtype=torch.uint8, device=device), need


def dora_norm(W0, A, B, m, s: float, *, norm_out=None, g_out=None, gm1_out=None, ws=None, stream=None):
    """Per-row norm C of W0 + s B A (factored form), g = m / C, gm1 = (m - C) / C."""
    torch = _torch()
    lib = load_library()
    d_out, d_in = W0.shape
    r = A.shape[0]
    _args(W0.dtype, W0.device, A=(A, (r, d_in), "t"), B=(B, (d_out, r), "t"), m=(m, (d_out,), "f"),
          norm_out=(norm_out, (d_out,), "f"), g_out=(g_out, (d_out,), "f"), gm1_out=(gm1_out, (d_out,), "f"))
    desc = _desc(d_out, d_in, r, W0.dtype, s)
    f32 = dict(dtype=torch.float32, device=W0.device)
    norm_out = torch.empty(d_out, **f32) if norm_out is None else norm_out
    g_out = torch.empty(d_out, **f32) if g_out is None else g_out
    gm1_out = torch.empty(d_out, **f32) if gm1_out is None else gm1_out
    wsb, nbytes = _workspace(desc, 0, DORA_OP_NORM, W0.device, ws)
    _check(lib.dora_norm(ctypes.byref(desc), _ptr(W0), _ptr(A), _ptr(B), _ptr(m), _ptr(norm_out), _ptr(g_out),
                         _ptr(gm1_out), _ptr(wsb), nbytes, _stream_ptr(stream)))
    return norm_out, g_out, gm1_out


def dora_forward(x, W0, A, B, gm1, s: float, *, save_for_backward: bool = True, y=None, su_save=None,
                 pre_save=None, ws=None, stream=None):
    """y = x (diag(g) (W0 + s B A))^T composed as pre + gm1 * pre.

    Returns (y, su, pre); su = s x A^T and pre (the un-scaled output) are the
    tensors dora_backward needs (None when save_for_backward is False).
    """
    torch = _torch()
    lib = load_library()
    T, d_in = x.shape
    d_out = W0.shape[0]
    r = A.shape[0]
    dev = x.device
    _args(W0.dtype, dev, x=(x, (T, d_in), "t"), W0=(W0, (d_out, d_in), "t"), A=(A, (r, d_in), "t"),
          B=(B, (d_out, r), "t"), gm1=(gm1, (d_out,), "f"), y=(y, (T, d_out), "t"),
          su_save=(su_save, (T, r), "t"), pre_save=(pre_save, (T, d_out), "t"))
    desc = _desc(d_out, d_in, r, W0.dtype, s)
    y = torch.empty(T, d_out, dtype=x.dtype, device=dev) if y is None else y
    if save_for_backward:
        su_save = torch.empty(T, r, dtype=x.dtype, device=dev) if su_save is None else su_save
        pre_save = torch.empty(T, d_out, dtype=x.dtype, device=dev) if pre_save is None else pre_save
    else:
        su_save = pre_save = None
    wsb, nbytes = _workspace(desc, T, DORA_OP_FORWARD, dev, ws)
    _check(lib.dora_forward(ctypes.byref(desc), T, _ptr(x), _ptr(W0), _ptr(A), _ptr(B), _ptr(gm1), _ptr(y),
                            _ptr(su_save), _ptr(pre_save), _ptr(wsb), nbytes, _stream_ptr(stream)))
    return y, su_save, pre_save


def dora_backward(dy, x, W0, A, B, norm, g, su_save, pre_save, s: float, *, need_dx: bool = True, full: bool = False,
                  dm=None, dA=None, dB=None, dx=None, ws=None, stream=None):
    """Gradients (dm, dA, dB, dx); dx is None when need_dx is False.

    Detached norm by default (dora_backward); full=True keeps the gradient
    through the norm (dora_backward_full), which changes dA and dB only.
    """
    torch = _torch()
    lib = load_library()
    T, d_in = x.shape
    d_out = W0.shape[0]
    r = A.shape[0]
    dev = x.device
    _args(W0.dtype, dev, dy=(dy, (T, d_out), "t"), x=(x, (T, d_in), "t"), W0=(W0, (d_out, d_in), "t"),
          A=(A, (r, d_in), "t"), B=(B, (d_out, r), "t"), norm=(norm, (d_out,), "f"), g=(g, (d_out,), "f"),
          su_save=(su_save, (T, r), "t"), pre_save=(pre_save, (T, d_out), "t"), dm=(dm, (d_out,), "f"),
          dA=(dA, (r, d_in), "t"), dB=(dB, (d_out, r), "t"), dx=(dx if need_dx else None, (T, d_in), "t"))
    if su_save is None or pre_save is None:
        raise ValueError("su_save and pre_save (from dora_forward) are required")
    desc = _desc(d_out, d_in, r, W0.dtype, s)
    dm = torch.empty(d_out, dtype=torch.float32, device=dev) if dm is None else dm
    dA = torch.empty(r, d_in, dtype=x.dtype, device=dev) if dA is None else dA
    dB = torch.empty(d_out, r, dtype=x.dtype, device=dev) if dB is None else dB
    if need_dx and dx is None:
        dx = torch.empty(T, d_in, dtype=x.dtype, device=dev)
    if not need_dx:
        dx = None
    wsb, nbytes = _workspace(desc, T, DORA_OP_BACKWARD_FULL if full else DORA_OP_BACKWARD, dev, ws)
    fn = lib.dora_backward_full if full else lib.dora_backward
    _check(fn(ctypes.byref(desc), T, _ptr(dy), _ptr(x), _ptr(W0), _ptr(A), _ptr(B), _ptr(norm), _ptr(g),
              _ptr(su_save), _ptr(pre_save), _ptr(dm), _ptr(dA), _ptr(dB), _ptr(dx), _ptr(wsb), nbytes,
              _stream_ptr(stream)))
    return dm, dA, dB, dx


def dora_merge(W0, A, B, g, s: float, *, out=None, ws=None, stream=None):
    """Merged weight diag(g) (W0 + s B A) for deployment; out may be W0 (in place)."""
    torch = _torch()
    lib = load_library()
    d_out, d_in = W0.shape
    r = A.shape[0]
    _args(W0.dtype, W0.device, A=(A, (r, d_in), "t"), B=(B, (d_out, r), "t"), g=(g, (d_out,), "f"),
          out=(out, (d_out, d_in), "t"))
    desc = _desc(d_out, d_in, r, W0.dtype, s)
    out = torch.empty_like(W0) if out is None else out
    wsb, nbytes = _workspace(desc, 0, DORA_OP_MERGE, W0.device, ws)
    _check(lib.dora_merge(ctypes.byref(desc), _ptr(W0), _ptr(A), _ptr(B), _ptr(g), _ptr(out), _ptr(wsb), nbytes,
                          _stream_ptr(stream)))
    return out


def dora_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the kernels' timeout flags."""
    flags = ctypes.c_uint(0)
    st = load_library().dora_device_status(_stream_ptr(stream), ctypes.byref(flags))
    if st not in (0, 5):
        _check(st)
    return int(flags.value)


def dora_selftest_timeout(limit_us: int = 20000, stream=None) -> int:
    """Run the failure-detection self-test kernel (a bounded wait that runs out).

    Returns the word the kernel wrote (1 = its wait ran out); the timeout is
    also left in the device status word for the next dora_device_status.
    """
    torch = _torch()
    scratch = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(load_library().dora_selftest_timeout(int(limit_us), _ptr(scratch), _stream_ptr(stream)))
    return int(scratch.item())


def dora_profile_start(capacity: int = 4096) -> None:
    """Time every kernel the library launches from now on (see include/dora.h)."""
    _check(load_library().dora_profile_start(int(capacity)))


def dora_profile_stop() -> None:
    _check(load_library().dora_profile_stop())


def dora_profile_count() -> int:
    return int(load_library().dora_profile_count())


def dora_profile_read() -> list[tuple[str, float]]:
    """[(kernel name, milliseconds)] for the recorded launches, in launch order."""
    lib = load_library()
    n = lib.dora_profile_count()
    recs = (ProfileRecord * max(n, 1))()
    got = ctypes.c_int(0)
    _check(lib.dora_profile_read(recs, n, ctypes.byref(got)))
    return [(recs[i].name.decode(), float(recs[i].ms)) for i in range(got.value)]


def dora_norm_noalloc(W0, A, B, m, s: float, *, norm_out=None, g_out=None, gm1_out=None, stream=None):
    """dora_norm for callers that cannot allocate device memory for a workspace.

    The library uses its own built-in 16 MiB device scratch array instead (see
    include/dora.h); outputs may be passed in preallocated. Calls on one device
    share that array, so calls that may overlap on the GPU must be ordered.
    """
    torch = _torch()
    lib = load_library()
    fn = lib.dora_norm_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(DoraDesc), P, P, P, P, P, P, P, P]
    fn.restype = ctypes.c_int
    d_out, d_in = W0.shape
    r = A.shape[0]
    _args(W0.dtype, W0.device, A=(A, (r, d_in), "t"), B=(B, (d_out, r), "t"), m=(m, (d_out,), "f"),
          norm_out=(norm_out, (d_out,), "f"), g_out=(g_out, (d_out,), "f"), gm1_out=(gm1_out, (d_out,), "f"))
    desc = _desc(d_out, d_in, r, W0.dtype, s)
    f32 = dict(dtype=torch.float32, device=W0.device)
    norm_out = torch.empty(d_out, **f32) if norm_out is None else norm_out
    g_out = torch.empty(d_out, **f32) if g_out is None else g_out
    gm1_out = torch.empty(d_out, **f32) if gm1_out is None else gm1_out
    _check(fn(ctypes.byref(desc), _ptr(W0), _ptr(A), _ptr(B), _ptr(m), _ptr(norm_out), _ptr(g_out), _ptr(gm1_out),
              _stream_ptr(stream)))
    return norm_out, g_out, gm1_out


def dora_backward_full(dy, x, W0, A, B, norm, g, su_save, pre_save, s: float, **kw):
    """dora_backward with the gradient through the norm kept (appendix A eq. A.1)."""
    return dora_backward(dy, x, W0, A, B, norm, g, su_save, pre_save, s, full=True, **kw)


def dora_vera_compose(B_shared, b, d, *, out=None, s: float = 1.0, stream=None):
    """DVoRA's B' = diag(b) B_shared diag(d) [d_out x r]; b, d float32."""
    torch = _torch()
    lib = load_library()
    d_out, r = B_shared.shape
    _args(B_shared.dtype, B_shared.device, b=(b, (d_out,), "f"), d=(d, (r,), "f"), out=(out, (d_out, r), "t"))
    desc = _desc(d_out, 8, r, B_shared.dtype, s)
    out = torch.empty_like(B_shared) if out is None else out
    _check(lib.dora_vera_compose(ctypes.byref(desc), _ptr(B_shared), _ptr(b), _ptr(d), _ptr(out),
                                 _stream_ptr(stream)))
    return out


def dora_vera_grad(B_shared, b, d, dB, *, s: float = 1.0, db=None, dd=None, ws=None, stream=None):
    """Gradients (db [d_out], dd [r], float32) of DVoRA's trained vectors from dB' = dL/dB'."""
    torch = _torch()
    lib = load_library()
    d_out, r = B_shared.shape
    _args(B_shared.dtype, B_shared.device, b=(b, (d_out,), "f"), d=(d, (r,), "f"), dB=(dB, (d_out, r), "t"),
          db=(db, (d_out,), "f"), dd=(dd, (r,), "f"))
    desc = _desc(d_out, 8, r, B_shared.dtype, s)
    db = torch.empty(d_out, dtype=torch.float32, device=B_shared.device) if db is None else db
    dd = torch.empty(r, dtype=torch.float32, device=B_shared.device) if dd is None else dd
    wsb, nbytes = _workspace(desc, 0, DORA_OP_VERA_GRAD, B_shared.device, ws)
    _check(lib.dora_vera_grad(ctypes.byref(desc), _ptr(B_shared), _ptr(b), _ptr(d), _ptr(dB), _ptr(db), _ptr(dd),
                              _ptr(wsb), nbytes, _stream_ptr(stream)))
    return db, dd
