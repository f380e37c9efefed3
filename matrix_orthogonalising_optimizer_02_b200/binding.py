"""Thin Python binding of ``include/muon_b200.h`` (ctypes).

Argument marshalling only: every step of the path runs in ``libmuon_b200.so``.
Tensors are passed by ``data_ptr()``; the stream defaults to torch's current
CUDA stream.  There is no fallback: if the library is not built, or a call
fails, a ``MuonError`` is raised.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_float, c_int, c_longlong, c_size_t, c_void_p
from dataclasses import dataclass
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmuon_b200.so")

# enums of muon_b200.h
MUON_OK, MUON_ERR_INVALID_ARG, MUON_ERR_UNSUPPORTED_SHAPE, MUON_ERR_ALIGNMENT = 0, 1, 2, 3
MUON_ERR_WORKSPACE_TOO_SMALL, MUON_ERR_CUDA, MUON_ERR_NONFINITE, MUON_ERR_DEVICE_TIMEOUT = 4, 5, 6, 7
MUON_ERR_DEVICE_UNDRAINED = 8
MUON_BF16, MUON_F32 = 0, 1
SCALE_MODES = {"moonlight": 0, "kellerjordan": 1, "mup": 2, "naive": 3}
MUON_MAX_NS_ITERS = 32
KERNEL_KINDS = {"momentum": 0, "scale": 1, "ns_gemm": 2, "update": 3, "simt_gemm": 4, "lu": 5, "misc": 6,
                "tc_f32": 7, "simt_gemm_f64": 8}

#: Exported entry points, as declared in include/muon_b200.h.
EXPORTED = (
    "muon_step_workspace_size", "muon_step_workspace_min", "muon_step_batched",
    "ns_workspace_size", "ns_orthogonalize", "stiefel_workspace_size", "stiefel_cayley_step",
    "muon_workspace_device_status", "muon_timing_enable", "muon_timing_reset", "muon_timing_read",
    "muon_status_string", "muon_build_info", "muon_frobenius_prescale_static",
    "muon_cayley_workspace_size", "muon_cayley_step", "muon_step_host_grad_workspace_size",
    "muon_step_batched_host_grad", "muon_last_error", "muon_selftest_wait_timeout",
)


class MuonError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().muon_status_string(status).decode() if _LIB is not None else str(status)
        if status == MUON_ERR_CUDA and _LIB is not None:
            detail = _LIB.muon_last_error()
            if detail:
                msg += f": {detail.decode()}"
        super().__init__(f"{where}: {msg} (status {status})")


class NsSchedule(ctypes.Structure):
    _fields_ = [("n_iters", c_int), ("coeffs", POINTER(c_float)), ("n_split_iters", c_int),
                ("fp32_mode", c_int), ("eps", c_float)]


class MatrixDesc(ctypes.Structure):
    _fields_ = [("W", c_void_p), ("G", c_void_p), ("M", c_void_p), ("O_out", c_void_p),
                ("rows", c_int), ("cols", c_int), ("w_dtype", c_int), ("g_dtype", c_int)]


class Hyper(ctypes.Structure):
    _fields_ = [("lr", c_float), ("beta", c_float), ("weight_decay", c_float), ("nesterov", c_int),
                ("scale_mode", c_int), ("ns", NsSchedule)]


_LIB = None


def _lib():
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m matrix_orthogonalising_optimizer_02_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "muon_step_workspace_size": (c_size_t, [POINTER(MatrixDesc), c_int, POINTER(Hyper)]),
        "muon_step_workspace_min": (c_size_t, [POINTER(MatrixDesc), c_int, POINTER(Hyper)]),
        "muon_step_batched": (c_int, [POINTER(MatrixDesc), c_int, POINTER(Hyper), c_void_p, c_size_t, c_void_p]),
        "muon_step_host_grad_workspace_size": (c_size_t, [POINTER(MatrixDesc), c_int, POINTER(Hyper)]),
        "muon_step_batched_host_grad": (c_int, [POINTER(MatrixDesc), c_int, POINTER(Hyper), c_void_p, c_size_t,
                                                c_void_p]),
        "ns_workspace_size": (c_size_t, [c_int, c_int, c_int, POINTER(NsSchedule)]),
        "ns_orthogonalize": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, POINTER(NsSchedule),
                                     c_void_p, c_size_t, c_void_p]),
        "stiefel_workspace_size": (c_size_t, [c_int, c_int, c_int]),
        "stiefel_cayley_step": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_float, c_void_p, c_size_t,
                                        c_void_p]),
        "muon_workspace_device_status": (c_int, [c_void_p, c_size_t, POINTER(c_int), c_void_p]),
        "muon_timing_enable": (c_int, [c_int]),
        "muon_timing_reset": (c_int, []),
        "muon_timing_read": (c_int, [c_int, POINTER(c_double), POINTER(c_longlong), POINTER(c_double)]),
        "muon_status_string": (ctypes.c_char_p, [c_int]),
        "muon_last_error": (ctypes.c_char_p, []),
        "muon_selftest_wait_timeout": (c_int, [c_void_p, c_size_t, c_void_p]),
        "muon_build_info": (ctypes.c_char_p, []),
        "muon_cayley_workspace_size": (c_size_t, [c_int, c_int, c_int]),
        "muon_cayley_step": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_float, c_float, c_int,
                                     c_void_p, c_size_t, c_void_p]),
        "muon_frobenius_prescale_static": (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                                   c_float, c_void_p, c_void_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name, None)
        if fn is None:       # reported by the export test; calling it raises AttributeError
            continue
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def load():
    """Loads the shared library (raises if it is missing) and returns the ctypes handle."""
    return _lib()


def _check(status: int, where: str):
    if status != MUON_OK:
        raise MuonError(status, where)


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return MUON_BF16
    if t.dtype == torch.float32:
        return MUON_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or fp32 expected")


class Schedule:
    """Newton-Schulz schedule: per-iteration (a, b, c), split-bf16 prefix, fp32 mode, eps."""

    def __init__(self, coeffs: Sequence[Sequence[float]], n_split_iters: int = 0, fp32_mode: bool = False,
                 eps: float = 1e-7):
        flat = [float(x) for abc in coeffs for x in abc]
        self._arr = (c_float * max(1, len(flat)))(*flat)
        self.c = NsSchedule(len(coeffs), ctypes.cast(self._arr, POINTER(c_float)), int(n_split_iters),
                            int(bool(fp32_mode)), float(eps))
        self.coeffs = [tuple(abc) for abc in coeffs]

    @classmethod
    def fixed(cls, steps: int = 5, coeffs=(3.4445, -4.7750, 2.0315), **kw):
        return cls([coeffs] * steps, **kw)

    @classmethod
    def hybrid(cls, n_fast: int = 8, n_stable: int = 2, fast=(3.4445, -4.7750, 2.0315),
               stable=(1.875, -1.25, 0.375), **kw):
        return cls([fast] * n_fast + [stable] * n_stable, **kw)


@dataclass
class Matrix:
    """One Muon matrix: W (bf16/fp32, updated in place), G (bf16/fp32), M (fp32, updated in
    place), optional O_out receiving the Newton-Schulz output."""
    W: object
    G: object
    M: object
    O_out: Optional[object] = None


def _need(t, name: str, cuda: bool = True, device=None):
    """Checks a tensor handed to the library by its data pointer: dense (a strided view's
    pointer would be read as another matrix) and on the expected device."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (the library reads it as a dense row-major array)")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if cuda and device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _descs(mats: Sequence[Matrix], g_on_host: bool = False):
    import torch
    arr = (MatrixDesc * len(mats))()
    for i, m in enumerate(mats):
        if m.W.dim() != 2:
            raise ValueError("W must be a 2-D matrix")
        rows, cols = m.W.shape
        if tuple(m.G.shape) != (rows, cols) or tuple(m.M.shape) != (rows, cols):
            raise ValueError("W, G and M must have the same 2-D shape")
        if m.M.dtype != torch.float32:
            raise TypeError("the momentum buffer M must be fp32")
        _need(m.W, "W")
        _need(m.M, "M", device=m.W.device)
        _need(m.G, "G", cuda=not g_on_host, device=m.W.device)
        if m.O_out is not None:
            if tuple(m.O_out.shape) != (rows, cols):
                raise ValueError("O_out must have W's shape")
            _need(m.O_out, "O_out", device=m.W.device)
        arr[i] = MatrixDesc(m.W.data_ptr(), m.G.data_ptr(), m.M.data_ptr(),
                            m.O_out.data_ptr() if m.O_out is not None else None,
                            rows, cols, _dtype_code(m.W), _dtype_code(m.G))
    return arr


def hyper(lr: float, beta: float = 0.95, weight_decay: float = 0.0, nesterov: bool = False,
          scale_mode: str = "moonlight", schedule: Optional[Schedule] = None) -> tuple:
    sch = schedule if schedule is not None else Schedule.fixed(5)
    h = Hyper(float(lr), float(beta), float(weight_decay), int(bool(nesterov)), SCALE_MODES[scale_mode], sch.c)
    return (h, sch)   # keep the schedule (and its coefficient array) alive with the struct


def muon_step_workspace_size(mats: Sequence[Matrix], hp) -> int:
    return int(_lib().muon_step_workspace_size(_descs(mats), len(mats), ctypes.byref(hp[0])))


def muon_step_workspace_min(mats: Sequence[Matrix], hp) -> int:
    return int(_lib().muon_step_workspace_min(_descs(mats), len(mats), ctypes.byref(hp[0])))


def muon_step_batched(mats: Sequence[Matrix], hp, workspace, stream=None):
    st = _lib().muon_step_batched(_descs(mats), len(mats), ctypes.byref(hp[0]), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "muon_step_batched")


def muon_step_host_grad_workspace_size(mats: Sequence[Matrix], hp) -> int:
    return int(_lib().muon_step_host_grad_workspace_size(_descs(mats, g_on_host=True), len(mats),
                                                         ctypes.byref(hp[0])))


def muon_step_batched_host_grad(mats: Sequence[Matrix], hp, workspace, stream=None):
    """muon_step_batched with every G a pinned CPU tensor: the library streams the gradients
    in chunk by chunk, overlapping the copies with the step of earlier chunks."""
    for m in mats:
        if m.G.is_cuda or not m.G.is_pinned():
            raise ValueError("G must be a pinned CPU tensor (tensor.pin_memory())")
    st = _lib().muon_step_batched_host_grad(_descs(mats, g_on_host=True), len(mats), ctypes.byref(hp[0]),
                                            workspace.data_ptr(),
                                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "muon_step_batched_host_grad")


def ns_workspace_size(batch: int, rows: int, cols: int, schedule: Schedule) -> int:
    return int(_lib().ns_workspace_size(batch, rows, cols, ctypes.byref(schedule.c)))


def ns_orthogonalize(X_in, X_out, schedule: Schedule, workspace, stream=None):
    _need(X_in, "X_in")
    _need(X_out, "X_out", device=X_in.device)
    if X_in.dim() == 2:
        batch, (rows, cols) = 1, X_in.shape
    else:
        batch, rows, cols = X_in.shape
    if tuple(X_out.shape) != tuple(X_in.shape):
        raise ValueError("X_out must have X_in's shape")
    if not (X_in.is_contiguous() and X_out.is_contiguous()):
        raise ValueError("X_in and X_out must be contiguous")
    st = _lib().ns_orthogonalize(X_in.data_ptr(), _dtype_code(X_in), X_out.data_ptr(), _dtype_code(X_out),
                                 batch, rows, cols, ctypes.byref(schedule.c), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ns_orthogonalize")


def stiefel_workspace_size(batch: int, n: int, k: int) -> int:
    return int(_lib().stiefel_workspace_size(batch, n, k))


def stiefel_cayley_step(W, G, lr: float, workspace, stream=None):
    _need(W, "W")
    _need(G, "G", device=W.device)
    if W.dim() == 2:
        batch, (n, k) = 1, W.shape
    else:
        batch, n, k = W.shape
    if tuple(G.shape) != tuple(W.shape):
        raise ValueError("G must have W's shape")
    st = _lib().stiefel_cayley_step(W.data_ptr(), G.data_ptr(), batch, n, k, float(lr), workspace.data_ptr(),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "stiefel_cayley_step")


def frobenius_prescale_static(X_in, X_out, fp32_mode: bool = False, eps: float = 1e-7, scale_out=None,
                              stream=None):
    """X_out = X0 / (||X0||_F + eps) per matrix without a workspace: the library's fixed
    internal scratch is used instead (see muon_frobenius_prescale_static in the header)."""
    _need(X_in, "X_in")
    _need(X_out, "X_out", device=X_in.device)
    if X_in.dim() == 2:
        batch, (rows, cols) = 1, X_in.shape
    else:
        batch, rows, cols = X_in.shape
    if tuple(X_out.shape) != tuple(X_in.shape):
        raise ValueError("X_out must have X_in's shape")
    st = _lib().muon_frobenius_prescale_static(X_in.data_ptr(), _dtype_code(X_in), X_out.data_ptr(),
                                               _dtype_code(X_out), batch, rows, cols, int(bool(fp32_mode)),
                                               float(eps), scale_out.data_ptr() if scale_out is not None else None,
                                               _stream(stream))
    _check(st, "muon_frobenius_prescale_static")


def muon_cayley_workspace_size(batch: int, n: int, k: int) -> int:
    return int(_lib().muon_cayley_workspace_size(batch, n, k))


def muon_cayley_step(W, G, M, lr: float, beta: float, workspace, center: bool = True, stream=None):
    _need(W, "W")
    _need(G, "G", device=W.device)
    _need(M, "M", device=W.device)
    if W.dim() == 2:
        batch, (n, k) = 1, W.shape
    else:
        batch, n, k = W.shape
    if tuple(G.shape) != tuple(W.shape) or tuple(M.shape) != tuple(W.shape):
        raise ValueError("G and M must have W's shape")
    st = _lib().muon_cayley_step(W.data_ptr(), G.data_ptr(), M.data_ptr(), batch, n, k, float(lr), float(beta),
                                 int(bool(center)), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check(st, "muon_cayley_step")


def device_status(workspace, stream=None) -> int:
    out = c_int(-1)
    st = _lib().muon_workspace_device_status(workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                             ctypes.byref(out), _stream(stream))
    _check(st, "muon_workspace_device_status")
    return out.value


def timing_enable(on: bool = True):
    _check(_lib().muon_timing_enable(int(bool(on))), "muon_timing_enable")


def timing_reset():
    _check(_lib().muon_timing_reset(), "muon_timing_reset")


def timing_read(kind: str):
    ms, n, work = c_double(), c_longlong(), c_double()
    _check(_lib().muon_timing_read(KERNEL_KINDS[kind], ctypes.byref(ms), ctypes.byref(n), ctypes.byref(work)),
           "muon_timing_read")
    return ms.value, n.value, work.value


def workspace(nbytes: int, device=None):
    """A caller-owned workspace tensor of at least nbytes (allocated by torch)."""
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")
