"""Python binding of liblora_linear.so (argument marshalling only).

Every function has the name of its C entry point (include/lora_linear.h), takes
torch tensors that already live on the GPU, passes their pointers, sizes and the
current CUDA stream through ctypes, and raises LoraError on a non-OK status.  All
arithmetic runs in the library's CUDA kernels; there is no fallback: if the shared
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblora_linear.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lora_linear.h")

LORA_OK = 0
STATUS = {0: "LORA_OK", 1: "LORA_ERR_INVALID_ARG", 2: "LORA_ERR_MISALIGNED", 3: "LORA_ERR_UNSUPPORTED",
          4: "LORA_ERR_WORKSPACE", 5: "LORA_ERR_CUDA", 6: "LORA_ERR_TIMEOUT"}
OP_FWD, OP_BWD, OP_FWD_Q4, OP_BWD_Q4, OP_FWD_FP8, OP_BWD_FP8, OP_FWD_NF4, OP_BWD_NF4 = 0, 1, 2, 3, 4, 5, 6, 7
KERNEL_KINDS = ["xa", "fwd_main", "g", "dx_main", "dadb"]


class LoraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({lora_status_string(status)})")


_lib = None


def load_library():
    """Load the in-tree CUDA library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run rank_linear_lora_b200/build.py)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I, F, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.lora_linear_workspace_size.argtypes = [I, I64, I64, I64, I]
    lib.lora_linear_workspace_size.restype = SZ
    lib.lora_linear_fwd.argtypes = [P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    lib.lora_linear_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    lib.lora_linear_fwd_q4.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    lib.lora_linear_bwd_q4.argtypes = [P, P, P, P, P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    lib.lora_linear_fwd_fp8.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    lib.lora_linear_fwd_nf4.argtypes = [P, P, P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    lib.lora_linear_bwd_nf4.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    lib.lora_linear_bwd_fp8.argtypes = [P, P, P, P, P, P, P, P, P, P, I64, I64, I64, I, F, P, SZ, P]
    for f in ("lora_linear_fwd", "lora_linear_bwd", "lora_linear_fwd_q4", "lora_linear_bwd_q4", "lora_linear_fwd_fp8",
              "lora_linear_bwd_fp8", "lora_linear_fwd_nf4", "lora_linear_bwd_nf4"):
        getattr(lib, f).restype = I
    lib.lora_linear_check.argtypes = [P, P]
    lib.lora_linear_check.restype = I
    lib.lora_status_string.argtypes = [I]
    lib.lora_status_string.restype = ctypes.c_char_p
    lib.lora_linear_launch_count.restype = I64
    lib.lora_linear_timing_enable.argtypes = [I]
    lib.lora_linear_timing_enable.restype = I
    lib.lora_linear_timing_read.argtypes = [P, P, I]
    lib.lora_linear_timing_read.restype = I
    lib.lora_linear_trace_enable.argtypes = [P, SZ]
    lib.lora_linear_trace_enable.restype = I
    _lib = lib
    return lib


def declared_functions() -> list[str]:
    """Names of the functions include/lora_linear.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^LORA_API\s+[a-z_0-9 ]+?\*?\s*(lora_[a-z_0-9]+)\s*\(", text, re.M)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    elif stream.device_index != torch.cuda.current_device():
        raise ValueError(f"stream is on cuda:{stream.device_index}, the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(stream.cuda_stream)


def _on_current_device(t, name):
    """The library works on the current device: every tensor must live there."""
    if not t.is_cuda or t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name}: on {t.device}, the current device is cuda:{torch.cuda.current_device()}")


def _ws(ws):
    """(pointer, bytes) of a workspace tensor: contiguous, on the current device."""
    if ws is None or not ws.is_contiguous():
        raise ValueError("workspace: expected a contiguous CUDA tensor")
    _on_current_device(ws, "workspace")
    return _ptr(ws), ws.numel() * ws.element_size()


def _check(status: int, where: str):
    if status != LORA_OK:
        raise LoraError(status, where)


def _bf16(t, name, shape):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected a contiguous CUDA bfloat16 tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")
    _on_current_device(t, name)


def _f32(t, name, shape):
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected a contiguous CUDA float32 tensor of shape {tuple(shape)}")
    _on_current_device(t, name)


def lora_status_string(status: int) -> str:
    return load_library().lora_status_string(int(status)).decode()


def lora_linear_workspace_size(op: int, M: int, d_in: int, d_out: int, r: int) -> int:
    return int(load_library().lora_linear_workspace_size(op, M, d_in, d_out, r))


def workspace(op: int, M: int, d_in: int, d_out: int, r: int, device=None) -> torch.Tensor:
    """A zeroed uint8 workspace of the size the library asks for (torch allocates)."""
    n = lora_linear_workspace_size(op, M, d_in, d_out, r)
    if n == 0:
        raise ValueError("invalid sizes for the workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def lora_linear_fwd(x, W, A, B, h, xa_save, alpha, ws, stream=None):
    M, d_in = x.shape
    r = A.shape[0]
    d_out = W.shape[0]
    for t, n, s in ((x, "x", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)),
                    (h, "h", (M, d_out))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    st = load_library().lora_linear_fwd(_ptr(x), _ptr(W), _ptr(A), _ptr(B), _ptr(h), _ptr(xa_save), M, d_in, d_out,
                                        r, float(alpha), *_ws(ws), _stream(stream))
    _check(st, "lora_linear_fwd")


def lora_linear_bwd(dY, x, W, A, B, xa_save, dX, dA, dB, alpha, ws, stream=None):
    M, d_in = x.shape
    r = A.shape[0]
    d_out = W.shape[0]
    for t, n, s in ((dY, "dY", (M, d_out)), (x, "x", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)),
                    (B, "B", (d_out, r))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    if dX is not None:
        _bf16(dX, "dX", (M, d_in))
    _f32(dA, "dA", (r, d_in))
    _f32(dB, "dB", (d_out, r))
    st = load_library().lora_linear_bwd(_ptr(dY), _ptr(x), _ptr(W), _ptr(A), _ptr(B), _ptr(xa_save), _ptr(dX),
                                        _ptr(dA), _ptr(dB), M, d_in, d_out, r, float(alpha), *_ws(ws),
                                        _stream(stream))
    _check(st, "lora_linear_bwd")


def _q4(Wq, Wscale, d_out, d_in):
    if Wq.dtype != torch.uint8 or not Wq.is_cuda or not Wq.is_contiguous() or tuple(Wq.shape) != (d_out, d_in // 2):
        raise ValueError(f"Wq: expected a contiguous CUDA uint8 tensor of shape {(d_out, d_in // 2)}")
    _on_current_device(Wq, "Wq")
    _bf16(Wscale, "Wscale", (d_out, d_in // 64))


def lora_linear_fwd_q4(x, Wq, Wscale, A, B, h, xa_save, alpha, ws, stream=None):
    M, d_in = x.shape
    r = A.shape[0]
    d_out = Wq.shape[0]
    _q4(Wq, Wscale, d_out, d_in)
    for t, n, s in ((x, "x", (M, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)), (h, "h", (M, d_out))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    st = load_library().lora_linear_fwd_q4(_ptr(x), _ptr(Wq), _ptr(Wscale), _ptr(A), _ptr(B), _ptr(h),
                                           _ptr(xa_save), M, d_in, d_out, r, float(alpha), *_ws(ws),
                                           _stream(stream))
    _check(st, "lora_linear_fwd_q4")


def lora_linear_bwd_q4(dY, x, Wq, Wscale, A, B, xa_save, dX, dA, dB, alpha, ws, stream=None):
    M, d_in = x.shape
    r = A.shape[0]
    d_out = Wq.shape[0]
    _q4(Wq, Wscale, d_out, d_in)
    for t, n, s in ((dY, "dY", (M, d_out)), (x, "x", (M, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    if dX is not None:
        _bf16(dX, "dX", (M, d_in))
    _f32(dA, "dA", (r, d_in))
    _f32(dB, "dB", (d_out, r))
    st = load_library().lora_linear_bwd_q4(_ptr(dY), _ptr(x), _ptr(Wq), _ptr(Wscale), _ptr(A), _ptr(B),
                                           _ptr(xa_save), _ptr(dX), _ptr(dA), _ptr(dB), M, d_in, d_out, r,
                                           float(alpha), *_ws(ws), _stream(stream))
    _check(st, "lora_linear_bwd_q4")


def _fp8(W8, W8scale, d_out, d_in):
    if W8.dtype != torch.uint8 or not W8.is_cuda or not W8.is_contiguous() or tuple(W8.shape) != (d_out, d_in):
        raise ValueError(f"W8: expected a contiguous CUDA uint8 tensor of shape {(d_out, d_in)} (E4M3 codes)")
    _on_current_device(W8, "W8")
    _bf16(W8scale, "W8scale", (d_out,))


def lora_linear_fwd_fp8(x, W8, W8scale, A, B, h, xa_save, alpha, ws, stream=None):
    M, d_in = x.shape
    r = A.shape[0]
    d_out = W8.shape[0]
    _fp8(W8, W8scale, d_out, d_in)
    for t, n, s in ((x, "x", (M, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)), (h, "h", (M, d_out))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    st = load_library().lora_linear_fwd_fp8(_ptr(x), _ptr(W8), _ptr(W8scale), _ptr(A), _ptr(B), _ptr(h),
                                            _ptr(xa_save), M, d_in, d_out, r, float(alpha), *_ws(ws),
                                            _stream(stream))
    _check(st, "lora_linear_fwd_fp8")


def lora_linear_bwd_fp8(dY, x, W8, W8scale, A, B, xa_save, dX, dA, dB, alpha, ws, stream=None):
    M, d_in = x.shape
    r = A.shape[0]
    d_out = W8.shape[0]
    _fp8(W8, W8scale, d_out, d_in)
    for t, n, s in ((dY, "dY", (M, d_out)), (x, "x", (M, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    if dX is not None:
        _bf16(dX, "dX", (M, d_in))
    _f32(dA, "dA", (r, d_in))
    _f32(dB, "dB", (d_out, r))
    st = load_library().lora_linear_bwd_fp8(_ptr(dY), _ptr(x), _ptr(W8), _ptr(W8scale), _ptr(A), _ptr(B),
                                            _ptr(xa_save), _ptr(dX), _ptr(dA), _ptr(dB), M, d_in, d_out, r,
                                            float(alpha), *_ws(ws), _stream(stream))
    _check(st, "lora_linear_bwd_fp8")


class lora_plan_t(ctypes.Structure):
    """The plan of one layer shape (include/lora_linear.h); 0 = the library's choice."""
    _fields_ = [("side_fwd", ctypes.c_int32), ("side_bwd", ctypes.c_int32), ("xa_cluster", ctypes.c_int32),
                ("g_cluster", ctypes.c_int32), ("g_group", ctypes.c_int32), ("da_cluster", ctypes.c_int32),
                ("fwd_tail", ctypes.c_int32), ("dx_overlap", ctypes.c_int32), ("splitk", ctypes.c_int32 * 4)]

    FIELDS = ("side_fwd", "side_bwd", "xa_cluster", "g_cluster", "g_group", "da_cluster", "fwd_tail", "dx_overlap")

    def as_dict(self) -> dict:
        d = {k: int(getattr(self, k)) for k in self.FIELDS}
        d["splitk"] = [int(v) for v in self.splitk]
        return d

    @classmethod
    def from_dict(cls, d: dict) -> "lora_plan_t":
        p = cls()
        for k in cls.FIELDS:
            setattr(p, k, int(d.get(k, 0)))
        for i, v in enumerate(d.get("splitk", [0, 0, 0, 0])):
            p.splitk[i] = int(v)
        return p


def lora_linear_set_plan(M: int, d_in: int, d_out: int, r: int, plan):
    """Install a plan (a lora_plan_t or a dict of its fields) for this shape; None removes it."""
    fn = load_library().lora_linear_set_plan
    fn.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    if plan is None:
        _check(fn(M, d_in, d_out, r, None), "lora_linear_set_plan")
        return
    p = plan if isinstance(plan, lora_plan_t) else lora_plan_t.from_dict(plan)
    _check(fn(M, d_in, d_out, r, ctypes.byref(p)), "lora_linear_set_plan")


def lora_linear_get_plan(op: int, M: int, d_in: int, d_out: int, r: int) -> dict:
    """The plan `op` uses for this shape, as a dict of lora_plan_t's fields."""
    fn = load_library().lora_linear_get_plan
    fn.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    p = lora_plan_t()
    _check(fn(op, M, d_in, d_out, r, ctypes.byref(p)), "lora_linear_get_plan")
    return p.as_dict()


def _codebook(codebook):
    """16 host float32 values (any sequence; a CUDA tensor is copied to the host)."""
    import numpy as np
    cb = codebook.detach().cpu().numpy() if isinstance(codebook, torch.Tensor) else codebook
    cb = np.ascontiguousarray(np.asarray(cb, dtype=np.float32).reshape(-1))
    if cb.shape != (16,):
        raise ValueError("codebook: expected 16 values")
    return cb, cb.ctypes.data_as(ctypes.c_void_p)


def lora_linear_fwd_nf4(x, Wq, Wscale, codebook, A, B, h, xa_save, alpha, ws, stream=None):
    """Forward with a 4-bit codebook weight (e.g. NF4): w' = codebook[q] * Wscale[n, k/64]."""
    M, d_in = x.shape
    r = A.shape[0]
    d_out = Wq.shape[0]
    _q4(Wq, Wscale, d_out, d_in)
    for t, n, s in ((x, "x", (M, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)), (h, "h", (M, d_out))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    keep, cbp = _codebook(codebook)
    st = load_library().lora_linear_fwd_nf4(_ptr(x), _ptr(Wq), _ptr(Wscale), cbp, _ptr(A), _ptr(B), _ptr(h),
                                            _ptr(xa_save), M, d_in, d_out, r, float(alpha), *_ws(ws),
                                            _stream(stream))
    del keep
    _check(st, "lora_linear_fwd_nf4")


def lora_linear_bwd_nf4(dY, x, Wq, Wscale, codebook, A, B, xa_save, dX, dA, dB, alpha, ws, stream=None):
    M, d_in = x.shape
    r = A.shape[0]
    d_out = Wq.shape[0]
    _q4(Wq, Wscale, d_out, d_in)
    for t, n, s in ((dY, "dY", (M, d_out)), (x, "x", (M, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    if dX is not None:
        _bf16(dX, "dX", (M, d_in))
    _f32(dA, "dA", (r, d_in))
    _f32(dB, "dB", (d_out, r))
    keep, cbp = _codebook(codebook)
    st = load_library().lora_linear_bwd_nf4(_ptr(dY), _ptr(x), _ptr(Wq), _ptr(Wscale), cbp, _ptr(A), _ptr(B),
                                            _ptr(xa_save), _ptr(dX), _ptr(dA), _ptr(dB), M, d_in, d_out, r,
                                            float(alpha), *_ws(ws), _stream(stream))
    del keep
    _check(st, "lora_linear_bwd_nf4")


def lora_linear_check(ws, stream=None):
    ptr = None if ws is None else _ws(ws)[0]  # no workspace: only wait for the stream
    _check(load_library().lora_linear_check(ptr, _stream(stream)), "lora_linear_check")


def lora_linear_merge(W, A, B, W_out, alpha, stream=None):
    """W_out = W + (alpha / r) * B . A in bf16 (W_out may be W: in place)."""
    d_out, d_in = W.shape
    r = A.shape[0]
    for t, n, s in ((W, "W", (d_out, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)), (W_out, "W_out", (d_out, d_in))):
        _bf16(t, n, s)
    fn = load_library().lora_linear_merge
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, I64, I64, I, F, P]
    fn.restype = I
    _check(fn(_ptr(W), _ptr(A), _ptr(B), _ptr(W_out), d_in, d_out, r, float(alpha), _stream(stream)),
           "lora_linear_merge")


def lora_linear_merge_q4(Wq, Wscale, A, B, W_out, alpha, stream=None):
    """W_out = decode(Wq, Wscale) + (alpha / r) * B . A in bf16."""
    d_out = Wq.shape[0]
    r, d_in = A.shape
    _q4(Wq, Wscale, d_out, d_in)
    for t, n, s in ((A, "A", (r, d_in)), (B, "B", (d_out, r)), (W_out, "W_out", (d_out, d_in))):
        _bf16(t, n, s)
    fn = load_library().lora_linear_merge_q4
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, P, I64, I64, I, F, P]
    fn.restype = I
    _check(fn(_ptr(Wq), _ptr(Wscale), _ptr(A), _ptr(B), _ptr(W_out), d_in, d_out, r, float(alpha), _stream(stream)),
           "lora_linear_merge_q4")


def lora_linear_merge_fp8(W8, W8scale, A, B, W_out, alpha, stream=None):
    """W_out = e4m3(W8) * W8scale[row] + (alpha / r) * B . A in bf16."""
    d_out, d_in = W8.shape
    r = A.shape[0]
    _fp8(W8, W8scale, d_out, d_in)
    for t, n, s in ((A, "A", (r, d_in)), (B, "B", (d_out, r)), (W_out, "W_out", (d_out, d_in))):
        _bf16(t, n, s)
    fn = load_library().lora_linear_merge_fp8
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, P, I64, I64, I, F, P]
    fn.restype = I
    _check(fn(_ptr(W8), _ptr(W8scale), _ptr(A), _ptr(B), _ptr(W_out), d_in, d_out, r, float(alpha),
              _stream(stream)), "lora_linear_merge_fp8")


def lora_linear_merge_nf4(Wq, Wscale, codebook, A, B, W_out, alpha, stream=None):
    """W_out = codebook[Wq] * Wscale[n, k/64] + (alpha / r) * B . A in bf16."""
    d_out = Wq.shape[0]
    r, d_in = A.shape
    _q4(Wq, Wscale, d_out, d_in)
    for t, n, s in ((A, "A", (r, d_in)), (B, "B", (d_out, r)), (W_out, "W_out", (d_out, d_in))):
        _bf16(t, n, s)
    keep, cbp = _codebook(codebook)
    fn = load_library().lora_linear_merge_nf4
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, P, P, I64, I64, I, F, P]
    fn.restype = I
    st = fn(_ptr(Wq), _ptr(Wscale), cbp, _ptr(A), _ptr(B), _ptr(W_out), d_in, d_out, r, float(alpha),
            _stream(stream))
    del keep
    _check(st, "lora_linear_merge_nf4")


def lora_linear_merge_check(stream=None):
    fn = load_library().lora_linear_merge_check
    fn.argtypes = [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(_stream(stream)), "lora_linear_merge_check")


def lora_linear_selftest_timeout(ws, limit_us: int = 1000, stream=None):
    """Enqueue the failure-path self-test on the workspace's error word (a bounded wait
    that runs out after limit_us); lora_linear_check then raises LORA_ERR_TIMEOUT."""
    lib = load_library()
    fn = lib.lora_linear_selftest_timeout
    fn.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(*_ws(ws), int(limit_us), _stream(stream)),
           "lora_linear_selftest_timeout")


def lora_linear_launch_count() -> int:
    return int(load_library().lora_linear_launch_count())


def lora_linear_timing_enable(on: bool):
    _check(load_library().lora_linear_timing_enable(1 if on else 0), "lora_linear_timing_enable")


def lora_linear_timing_read():
    """{kind: (total_ms, launches)} for every kernel kind since the last read."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(load_library().lora_linear_timing_read(ms, cnt, n), "lora_linear_timing_read")
    return {k: (ms[i], int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}


TRACE_WORDS = 32
TRACE_FIELDS = ["entry", "setup", "prod_end", "mma_end", "epi_end", "exit", "smid", "tiles"]


def lora_linear_trace_enable(buf):
    """Trace into a CUDA int64 tensor (None switches tracing off)."""
    if buf is None:
        _check(load_library().lora_linear_trace_enable(None, 0), "lora_linear_trace_enable")
    else:
        _check(load_library().lora_linear_trace_enable(_ptr(buf), buf.numel() * buf.element_size()),
               "lora_linear_trace_enable")


def lora_linear_fwd_noalloc(x, W, A, B, h, xa_save, alpha, stream=None):
    """Forward without a workspace, for callers that cannot allocate device memory
    (the library's fixed 4 MiB device scratch is used instead; see the header for the
    size limit and for why concurrent calls must not overlap)."""
    lib = load_library()
    fn = lib.lora_linear_fwd_noalloc
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, P, P, I64, I64, I64, I, F, P]
    fn.restype = I
    M, d_in = x.shape
    r = A.shape[0]
    d_out = W.shape[0]
    for t, n, s in ((x, "x", (M, d_in)), (W, "W", (d_out, d_in)), (A, "A", (r, d_in)), (B, "B", (d_out, r)),
                    (h, "h", (M, d_out))):
        _bf16(t, n, s)
    if xa_save is not None:
        _bf16(xa_save, "xa_save", (M, r))
    st = fn(_ptr(x), _ptr(W), _ptr(A), _ptr(B), _ptr(h), _ptr(xa_save), M, d_in, d_out, r, float(alpha),
            _stream(stream))
    _check(st, "lora_linear_fwd_noalloc")


def lora_linear_noalloc_check(stream=None):
    """Wait for the stream, then read and clear the workspace-free forward's device error
    word (raises LoraError LORA_ERR_TIMEOUT if a bounded wait of an earlier call ran out)."""
    fn = load_library().lora_linear_noalloc_check
    fn.argtypes = [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(_stream(stream)), "lora_linear_noalloc_check")


def lora_linear_noalloc_selftest_timeout(limit_us: int = 1000, stream=None):
    """Enqueue the failure-path self-test on the workspace-free forward's error word."""
    fn = load_library().lora_linear_noalloc_selftest_timeout
    fn.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(int(limit_us), _stream(stream)), "lora_linear_noalloc_selftest_timeout")
