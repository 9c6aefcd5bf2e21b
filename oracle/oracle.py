"""ctypes front of oracle.c (fp64 CPU reference; test infrastructure only).

Inputs are numpy arrays of bf16 bit patterns (uint16).  A frozen weight is W (bf16),
or the 4-bit code Wq (uint8, two codes per byte along d_in, low nibble = even index)
with bf16 scales Wscale per 64-element block, or FP8 E4M3 codes W8 (uint8, one per
element) with a bf16 scale W8scale per row.  Results are fp64 numpy arrays.  Each
function is one step of the layer's definition (see oracle.c for the formulas and the
passages they follow).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def lib_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (IEEE fp64: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P, I64, D, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_int
        lib.oracle_threads.restype = I
        lib.oracle_set_codebook.argtypes = [P]
        lib.oracle_set_threads.argtypes = [I]
        lib.oracle_weight.argtypes = [I, P, P, P, I64, I64, P]
        lib.oracle_xa.argtypes = [P, P, I64, I64, I64, P]
        lib.oracle_h.argtypes = [P, I, P, P, P, P, P, D, I64, I64, I64, I64, P, I64, P]
        lib.oracle_g.argtypes = [P, P, I64, I64, I64, P]
        lib.oracle_dx.argtypes = [P, I, P, P, P, P, P, D, I64, I64, I64, I64, P, I64, P]
        lib.oracle_db.argtypes = [P, P, D, I64, I64, I64, P]
        lib.oracle_da.argtypes = [P, P, D, I64, I64, I64, P]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def threads() -> int:
    return _load().oracle_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def _wargs(W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None):
    if W is not None:
        return 0, _u16(W), None, None
    if W8 is not None:
        return 2, None, np.ascontiguousarray(W8, dtype=np.uint8), _u16(W8scale)
    if codebook is not None:
        cb = np.ascontiguousarray(codebook, dtype=np.float64)
        if cb.shape != (16,):
            raise ValueError("codebook: 16 values")
        _load().oracle_set_codebook(cb.ctypes.data_as(ctypes.c_void_p))
        return 3, None, np.ascontiguousarray(Wq, dtype=np.uint8), _u16(Wscale)
    return 1, None, np.ascontiguousarray(Wq, dtype=np.uint8), _u16(Wscale)


def weight(d_out, d_in, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None) -> np.ndarray:
    fmt, w, q, sc = _wargs(W, Wq, Wscale, W8, W8scale, codebook)
    out = np.empty((d_out, d_in), dtype=np.float64)
    _load().oracle_weight(fmt, _p(w), _p(q), _p(sc), d_out, d_in, _p(out))
    return out


def xa(x, A) -> np.ndarray:
    """Step 1: xa = x . A^T, [M, r]."""
    x, A = _u16(x), _u16(A)
    M, d_in = x.shape
    r = A.shape[0]
    out = np.empty((M, r), dtype=np.float64)
    _load().oracle_xa(_p(x), _p(A), M, d_in, r, _p(out))
    return out


def h(x, B, xa_, s, *, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None,
      rows=None) -> np.ndarray:
    """Step 2: h = x . W^T + s * xa . B^T for all rows, or only ``rows``."""
    x, B = _u16(x), _u16(B)
    M, d_in = x.shape
    d_out, r = B.shape
    xa_ = np.ascontiguousarray(xa_, dtype=np.float64)
    fmt, w, q, sc = _wargs(W, Wq, Wscale, W8, W8scale, codebook)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = M if rr is None else len(rr)
    out = np.empty((n, d_out), dtype=np.float64)
    _load().oracle_h(_p(x), fmt, _p(w), _p(q), _p(sc), _p(B), _p(xa_), float(s), M, d_in, d_out, r,
                     _p(rr), n, _p(out))
    return out


def g(dY, B) -> np.ndarray:
    """Step 3: g = dY . B, [M, r]."""
    dY, B = _u16(dY), _u16(B)
    M, d_out = dY.shape
    r = B.shape[1]
    out = np.empty((M, r), dtype=np.float64)
    _load().oracle_g(_p(dY), _p(B), M, d_out, r, _p(out))
    return out


def dx(dY, A, g_, s, *, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None,
       rows=None) -> np.ndarray:
    """Step 4: dX = dY . W + s * g . A for all rows, or only ``rows``."""
    dY, A = _u16(dY), _u16(A)
    M, d_out = dY.shape
    r, d_in = A.shape
    g_ = np.ascontiguousarray(g_, dtype=np.float64)
    fmt, w, q, sc = _wargs(W, Wq, Wscale, W8, W8scale, codebook)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = M if rr is None else len(rr)
    out = np.empty((n, d_in), dtype=np.float64)
    _load().oracle_dx(_p(dY), fmt, _p(w), _p(q), _p(sc), _p(A), _p(g_), float(s), M, d_in, d_out, r,
                      _p(rr), n, _p(out))
    return out


def db(dY, xa_, s) -> np.ndarray:
    """Step 5: dB = s * dY^T . xa, [d_out, r]."""
    dY = _u16(dY)
    M, d_out = dY.shape
    xa_ = np.ascontiguousarray(xa_, dtype=np.float64)
    r = xa_.shape[1]
    out = np.empty((d_out, r), dtype=np.float64)
    _load().oracle_db(_p(dY), _p(xa_), float(s), M, d_out, r, _p(out))
    return out


def da(x, g_, s) -> np.ndarray:
    """Step 6: dA = s * g^T . x, [r, d_in]."""
    x = _u16(x)
    M, d_in = x.shape
    g_ = np.ascontiguousarray(g_, dtype=np.float64)
    r = g_.shape[1]
    out = np.empty((r, d_in), dtype=np.float64)
    _load().oracle_da(_p(x), _p(g_), float(s), M, d_in, r, _p(out))
    return out


def forward(x, A, B, s, *, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None, rows=None):
    """Steps 1-2.  Returns (h, xa)."""
    xa_ = xa(x, A)
    return h(x, B, xa_, s, W=W, Wq=Wq, Wscale=Wscale, W8=W8, W8scale=W8scale, codebook=codebook, rows=rows), xa_


def backward(dY, x, A, B, s, *, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None, rows=None,
             xa_=None):
    """Steps 1, 3-6.  Returns dict with dX (all rows or ``rows``), dA, dB, g, xa."""
    if xa_ is None:
        xa_ = xa(x, A)
    g_ = g(dY, B)
    return {
        "dX": dx(dY, A, g_, s, W=W, Wq=Wq, Wscale=Wscale, W8=W8, W8scale=W8scale, codebook=codebook, rows=rows),
        "dA": da(x, g_, s),
        "dB": db(dY, xa_, s),
        "g": g_,
        "xa": xa_,
    }


# ------------------------------------------------------------------ projections
# Properties of steps 2 and 4 that hold at any size: a projection of h (or dX) on a
# vector follows from the definition by associativity, and costs O(M d) instead of
# O(M d_in d_out).  Checking every row projection and every column projection of a
# GPU result touches every element of it.  The weight is dequantised (oracle_weight,
# the same rule as steps 2 and 4) a block of rows at a time, never as a whole.

def _f64(bits) -> np.ndarray:
    """bf16 bit patterns -> fp64 (exact)."""
    return (_u16(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _weight_blocks(d_out, d_in, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, rows=2048, codebook=None):
    """(n0, fp64 rows n0 .. n0+k) of the dequantised weight, block by block."""
    for n0 in range(0, d_out, rows):
        n1 = min(d_out, n0 + rows)
        if W is not None:
            yield n0, weight(n1 - n0, d_in, W=_u16(W)[n0:n1])
        elif W8 is not None:
            yield n0, weight(n1 - n0, d_in, W8=np.ascontiguousarray(W8)[n0:n1], W8scale=_u16(W8scale)[n0:n1])
        else:
            yield n0, weight(n1 - n0, d_in, Wq=np.ascontiguousarray(Wq)[n0:n1], Wscale=_u16(Wscale)[n0:n1],
                             codebook=codebook)


def h_projections(x, A, B, s, v, u, *, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None,
                  xa_=None, block_rows=2048):
    """Step 2 projected: (h . v [M], u^T . h [d_out]) for v [d_out], u [M], with
    h . v = x . (W^T v) + s * xa . (B^T v) and u^T . h = W (x^T u) + s * B (xa^T u)."""
    M, d_in = np.shape(x)
    d_out = np.shape(B)[0]
    xa_ = xa(x, A) if xa_ is None else xa_
    xf, Bf = _f64(x), _f64(B)
    wt_v = np.zeros(d_in)
    xt_u = xf.T @ u
    col = np.empty(d_out)
    for n0, Wb in _weight_blocks(d_out, d_in, W, Wq, Wscale, W8, W8scale, rows=block_rows, codebook=codebook):
        wt_v += Wb.T @ v[n0:n0 + len(Wb)]
        col[n0:n0 + len(Wb)] = Wb @ xt_u
    row = xf @ wt_v + s * (xa_ @ (Bf.T @ v))
    col += s * (Bf @ (xa_.T @ u))
    return row, col


def dx_projections(dY, A, B, s, v, u, *, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None,
                   g_=None, block_rows=2048):
    """Step 4 projected: (dX . v [M], u^T . dX [d_in]) for v [d_in], u [M], with
    dX . v = dY . (W v) + s * g . (A v) and u^T . dX = (dY^T u)^T W + s * (g^T u)^T A."""
    M, d_out = np.shape(dY)
    d_in = np.shape(A)[1]
    g_ = g(dY, B) if g_ is None else g_
    dYf, Af = _f64(dY), _f64(A)
    w_v = np.empty(d_out)
    dyt_u = dYf.T @ u
    col = np.zeros(d_in)
    for n0, Wb in _weight_blocks(d_out, d_in, W, Wq, Wscale, W8, W8scale, rows=block_rows, codebook=codebook):
        w_v[n0:n0 + len(Wb)] = Wb @ v
        col += dyt_u[n0:n0 + len(Wb)] @ Wb
    row = dYf @ w_v + s * (g_ @ (Af @ v))
    col += s * ((g_.T @ u) @ Af)
    return row, col


def merged_weight(A, B, s, *, W=None, Wq=None, Wscale=None, W8=None, W8scale=None, codebook=None) -> np.ndarray:
    """The merged weight of step 2, W + s * B . A, in fp64 [d_out, d_in]: the weight for
    which h = x . (W + s B A)^T (the adapter folded in for deployment).  The 4-bit weight
    is decoded by the same rule as steps 2 and 4."""
    d_out, d_in = np.shape(B)[0], np.shape(A)[1]
    return weight(d_out, d_in, W=W, Wq=Wq, Wscale=Wscale, W8=W8, W8scale=W8scale, codebook=codebook) + s * (
        _f64(B) @ _f64(A))


# ------------------------------------------------------------------ whole tensors at full size
# Steps 2 and 4 for a block of token rows, with numpy's fp64 matrix product (a library
# primitive) as the summation step in place of oracle.c's loops.  The inputs are the
# same exact fp64 widenings and the weight is dequantised by oracle.c's own rule
# (weight()); only the order of the fp64 additions differs from oracle.c, which puts
# the two within ~1e-13 of each other (pinned in the CPU tests).  This is what lets
# the tests compare every element of h and dX of the full-size workloads (up to 2e12
# multiply-adds per output) in seconds rather than the minutes oracle.c's plain loops
# take on the host cores.

def h_dense(x, B, xa_, s, Wf) -> np.ndarray:
    """Step 2 for the given token rows: h = x . Wf^T + s * xa . B^T, with Wf the fp64
    weight [d_out, d_in] from weight() and xa_ the fp64 step-1 rows of the same tokens."""
    return _f64(x) @ np.asarray(Wf, dtype=np.float64).T + s * (np.asarray(xa_, dtype=np.float64) @ _f64(B).T)


def dx_dense(dY, A, g_, s, Wf) -> np.ndarray:
    """Step 4 for the given token rows: dX = dY . Wf + s * g . A, with Wf the fp64 weight
    [d_out, d_in] from weight() and g_ the fp64 step-3 rows of the same tokens."""
    return _f64(dY) @ np.asarray(Wf, dtype=np.float64) + s * (np.asarray(g_, dtype=np.float64) @ _f64(A))
