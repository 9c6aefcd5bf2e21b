"""The C ABI on the CPU: the library loads, exports every declared symbol, sizes
workspaces, and rejects bad arguments before touching a device."""
import ctypes

import pytest

from rank_linear_lora_b200 import build as B
from rank_linear_lora_b200 import lora_linear as L


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load_library()


def test_exports_every_declared_symbol(lib):
    names = L.declared_functions()
    expected = {"lora_linear_workspace_size", "lora_linear_fwd", "lora_linear_bwd", "lora_linear_fwd_q4",
                "lora_linear_bwd_q4", "lora_linear_check", "lora_status_string", "lora_linear_launch_count",
                "lora_linear_timing_enable", "lora_linear_timing_read"}
    assert expected <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(7):
        s = L.lora_status_string(code)
        assert isinstance(s, str) and s
    assert L.lora_status_string(99) == "unknown status"


def test_workspace_sizes(lib):
    for op in (L.OP_FWD, L.OP_BWD, L.OP_FWD_Q4, L.OP_BWD_Q4):
        assert L.lora_linear_workspace_size(op, 4096, 8192, 28672, 16) > 0
    # the bf16 forward holds the K-split hand-over buffer when its last wave is cut along K
    # (34 tail tiles of 256 x 256 fp32 at 4096 x 4096 x 4096); the 4-bit forward does not
    assert L.lora_linear_workspace_size(L.OP_FWD, 4096, 4096, 4096, 8) >= 34 * 256 * 256 * 4
    assert L.lora_linear_workspace_size(L.OP_BWD, 4096, 4096, 4096, 8) > L.lora_linear_workspace_size(
        L.OP_FWD_Q4, 4096, 4096, 4096, 8)
    assert L.lora_linear_get_plan(L.OP_FWD, 4096, 4096, 4096, 8)["fwd_tail"] == 3
    assert L.lora_linear_get_plan(L.OP_FWD_Q4, 4096, 4096, 4096, 8)["fwd_tail"] == 1
    # invalid sizes -> 0
    assert L.lora_linear_workspace_size(L.OP_FWD, 0, 256, 256, 8) == 0
    assert L.lora_linear_workspace_size(L.OP_FWD, 64, 250, 256, 8) == 0
    assert L.lora_linear_workspace_size(L.OP_FWD, 64, 256, 256, 12) == 0
    assert L.lora_linear_workspace_size(L.OP_FWD, 64, 256, 256, 264) == 0
    assert L.lora_linear_workspace_size(L.OP_FWD_Q4, 64, 96, 256, 8) == 0
    assert L.lora_linear_workspace_size(8, 64, 256, 256, 8) == 0


def _fwd(lib, x=0x1000, W=0x2000, A=0x3000, B_=0x4000, h=0x5000, xa=None, M=64, di=256, do=256, r=8,
         alpha=16.0, ws=0x10000, nws=1 << 30):
    P = ctypes.c_void_p
    return lib.lora_linear_fwd(P(x), P(W), P(A), P(B_), P(h), P(xa), M, di, do, r, alpha, P(ws), nws, None)


def test_validation_before_any_device_work(lib):
    """Every case below fails validation, so no pointer is ever dereferenced."""
    assert _fwd(lib, x=None) == 1
    assert _fwd(lib, h=None) == 1
    assert _fwd(lib, M=0) == 1
    assert _fwd(lib, di=250) == 1
    assert _fwd(lib, r=0) == 1
    assert _fwd(lib, r=12) == 1
    assert _fwd(lib, alpha=float("nan")) == 1
    assert _fwd(lib, M=(1 << 30) + 1) == 1
    assert _fwd(lib, di=(1 << 24) + 8) == 1
    assert _fwd(lib, M=1 << 30, di=1 << 24) == 1   # 2^22 x 2^17 tiles: past 32-bit counts
    # the bound itself: 2^23 x 255 tiles pass, 2^23 x 256 = 2^31 do not
    assert L.lora_linear_workspace_size(L.OP_FWD, 1 << 30, 32640, 32640, 8) > 0
    assert L.lora_linear_workspace_size(L.OP_FWD, 1 << 30, 32768, 64, 8) == 0
    assert _fwd(lib, x=0x1008) == 2
    assert _fwd(lib, xa=0x6004) == 2
    P = ctypes.c_void_p
    st = lib.lora_linear_bwd(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), None, None, None, P(0x7000),
                             64, 256, 256, 8, 16.0, P(0x10000), 1 << 30, None)
    assert st == 1  # dA is required


def test_selftest_timeout_argument_checks(lib):
    """The failure-path self-test rejects bad arguments on the host, before any launch."""
    fn = lib.lora_linear_selftest_timeout
    fn.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    P = ctypes.c_void_p
    assert fn(None, 1024, 1000, None) == 4           # LORA_ERR_WORKSPACE
    assert fn(P(0x1000), 2, 1000, None) == 4         # smaller than the error word
    assert fn(P(0x1004), 1024, 1000, None) == 2      # LORA_ERR_MISALIGNED
    assert fn(P(0x1000), 1024, 0, None) == 1         # LORA_ERR_INVALID_ARG
    assert fn(P(0x1000), 1024, 2000001, None) == 1


def test_merge_argument_checks(lib):
    """The deploy-time merge validates before touching a device: null or misaligned
    pointers (every one, B and the 4-bit scales included), shapes, r and alpha."""
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    mg = lib.lora_linear_merge
    mg.argtypes = [P, P, P, P, I64, I64, I, F, P]
    mg.restype = I
    mq = lib.lora_linear_merge_q4
    mq.argtypes = [P, P, P, P, P, I64, I64, I, F, P]
    mq.restype = I

    def m(W=0x1000, A=0x2000, B_=0x3000, out=0x4000, di=256, do=64, r=8, alpha=16.0):
        return mg(P(W), P(A), P(B_), P(out), di, do, r, alpha, None)

    def q(Wq=0x1000, sc=0x5000, A=0x2000, B_=0x3000, out=0x4000, di=256, do=64, r=8, alpha=16.0):
        return mq(P(Wq), P(sc), P(A), P(B_), P(out), di, do, r, alpha, None)

    for bad in (dict(W=None), dict(A=None), dict(B_=None), dict(out=None), dict(di=4), dict(di=260),
                dict(do=0), dict(di=(1 << 24) + 8), dict(r=0), dict(r=12), dict(r=264),
                dict(alpha=float("nan")), dict(alpha=float("inf"))):
        assert m(**bad) == 1, bad                     # LORA_ERR_INVALID_ARG
    for bad in (dict(W=0x1008), dict(A=0x2004), dict(B_=0x3002), dict(out=0x4008)):
        assert m(**bad) == 2, bad                     # LORA_ERR_MISALIGNED
    assert q(sc=None) == 1                            # the scales are required
    assert q(di=96) == 1                              # 4-bit weight: d_in % 64 == 0
    assert q(sc=0x5002) == 2 and q(Wq=0x1008) == 2


def test_merge_fp8_and_nf4_argument_checks(lib):
    """The FP8 and codebook merges: scales (and the codebook) required and finite, the
    formats' d_in rules, alignment, all before any launch."""
    import numpy as np
    assert {"lora_linear_merge_fp8", "lora_linear_merge_nf4"} <= set(L.declared_functions())
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    m8 = lib.lora_linear_merge_fp8
    m8.argtypes = [P, P, P, P, P, I64, I64, I, F, P]
    m8.restype = I
    mn = lib.lora_linear_merge_nf4
    mn.argtypes = [P, P, P, P, P, P, I64, I64, I, F, P]
    mn.restype = I
    good = np.linspace(-1.0, 1.0, 16).astype(np.float32)
    bad_cb = good.copy()
    bad_cb[3] = np.nan

    def f(W8=0x1000, sc=0x5000, A=0x2000, B_=0x3000, out=0x4000, di=256, do=64, r=8, alpha=16.0):
        return m8(P(W8), P(sc), P(A), P(B_), P(out), di, do, r, alpha, None)

    def n(Wq=0x1000, sc=0x5000, cb=good, A=0x2000, B_=0x3000, out=0x4000, di=256, do=64, r=8, alpha=16.0):
        cbp = None if cb is None else cb.ctypes.data_as(P)
        return mn(P(Wq), P(sc), cbp, P(A), P(B_), P(out), di, do, r, alpha, None)

    assert f(sc=None) == 1 and f(W8=None) == 1
    assert f(di=264) == 1                             # FP8 weight: d_in % 16 == 0
    assert f(r=72, alpha=float("nan")) == 1
    assert f(sc=0x5008) == 2 and f(W8=0x1004) == 2
    assert n(cb=None) == 1 and n(sc=None) == 1
    assert n(cb=bad_cb) == 1                          # a non-finite codebook value
    assert n(di=320 + 32) == 1                        # codebook weight: d_in % 64 == 0
    assert n(Wq=0x1008) == 2 and n(out=0x4004) == 2


def test_fp8_validation_before_any_device_work(lib):
    """The FP8 entry points: workspace sizes for their ops, and argument checks (codes
    and scales required, 16-byte aligned, d_in % 16 == 0) before any launch."""
    assert {"lora_linear_fwd_fp8", "lora_linear_bwd_fp8"} <= set(L.declared_functions())
    for op in (L.OP_FWD_FP8, L.OP_BWD_FP8):
        assert L.lora_linear_workspace_size(op, 4096, 4096, 4096, 8) == L.lora_linear_workspace_size(
            op - 2, 4096, 4096, 4096, 8)  # the coded weights' workspaces do not depend on the format
    assert L.lora_linear_workspace_size(L.OP_FWD_FP8, 64, 1040, 256, 8) > 0      # d_in % 16 == 0 suffices
    assert L.lora_linear_workspace_size(L.OP_FWD_FP8, 64, 1032, 256, 8) == 0     # d_in % 16 != 0
    assert L.lora_linear_workspace_size(8, 64, 256, 256, 8) == 0
    P = ctypes.c_void_p
    fn = lib.lora_linear_fwd_fp8

    def fwd(W8=0x2000, Ws=0x2800, di=256, x=0x1000):
        return fn(P(x), P(W8), P(Ws), P(0x3000), P(0x4000), P(0x5000), None, 64, di, 256, 8, 16.0, P(0x10000),
                  1 << 30, None)
    assert fwd(W8=None) == 1
    assert fwd(Ws=None) == 1
    assert fwd(di=264) == 1        # not a multiple of 16
    assert fwd(W8=0x2004) == 2
    assert fwd(Ws=0x2808) == 2
    st = lib.lora_linear_bwd_fp8(P(0x1000), P(0x1000), P(0x2000), P(0x2800), P(0x3000), P(0x4000), None, None,
                                 None, P(0x7000), 64, 256, 256, 8, 16.0, P(0x10000), 1 << 30, None)
    assert st == 1  # dA is required


def test_nf4_validation_before_any_device_work(lib):
    """The 4-bit codebook entry points: workspace sizes, and argument checks (codes,
    scales and a host codebook of finite values required, d_in % 64 == 0) before any
    launch."""
    import numpy as np
    assert {"lora_linear_fwd_nf4", "lora_linear_bwd_nf4"} <= set(L.declared_functions())
    for op in (L.OP_FWD_NF4, L.OP_BWD_NF4):
        assert L.lora_linear_workspace_size(op, 4096, 8192, 28672, 16) == L.lora_linear_workspace_size(
            op - 4, 4096, 8192, 28672, 16)
    assert L.lora_linear_workspace_size(L.OP_FWD_NF4, 64, 96, 256, 8) == 0  # d_in % 64 != 0
    P = ctypes.c_void_p
    cb = np.linspace(-1, 1, 16).astype(np.float32)
    bad = cb.copy()
    bad[5] = np.nan
    fn = lib.lora_linear_fwd_nf4

    def fwd(codebook=cb, Wq=0x2000, di=256):
        cbp = None if codebook is None else codebook.ctypes.data_as(P)
        return fn(P(0x1000), P(Wq), P(0x2800), cbp, P(0x3000), P(0x4000), P(0x5000), None, 64, di, 256, 8, 16.0,
                  P(0x10000), 1 << 30, None)
    assert fwd(codebook=None) == 1
    assert fwd(codebook=bad) == 1
    assert fwd(Wq=None) == 1
    assert fwd(di=288) == 1        # not a multiple of 64
    assert fwd(Wq=0x2004) == 2
