"""Shared helpers of the GPU tests: move generator output to the device, run the
library through its C ABI, ask the oracle for the same quantities, compare."""
from __future__ import annotations

import time

import numpy as np
import torch

import oracle
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200 import lora_linear as L

# Tolerances of the contract: ||gpu - ref||_inf <= rel * ||ref||_inf + abs.
TOL_HX = (1e-2, 1e-3)   # h, dX
TOL_AB = (2e-2, 0.0)    # dA, dB
# Tighter diagnostic on the rms error (bf16 output rounding is ~2^-9 relative), so a
# dropped piece of the low-rank term cannot hide under the max-norm bound.
RMS_HX = 4e-3
RMS_AB = 1e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class DeviceLayer:
    """Device copies of one layer's inputs plus output buffers and workspaces."""

    def __init__(self, inp: inputs.LayerInputs):
        sp = inp.spec
        self.spec, self.inp = sp, inp
        self.x, self.A, self.B, self.dY = (dev_bf16(a) for a in (inp.x, inp.A, inp.B, inp.dY))
        self.q4 = sp.q4
        self.fp8 = getattr(sp, "fp8", False)
        self.nf4 = getattr(sp, "nf4", False)
        self.W = None
        if sp.q4 or self.nf4:
            self.Wq, self.Wscale = dev_u8(inp.Wq), dev_bf16(inp.Wscale)
        elif self.fp8:
            self.W8, self.W8scale = dev_u8(inp.W8), dev_bf16(inp.W8scale)
        else:
            self.W = dev_bf16(inp.W)
        M, di, do, r = sp.M, sp.d_in, sp.d_out, sp.r
        self.h = torch.empty(M, do, dtype=torch.bfloat16, device="cuda")
        self.xa = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
        self.dX = torch.empty(M, di, dtype=torch.bfloat16, device="cuda")
        self.dA = torch.empty(r, di, dtype=torch.float32, device="cuda")
        self.dB = torch.empty(do, r, dtype=torch.float32, device="cuda")
        fop, bop = ((L.OP_FWD_Q4, L.OP_BWD_Q4) if sp.q4 else (L.OP_FWD_FP8, L.OP_BWD_FP8) if self.fp8
                    else (L.OP_FWD_NF4, L.OP_BWD_NF4) if self.nf4 else (L.OP_FWD, L.OP_BWD))
        self.ws_f = L.workspace(fop, M, di, do, r)
        self.ws_b = L.workspace(bop, M, di, do, r)

    def forward(self, save_xa=True):
        xa = self.xa if save_xa else None
        if self.q4:
            L.lora_linear_fwd_q4(self.x, self.Wq, self.Wscale, self.A, self.B, self.h, xa, self.spec.alpha, self.ws_f)
        elif self.fp8:
            L.lora_linear_fwd_fp8(self.x, self.W8, self.W8scale, self.A, self.B, self.h, xa, self.spec.alpha,
                                  self.ws_f)
        elif self.nf4:
            L.lora_linear_fwd_nf4(self.x, self.Wq, self.Wscale, self.inp.codebook, self.A, self.B, self.h, xa,
                                  self.spec.alpha, self.ws_f)
        else:
            L.lora_linear_fwd(self.x, self.W, self.A, self.B, self.h, xa, self.spec.alpha, self.ws_f)

    def backward(self, use_xa=True, want_dx=True):
        xa = self.xa if use_xa else None
        dX = self.dX if want_dx else None
        if self.q4:
            L.lora_linear_bwd_q4(self.dY, self.x, self.Wq, self.Wscale, self.A, self.B, xa, dX, self.dA, self.dB,
                                 self.spec.alpha, self.ws_b)
        elif self.fp8:
            L.lora_linear_bwd_fp8(self.dY, self.x, self.W8, self.W8scale, self.A, self.B, xa, dX, self.dA, self.dB,
                                  self.spec.alpha, self.ws_b)
        elif self.nf4:
            L.lora_linear_bwd_nf4(self.dY, self.x, self.Wq, self.Wscale, self.inp.codebook, self.A, self.B, xa, dX,
                                  self.dA, self.dB, self.spec.alpha, self.ws_b)
        else:
            L.lora_linear_bwd(self.dY, self.x, self.W, self.A, self.B, xa, dX, self.dA, self.dB, self.spec.alpha,
                              self.ws_b)

    def check(self):
        L.lora_linear_check(self.ws_f)
        L.lora_linear_check(self.ws_b)

    def results(self, rows=None):
        torch.cuda.synchronize()
        sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device=t.device)])
        return {"h": host_f64(sel(self.h)), "dX": host_f64(sel(self.dX)), "xa": host_f64(self.xa),
                "dA": host_f64(self.dA), "dB": host_f64(self.dB)}


def shared_input_projections(M, d_in, d_outs, r, alpha, q4, seed) -> list:
    """Inputs of several projections of one x: each its own W, A, B and dY (streams
    offset by the projection's index), all with the first projection's x."""
    layers = [inputs.make_inputs(inputs.LayerSpec(f"p{p}", M, d_in, d, r, alpha, q4=q4, seed=seed, layer=p))
              for p, d in enumerate(d_outs)]
    for inp in layers[1:]:
        inp.x = layers[0].x
    return layers


def weight_kwargs(inp: inputs.LayerInputs) -> dict:
    """The oracle's keyword arguments for a layer's frozen weight, in its format."""
    sp = inp.spec
    if sp.q4:
        return dict(Wq=inp.Wq, Wscale=inp.Wscale)
    if getattr(sp, "fp8", False):
        return dict(W8=inp.W8, W8scale=inp.W8scale)
    if getattr(sp, "nf4", False):
        return dict(Wq=inp.Wq, Wscale=inp.Wscale, codebook=inp.codebook)
    return dict(W=inp.W)


def oracle_ref(inp: inputs.LayerInputs, rows=None) -> dict:
    sp = inp.spec
    wkw = weight_kwargs(inp)
    h, xa = oracle.forward(inp.x, inp.A, inp.B, sp.s, rows=rows, **wkw)
    bw = oracle.backward(inp.dY, inp.x, inp.A, inp.B, sp.s, rows=rows, xa_=xa, **wkw)
    return {"h": h, "xa": xa, "dX": bw["dX"], "dA": bw["dA"], "dB": bw["dB"], "g": bw["g"]}


def assert_close(name: str, got: np.ndarray, ref: np.ndarray, tol, rms_tol=None):
    rel, ab = tol
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = np.abs(got - ref)
    bound = rel * np.abs(ref).max() + ab
    assert err.max() <= bound, (f"{name}: max|err| {err.max():.4e} > {bound:.4e} "
                                f"at {np.unravel_index(err.argmax(), err.shape)}")
    if rms_tol is not None and np.abs(ref).max() > 0:
        rms = np.sqrt((err ** 2).mean()) / np.sqrt((ref ** 2).mean())
        assert rms <= rms_tol, f"{name}: rms rel err {rms:.3e} > {rms_tol:.1e}"


def compare_all(got: dict, ref: dict, s: float, check_xa=True):
    assert_close("h", got["h"], ref["h"], TOL_HX, RMS_HX)
    assert_close("dX", got["dX"], ref["dX"], TOL_HX, RMS_HX)
    assert_close("dA", got["dA"], ref["dA"], TOL_AB, RMS_AB)
    assert_close("dB", got["dB"], ref["dB"], TOL_AB, RMS_AB)
    if check_xa:
        # xa_save holds bf16(s . x.A^T): one bf16 rounding of the exact product.
        assert_close("xa_save", got["xa"], s * ref["xa"], (2 ** -8, 1e-6), RMS_HX)


def sample_rows(M: int, n_random: int = 24, seed: int = 0) -> np.ndarray:
    """Rows that cover the first and last tile, tile edges and a random spread."""
    fixed = {0, 1, 63, 64, 127, 128, M // 2, M - 129, M - 128, M - 2, M - 1}
    rng = np.random.default_rng(seed)
    rnd = set(rng.integers(0, M, size=n_random).tolist())
    return np.array(sorted(v for v in fixed | rnd if 0 <= v < M), dtype=np.int64)


def check_projections(dl: "DeviceLayer", inp: inputs.LayerInputs, ref: dict, seed: int = 0):
    """Every element of h and dX at sizes the oracle cannot produce whole: each row and
    each column of the GPU result, projected on a random +-1 vector (fp64, on the
    device), against the oracle's projection of the definition.  Per element the GPU
    result carries rounding error of at most ~2^-8 of the element scale (bf16 output,
    bf16 s.xa / s.g, fp32 accumulation; the 4-bit weight's bf16 rounding included), with
    independent signs, so a projection over N terms is allowed 8 sigma of that random
    walk, sigma = sqrt(N) * 2^-8 / sqrt(3) * rms(reference), rms taken from the oracle's
    exact rows `ref`.  A wrong tile, row, column or term moves its projections by far
    more.  Returns the largest residual / allowance (for reporting)."""
    sp = inp.spec
    rng = np.random.default_rng(0xC0DE + seed)
    M, di, do = sp.M, sp.d_in, sp.d_out
    wkw = weight_kwargs(inp)
    u = rng.choice([-1.0, 1.0], M)
    v_h = rng.choice([-1.0, 1.0], do)
    v_x = rng.choice([-1.0, 1.0], di)
    worst = 0.0
    for name, out, v, proj in (("h", dl.h, v_h, oracle.h_projections), ("dX", dl.dX, v_x, oracle.dx_projections)):
        if name == "h":
            row_ref, col_ref = proj(inp.x, inp.A, inp.B, sp.s, v, u, **wkw)
        else:
            row_ref, col_ref = proj(inp.dY, inp.A, inp.B, sp.s, v, u, **wkw)
        od = out.double()
        row = (od @ torch.from_numpy(v).to(od.device)).cpu().numpy()
        col = (torch.from_numpy(u).to(od.device) @ od).cpu().numpy()
        del od
        rms = float(np.sqrt(np.mean(ref[name] ** 2)))
        for what, got, want, n in (("row", row, row_ref, out.shape[1]), ("column", col, col_ref, out.shape[0])):
            allow = 8.0 * np.sqrt(n) * 2.0 ** -8 / np.sqrt(3.0) * rms
            resid = np.abs(got - want)
            i = int(np.argmax(resid))
            assert resid[i] <= allow, (f"{name} {what} projection {i}: got {got[i]:.6g}, oracle {want[i]:.6g}, "
                                       f"|diff| {resid[i]:.3g} > {allow:.3g}")
            worst = max(worst, float(resid[i] / allow))
    return worst


class ErrorTally:
    """Running max-norm and rms statistics of (got - ref) over blocks of one tensor, so
    that a tensor too large to hold twice in fp64 is still held to the contract's bound
    on every element: ||got - ref||_inf <= rel * ||ref||_inf + abs, over the whole tensor."""

    def __init__(self, name: str):
        self.name = name
        self.max_err = 0.0
        self.max_ref = 0.0
        self.where = None
        self.sq_err = 0.0
        self.sq_ref = 0.0
        self.n = 0

    def add(self, got: np.ndarray, ref: np.ndarray, row0: int = 0):
        assert got.shape == ref.shape, (self.name, got.shape, ref.shape)
        assert np.all(np.isfinite(got)), f"{self.name}: non-finite values in rows {row0}.."
        err = np.abs(got - ref)
        i = np.unravel_index(int(err.argmax()), err.shape)
        if err[i] > self.max_err:
            self.max_err = float(err[i])
            self.where = (row0 + int(i[0]),) + tuple(int(v) for v in i[1:])
        self.max_ref = max(self.max_ref, float(np.abs(ref).max()))
        self.sq_err += float((err ** 2).sum())
        self.sq_ref += float((ref ** 2).sum())
        self.n += err.size

    def check(self, tol, rms_tol=None):
        rel, ab = tol
        bound = rel * self.max_ref + ab
        assert self.max_err <= bound, (f"{self.name}: max|err| {self.max_err:.4e} > {bound:.4e} at {self.where} "
                                       f"({self.n} elements compared)")
        if rms_tol is not None and self.sq_ref > 0:
            rms = np.sqrt(self.sq_err / self.sq_ref)
            assert rms <= rms_tol, f"{self.name}: rms rel err {rms:.3e} > {rms_tol:.1e}"
        return self.max_err / bound if bound > 0 else 0.0  # a zero bound (exactly-zero reference) passed exactly


def compare_every_element(dl: "DeviceLayer", inp: inputs.LayerInputs, block_rows: int = 1024) -> dict:
    """Every element of h, dX, s.xa, dA and dB of a layer already run on the GPU against
    the oracle's whole tensors: steps 1, 3, 5 and 6 from oracle.c, steps 2 and 4 for
    every token row from the oracle's dense steps (numpy's fp64 product as the summation
    primitive), a block of rows at a time.  Returns the worst error / bound per output
    and the oracle's wall time."""
    sp = inp.spec
    wkw = weight_kwargs(inp)
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    t_oracle = 0.0
    t0 = time.perf_counter()
    Wf = oracle.weight(sp.d_out, sp.d_in, **wkw)
    xa_ = oracle.xa(inp.x, inp.A)
    g_ = oracle.g(inp.dY, inp.B)
    dA = oracle.da(inp.x, g_, sp.s)
    dB = oracle.db(inp.dY, xa_, sp.s)
    t_oracle += time.perf_counter() - t0
    tally = {k: ErrorTally(k) for k in ("h", "dX", "xa_save", "dA", "dB")}
    for r0 in range(0, sp.M, block_rows):
        r1 = min(sp.M, r0 + block_rows)
        t0 = time.perf_counter()
        h_ref = oracle.h_dense(inp.x[r0:r1], inp.B, xa_[r0:r1], sp.s, Wf)
        dx_ref = oracle.dx_dense(inp.dY[r0:r1], inp.A, g_[r0:r1], sp.s, Wf)
        t_oracle += time.perf_counter() - t0
        tally["h"].add(host_f64(dl.h[r0:r1]), h_ref, r0)
        tally["dX"].add(host_f64(dl.dX[r0:r1]), dx_ref, r0)
    tally["xa_save"].add(host_f64(dl.xa), sp.s * xa_)
    tally["dA"].add(host_f64(dl.dA), dA)
    tally["dB"].add(host_f64(dl.dB), dB)
    worst = {
        "h": tally["h"].check(TOL_HX, RMS_HX),
        "dX": tally["dX"].check(TOL_HX, RMS_HX),
        "xa_save": tally["xa_save"].check((2 ** -8, 1e-6), RMS_HX),
        "dA": tally["dA"].check(TOL_AB, RMS_AB),
        "dB": tally["dB"].check(TOL_AB, RMS_AB),
    }
    return {"worst": worst, "oracle_s": t_oracle, "elements": sum(t.n for t in tally.values())}
