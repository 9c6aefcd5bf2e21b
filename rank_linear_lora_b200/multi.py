"""Several LoRA projections of one input x run as one fused layer.

Projections p = 0..P-1 (q/k/v of an attention block, gate/up of an MLP) read the same
x [M, d_in]; each has its own frozen W_p [d_p, d_in], adapters A_p [r, d_in] and
B_p [d_p, r], and all share alpha and r, so s = alpha/r.  Stacked as

    W = [W_0; W_1; ...]              [sum d_p, d_in]
    A = [A_0; A_1; ...]              [P r, d_in]
    B = blockdiag(B_0, B_1, ...)     [sum d_p, P r]

they form one layer of the kind lora_linear_fwd / _bwd compute.  x A^T is
[x A_0^T | x A_1^T | ...] and the zero blocks of B keep each projection's LoRA term to
its own adapters, so h = x W^T + s (x A^T) B^T = [h_0 | h_1 | ...].  In the backward,
dY = [dY_0 | dY_1 | ...] gives g = dY B = [dY_0 B_0 | ...] and

* dX = sum_p (dY_p W_p + s g_p A_p), the gradient of the shared x through every
  projection, accumulated in fp32 inside one GEMM (P separate layers would each round
  their dX to bf16 before the sum);
* dA = [dA_0; dA_1; ...];
* the diagonal blocks of dB are the dB_p.  The off-diagonal blocks are gradients of
  entries held at zero; they are computed but never read.

The call passes r_call = P r and alpha_call = P alpha.  Both products are exact in fp32
(checked here for alpha as the library receives it, rounded to fp32), so the library's
s = alpha_call / r_call is bit for bit the s of a single projection's call.

What the stacking saves: the forward prologue reads x once for all P projections, one
main GEMM runs with N = sum d_p, the backward reads x once for dA, and dX needs no
extra pass to add P partial results.  Page "ms-swift高效微调组合：LoRA+UnSloth提速实践",
section 1.2, describes the layer (linear, LoRA_A, LoRA_B and the add) as one kernel;
section 2.3, step 2, has every linear of the block (q/k/v/o, gate/up/down) carry an
adapter.  The projections of one x are where that fusion can also be shared.

This module only lays out parameters and marshals arguments; every step of the layer
runs in the library's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import lora_linear as L
from .dp import PackedGrads


def _exact_f32_product(a: float, n: int) -> bool:
    """n times alpha as the library receives it (rounded to fp32) is exact in fp32."""
    with np.errstate(over="ignore"):
        a32 = np.float32(a)
        prod = np.float32(a32 * np.float32(n))
    return bool(np.isfinite(prod)) and float(prod) == float(a32) * n


class SharedInputProjections:
    """Stacked parameters of P LoRA projections of one x, with per-projection views.

    ``W`` (or ``Wq`` + ``Wscale`` for the 4-bit weight), ``A`` and ``B`` are the stacked
    device tensors the layer is called with.  ``W_p(p)``, ``A_p(p)``, ``B_p(p)`` are
    views of projection p's parts: an optimizer that updates ``A_p``/``B_p`` in place
    leaves the zero blocks of ``B`` untouched.  ``grads`` is one packed fp32 [dA | dB]
    buffer (a single all-reduce under data parallelism).
    """

    def __init__(self, d_in: int, d_outs, r: int, alpha: float, *, q4: bool = False, device=None):
        d_outs = [int(d) for d in d_outs]
        P = len(d_outs)
        if P < 1 or any(d < 1 for d in d_outs):
            raise ValueError(f"need at least one projection of positive width, got {d_outs}")
        if any(d % 8 for d in d_outs):
            raise ValueError(f"every projection width must be a multiple of 8 (16-byte rows), got {d_outs}")
        if r < 1 or r % 8 or P * r > 256:
            raise ValueError(f"r={r} with {P} projections: need r % 8 == 0 and P*r <= 256")
        if not _exact_f32_product(alpha, P):
            raise ValueError(f"alpha={alpha!r}: {P}*alpha must be exact in fp32")
        self.d_in, self.d_outs, self.r, self.alpha, self.q4 = d_in, d_outs, r, float(alpha), q4
        self.P = P
        self.offsets = np.concatenate([[0], np.cumsum(d_outs)]).astype(int).tolist()
        self.d_out = self.offsets[-1]
        self.r_call = P * r
        self.alpha_call = float(np.float32(alpha) * np.float32(P))
        do, rc = self.d_out, self.r_call
        if q4:
            if d_in % 64:
                raise ValueError("the 4-bit weight needs d_in % 64 == 0")
            self.W = None
            self.Wq = torch.zeros(do, d_in // 2, dtype=torch.uint8, device=device)
            self.Wscale = torch.zeros(do, d_in // 64, dtype=torch.bfloat16, device=device)
        else:
            self.W = torch.zeros(do, d_in, dtype=torch.bfloat16, device=device)
            self.Wq = self.Wscale = None
        self.A = torch.zeros(rc, d_in, dtype=torch.bfloat16, device=device)
        self.B = torch.zeros(do, rc, dtype=torch.bfloat16, device=device)
        self.grads = PackedGrads(rc, d_in, do, device=device)

    # ------------------------------------------------------------------ layout
    def rows(self, p: int) -> slice:
        """Projection p's rows of W and B, columns of h and dY."""
        return slice(self.offsets[p], self.offsets[p + 1])

    def ranks(self, p: int) -> slice:
        """Projection p's rows of A, columns of B and of xa_save."""
        return slice(p * self.r, (p + 1) * self.r)

    def W_p(self, p: int):
        if self.q4:
            return self.Wq[self.rows(p)], self.Wscale[self.rows(p)]
        return self.W[self.rows(p)]

    def A_p(self, p: int) -> torch.Tensor:
        return self.A[self.ranks(p)]

    def B_p(self, p: int) -> torch.Tensor:
        return self.B[self.rows(p), self.ranks(p)]

    def load(self, p: int, *, W=None, Wq=None, Wscale=None, A=None, B=None) -> None:
        """Copy projection p's tensors into the stacked parameters (model set-up)."""
        rows = self.rows(p)
        if W is not None:
            if self.q4:
                raise ValueError("this stack holds a 4-bit weight: pass Wq and Wscale")
            self.W[rows].copy_(W)
        if Wq is not None or Wscale is not None:
            if not self.q4 or Wq is None or Wscale is None:
                raise ValueError("Wq and Wscale go together, into a 4-bit stack")
            self.Wq[rows].copy_(Wq)
            self.Wscale[rows].copy_(Wscale)
        if A is not None:
            self.A_p(p).copy_(A)
        if B is not None:
            self.B_p(p).copy_(B)

    def split_h(self, h: torch.Tensor):
        """[h_0, h_1, ...] as column views of the stacked output [M, sum d_p]."""
        return [h[:, self.rows(p)] for p in range(self.P)]

    def split_xa(self, xa: torch.Tensor):
        return [xa[:, self.ranks(p)] for p in range(self.P)]

    def split_grads(self, dA: torch.Tensor | None = None, dB: torch.Tensor | None = None):
        """[(dA_p, dB_p)] as views of the stacked gradients (default: ``grads``)."""
        dA = self.grads.dA if dA is None else dA
        dB = self.grads.dB if dB is None else dB
        return [(dA[self.ranks(p)], dB[self.rows(p), self.ranks(p)]) for p in range(self.P)]

    # ------------------------------------------------------------------ calls
    def workspaces(self, M: int, device=None):
        """(forward workspace, backward workspace) for M tokens."""
        fop, bop = (L.OP_FWD_Q4, L.OP_BWD_Q4) if self.q4 else (L.OP_FWD, L.OP_BWD)
        return (L.workspace(fop, M, self.d_in, self.d_out, self.r_call, device=device),
                L.workspace(bop, M, self.d_in, self.d_out, self.r_call, device=device))

    def forward(self, x, h, xa_save, ws, stream=None) -> None:
        """h [M, sum d_p] = [h_0 | h_1 | ...]; xa_save [M, P r] (or None)."""
        if self.q4:
            L.lora_linear_fwd_q4(x, self.Wq, self.Wscale, self.A, self.B, h, xa_save, self.alpha_call, ws, stream)
        else:
            L.lora_linear_fwd(x, self.W, self.A, self.B, h, xa_save, self.alpha_call, ws, stream)

    def backward(self, dY, x, xa_save, dX, ws, dA=None, dB=None, stream=None) -> None:
        """dY [M, sum d_p] = [dY_0 | dY_1 | ...]; dX [M, d_in] summed over the
        projections (or None); dA, dB default to ``grads``."""
        dA = self.grads.dA if dA is None else dA
        dB = self.grads.dB if dB is None else dB
        if self.q4:
            L.lora_linear_bwd_q4(dY, x, self.Wq, self.Wscale, self.A, self.B, xa_save, dX, dA, dB, self.alpha_call,
                                 ws, stream)
        else:
            L.lora_linear_bwd(dY, x, self.W, self.A, self.B, xa_save, dX, dA, dB, self.alpha_call, ws, stream)
