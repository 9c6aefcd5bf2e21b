"""The fused LoRA linear layer as a PyTorch autograd function and module.

This is the framework-facing layer over the C ABI: ``LoraLinearFunction`` runs the
forward entry point of the frozen weight's format (bf16, 4-bit, FP8 or NF4 codes) in
its forward, keeps bf16(s . x.A^T) for the backward (so the backward never recomputes
x.A^T), and runs the matching backward, which returns dX, dA and dB (the weight is
frozen: no gradient).  ``LoraLinear.merged_weight`` folds the trained adapter into a
bf16 weight with the library's merge kernels.  Workspaces are allocated once per
(device, shape) by torch and reused; the library itself never allocates.

The switch from standard LoRA to the fused layer is one flag in the pages' training
frameworks, with standard LoRA taken when the accelerated path does not support the
case (page "ms-swift高效微调组合：LoRA+UnSloth提速实践", closing section; page
"Unsloth — 微调 2-5x 加速", section 踩过的坑).  Here the same holds: if the loaded
library answers LORA_ERR_UNSUPPORTED (a device other than sm_100, or a shape it does
not cover), or the environment sets LORA_LINEAR_FUSED=0, the function computes the
unfused composition x.W^T + s.(x.A^T).B^T with torch's own GPU operators and
autograd, and warns once.  If the library is missing it raises: there is no silent
fallback.
"""
from __future__ import annotations

import os
import threading
import warnings

import torch

from . import lora_linear as L

_ws_lock = threading.Lock()
_ws_cache: dict = {}
fallback_calls = 0  # forward calls that took the unfused composition


def fused_enabled() -> bool:
    return os.environ.get("LORA_LINEAR_FUSED", "1") != "0"


def _workspace(op: int, M: int, d_in: int, d_out: int, r: int, device) -> torch.Tensor:
    key = (str(device), op, M, d_in, d_out, r, L.lora_linear_workspace_size(op, M, d_in, d_out, r))
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None:
            ws = L.workspace(op, M, d_in, d_out, r, device=device)
            _ws_cache[key] = ws
        return ws


class FrozenWeight:
    """The frozen base weight [d_out, d_in] in one of the layer's storage formats:
    "bf16" (W), "q4" (codes Wq uint8 [d_out, d_in/2], bf16 scales [d_out, d_in/64]: w =
    (q - 8) * scale / 7), "fp8" (E4M3 codes W8 uint8 [d_out, d_in], one bf16 scale per
    row) or "nf4" (codes and scales as q4, w = codebook[q] * scale, 16 codebook values)."""

    KINDS = ("bf16", "q4", "fp8", "nf4")

    def __init__(self, kind: str, tensors: tuple, codebook=None):
        if kind not in self.KINDS:
            raise ValueError(f"weight format: one of {self.KINDS}")
        self.kind, self.tensors, self.codebook = kind, tuple(tensors), codebook
        first = self.tensors[0]
        self.d_out = first.shape[0]
        self.d_in = first.shape[1] * (2 if kind in ("q4", "nf4") else 1)

    def ops(self):
        return {"bf16": (L.OP_FWD, L.OP_BWD), "q4": (L.OP_FWD_Q4, L.OP_BWD_Q4), "fp8": (L.OP_FWD_FP8, L.OP_BWD_FP8),
                "nf4": (L.OP_FWD_NF4, L.OP_BWD_NF4)}[self.kind]

    def fwd(self, x, A, B, h, xa, alpha, ws):
        t = self.tensors
        if self.kind == "bf16":
            L.lora_linear_fwd(x, t[0], A, B, h, xa, alpha, ws)
        elif self.kind == "q4":
            L.lora_linear_fwd_q4(x, t[0], t[1], A, B, h, xa, alpha, ws)
        elif self.kind == "fp8":
            L.lora_linear_fwd_fp8(x, t[0], t[1], A, B, h, xa, alpha, ws)
        else:
            L.lora_linear_fwd_nf4(x, t[0], t[1], self.codebook, A, B, h, xa, alpha, ws)

    def bwd(self, dY, x, A, B, xa, dX, dA, dB, alpha, ws):
        t = self.tensors
        if self.kind == "bf16":
            L.lora_linear_bwd(dY, x, t[0], A, B, xa, dX, dA, dB, alpha, ws)
        elif self.kind == "q4":
            L.lora_linear_bwd_q4(dY, x, t[0], t[1], A, B, xa, dX, dA, dB, alpha, ws)
        elif self.kind == "fp8":
            L.lora_linear_bwd_fp8(dY, x, t[0], t[1], A, B, xa, dX, dA, dB, alpha, ws)
        else:
            L.lora_linear_bwd_nf4(dY, x, t[0], t[1], self.codebook, A, B, xa, dX, dA, dB, alpha, ws)

    def merge(self, A, B, W_out, alpha):
        """W_out = w + (alpha / r) * B . A on the device (the library's merge kernels)."""
        t = self.tensors
        if self.kind == "bf16":
            L.lora_linear_merge(t[0], A, B, W_out, alpha)
        elif self.kind == "q4":
            L.lora_linear_merge_q4(t[0], t[1], A, B, W_out, alpha)
        elif self.kind == "fp8":
            L.lora_linear_merge_fp8(t[0], t[1], A, B, W_out, alpha)
        else:
            L.lora_linear_merge_nf4(t[0], t[1], self.codebook, A, B, W_out, alpha)

    def dense(self) -> torch.Tensor:
        """The decoded weight as fp32, with torch operators (the unfused composition's
        weight; the fused path never forms it)."""
        t = self.tensors
        if self.kind == "bf16":
            return t[0].float()
        if self.kind == "fp8":
            return t[0].view(torch.float8_e4m3fn).float() * t[1].float()[:, None]
        q = torch.stack(((t[0] & 0x0F), (t[0] >> 4)), dim=-1).reshape(self.d_out, self.d_in).to(torch.int64)
        sc = t[1].float().repeat_interleave(64, dim=1)
        if self.kind == "q4":
            return (q - 8).float() * (sc / 7.0)
        cb = torch.as_tensor(self.codebook, dtype=torch.float32, device=q.device)
        return cb[q] * sc


def _unfused(x, wt: FrozenWeight, A, B, alpha):
    s = alpha / A.shape[0]
    W = wt.dense().to(x.dtype)
    return x @ W.t() + s * ((x @ A.t()) @ B.t())


class LoraLinearFunction(torch.autograd.Function):
    """h = x.w^T + (alpha / r).(x.A^T).B^T with a frozen weight w (a FrozenWeight, any of
    the layer's formats); x [M, d_in] bf16 on the GPU.  Gradients flow to x, A and B."""

    @staticmethod
    def forward(ctx, x, A, B, alpha: float, wt: FrozenWeight):
        M, d_in = x.shape
        r, d_out = A.shape[0], wt.d_out
        fop, _ = wt.ops()
        ws = _workspace(fop, M, d_in, d_out, r, x.device)
        h = torch.empty(M, d_out, dtype=torch.bfloat16, device=x.device)
        xa = torch.empty(M, r, dtype=torch.bfloat16, device=x.device)
        wt.fwd(x, A, B, h, xa, alpha, ws)
        ctx.save_for_backward(x, A, B, xa)
        ctx.alpha, ctx.wt = alpha, wt
        return h

    @staticmethod
    def backward(ctx, dY):
        x, A, B, xa = ctx.saved_tensors
        wt = ctx.wt
        M, d_in = x.shape
        r, d_out = A.shape[0], wt.d_out
        dY = dY.contiguous()
        _, bop = wt.ops()
        ws = _workspace(bop, M, d_in, d_out, r, x.device)
        dX = torch.empty_like(x) if ctx.needs_input_grad[0] else None
        dA = torch.empty(r, d_in, dtype=torch.float32, device=x.device)
        dB = torch.empty(d_out, r, dtype=torch.float32, device=x.device)
        wt.bwd(dY, x, A, B, xa, dX, dA, dB, ctx.alpha, ws)
        return dX, dA.to(A.dtype), dB.to(B.dtype), None, None


def lora_linear(x, W, A, B, alpha: float):
    """The fused layer, or the unfused composition where the library declines (see the
    module docstring).  W: a bf16 tensor [d_out, d_in] or a FrozenWeight."""
    global fallback_calls
    wt = W if isinstance(W, FrozenWeight) else FrozenWeight("bf16", (W,))
    if fused_enabled():
        try:
            return LoraLinearFunction.apply(x, A, B, alpha, wt)
        except L.LoraError as e:
            if e.status != 3:  # only LORA_ERR_UNSUPPORTED falls back
                raise
            reason = str(e)
    else:
        reason = "LORA_LINEAR_FUSED=0"
    fallback_calls += 1
    if fallback_calls == 1:
        warnings.warn(f"fused LoRA linear not used ({reason}); computing the unfused composition", RuntimeWarning)
    return _unfused(x, wt, A, B, alpha)


class LoraLinear(torch.nn.Module):
    """A frozen weight [d_out, d_in] with a trainable rank-r adapter (A [r, d_in],
    B [d_out, r]) on the fused layer; inputs [..., d_in] are flattened to tokens.  The
    weight is a bf16 tensor (`LoraLinear(W, r, alpha)`) or a coded one
    (`LoraLinear.from_q4 / from_fp8 / from_nf4`), kept as buffers, never trained."""

    def __init__(self, weight: torch.Tensor = None, r: int = 8, alpha: float = 16.0, *, frozen: FrozenWeight = None):
        super().__init__()
        if (weight is None) == (frozen is None):
            raise ValueError("give the bf16 weight or a FrozenWeight, not both")
        if weight is not None:
            self.weight = torch.nn.Parameter(weight.detach().to(torch.bfloat16).contiguous(), requires_grad=False)
            frozen = FrozenWeight("bf16", (self.weight,))
        else:
            for i, t in enumerate(frozen.tensors):
                self.register_buffer(f"frozen_{i}", t)
        self.frozen = frozen
        d_out, d_in = frozen.d_out, frozen.d_in
        dev = frozen.tensors[0].device
        bound = 1.0 / d_in ** 0.5
        self.lora_A = torch.nn.Parameter(torch.empty(r, d_in, dtype=torch.bfloat16, device=dev).uniform_(-bound, bound))
        self.lora_B = torch.nn.Parameter(torch.zeros(d_out, r, dtype=torch.bfloat16, device=dev))
        self.r, self.alpha = r, float(alpha)

    @classmethod
    def from_q4(cls, Wq, Wscale, r: int, alpha: float):
        return cls(r=r, alpha=alpha, frozen=FrozenWeight("q4", (Wq, Wscale)))

    @classmethod
    def from_fp8(cls, W8, W8scale, r: int, alpha: float):
        return cls(r=r, alpha=alpha, frozen=FrozenWeight("fp8", (W8, W8scale)))

    @classmethod
    def from_nf4(cls, Wq, Wscale, codebook, r: int, alpha: float):
        return cls(r=r, alpha=alpha, frozen=FrozenWeight("nf4", (Wq, Wscale), codebook=codebook))

    def _frozen(self) -> FrozenWeight:
        """The frozen weight over this module's current tensors (after .to() / .cuda())."""
        if self.frozen.kind == "bf16":
            self.frozen.tensors = (self.weight,)
        else:
            self.frozen.tensors = tuple(getattr(self, f"frozen_{i}") for i in range(len(self.frozen.tensors)))
        return self.frozen

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        shape = x.shape
        h = lora_linear(x.reshape(-1, shape[-1]).contiguous(), self._frozen(), self.lora_A, self.lora_B, self.alpha)
        return h.reshape(*shape[:-1], h.shape[-1])

    @torch.no_grad()
    def merged_weight(self) -> torch.Tensor:
        """W' = w + (alpha / r) * B . A in bf16, for deployment without the adapter: the
        library's merge kernels, or the unfused composition where the fused path is off."""
        wt = self._frozen()
        if fused_enabled():
            out = torch.empty(wt.d_out, wt.d_in, dtype=torch.bfloat16, device=self.lora_A.device)
            wt.merge(self.lora_A.contiguous(), self.lora_B.contiguous(), out, self.alpha)
            return out
        s = self.alpha / self.r
        return (wt.dense() + s * (self.lora_B.float() @ self.lora_A.float())).to(torch.bfloat16)
