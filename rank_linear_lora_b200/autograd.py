"""The fused LoRA linear layer as a PyTorch autograd function and module.

This is the framework-facing layer over the C ABI: ``LoraLinearFunction`` runs
lora_linear_fwd in its forward, keeps bf16(s . x.A^T) for the backward (so the
backward never recomputes x.A^T), and runs lora_linear_bwd in its backward, which
returns dX, dA and dB (W is frozen: no gradient).  Workspaces are allocated once per
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


def _unfused(x, W, A, B, alpha):
    s = alpha / A.shape[0]
    return x @ W.t() + s * ((x @ A.t()) @ B.t())


class LoraLinearFunction(torch.autograd.Function):
    """h = x.W^T + (alpha / r).(x.A^T).B^T with frozen W; x [M, d_in] bf16 on the GPU.
    Gradients flow to x, A and B."""

    @staticmethod
    def forward(ctx, x, W, A, B, alpha: float):
        M, d_in = x.shape
        r, d_out = A.shape[0], W.shape[0]
        ws = _workspace(L.OP_FWD, M, d_in, d_out, r, x.device)
        h = torch.empty(M, d_out, dtype=torch.bfloat16, device=x.device)
        xa = torch.empty(M, r, dtype=torch.bfloat16, device=x.device)
        L.lora_linear_fwd(x, W, A, B, h, xa, alpha, ws)
        ctx.save_for_backward(x, W, A, B, xa)
        ctx.alpha = alpha
        return h

    @staticmethod
    def backward(ctx, dY):
        x, W, A, B, xa = ctx.saved_tensors
        M, d_in = x.shape
        r, d_out = A.shape[0], W.shape[0]
        dY = dY.contiguous()
        ws = _workspace(L.OP_BWD, M, d_in, d_out, r, x.device)
        dX = torch.empty_like(x) if ctx.needs_input_grad[0] else None
        dA = torch.empty(r, d_in, dtype=torch.float32, device=x.device)
        dB = torch.empty(d_out, r, dtype=torch.float32, device=x.device)
        L.lora_linear_bwd(dY, x, W, A, B, xa, dX, dA, dB, ctx.alpha, ws)
        return dX, None, dA.to(A.dtype), dB.to(B.dtype), None


def lora_linear(x, W, A, B, alpha: float):
    """The fused layer, or the unfused composition where the library declines (see the
    module docstring)."""
    global fallback_calls
    if fused_enabled():
        try:
            return LoraLinearFunction.apply(x, W, A, B, alpha)
        except L.LoraError as e:
            if e.status != 3:  # only LORA_ERR_UNSUPPORTED falls back
                raise
            reason = str(e)
    else:
        reason = "LORA_LINEAR_FUSED=0"
    fallback_calls += 1
    if fallback_calls == 1:
        warnings.warn(f"fused LoRA linear not used ({reason}); computing the unfused composition", RuntimeWarning)
    return _unfused(x, W, A, B, alpha)


class LoraLinear(torch.nn.Module):
    """A frozen bf16 weight [d_out, d_in] with a trainable rank-r adapter (A [r, d_in],
    B [d_out, r]) on the fused layer; inputs [..., d_in] are flattened to tokens."""

    def __init__(self, weight: torch.Tensor, r: int, alpha: float):
        super().__init__()
        d_out, d_in = weight.shape
        self.weight = torch.nn.Parameter(weight.detach().to(torch.bfloat16).contiguous(), requires_grad=False)
        bound = 1.0 / d_in ** 0.5
        self.lora_A = torch.nn.Parameter(
            torch.empty(r, d_in, dtype=torch.bfloat16, device=weight.device).uniform_(-bound, bound))
        self.lora_B = torch.nn.Parameter(torch.zeros(d_out, r, dtype=torch.bfloat16, device=weight.device))
        self.r, self.alpha = r, float(alpha)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        shape = x.shape
        h = lora_linear(x.reshape(-1, shape[-1]).contiguous(), self.weight, self.lora_A, self.lora_B, self.alpha)
        return h.reshape(*shape[:-1], h.shape[-1])
