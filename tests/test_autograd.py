"""The framework shim (rank_linear_lora_b200.autograd) on the CPU: the unfused
composition it falls back to when asked (LORA_LINEAR_FUSED=0), and that the fused path
never falls back silently (tensors the library cannot take raise)."""
import warnings

import pytest
import torch

from rank_linear_lora_b200 import autograd as LA


def _layer(seed=0):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(24, 40, generator=g) / 40 ** 0.5).to(torch.bfloat16)
    m = LA.LoraLinear(W, r=8, alpha=16.0)
    with torch.no_grad():
        m.lora_B.copy_((0.02 * torch.randn(24, 8, generator=g)).to(torch.bfloat16))
    x = torch.randn(2, 5, 40, generator=g).to(torch.bfloat16).requires_grad_(True)
    return m, x


def test_switch_gives_the_unfused_composition(monkeypatch):
    monkeypatch.setenv("LORA_LINEAR_FUSED", "0")
    m, x = _layer()
    n0 = LA.fallback_calls
    with warnings.catch_warnings(record=True):
        warnings.simplefilter("always")
        h = m(x)
    assert LA.fallback_calls == n0 + 1
    assert h.shape == (2, 5, 24)
    s = 16.0 / 8
    xs = x.detach().reshape(-1, 40).double()
    want = xs @ m.weight.double().t() + s * (xs @ m.lora_A.double().t()) @ m.lora_B.double().t()
    torch.testing.assert_close(h.reshape(-1, 24).double(), want, rtol=2e-2, atol=2e-2)
    h.float().sum().backward()
    assert m.weight.grad is None  # frozen
    assert m.lora_A.grad is not None and m.lora_B.grad is not None and x.grad is not None


def test_fused_path_does_not_fall_back_on_tensors_it_cannot_take(monkeypatch):
    monkeypatch.setenv("LORA_LINEAR_FUSED", "1")
    m, x = _layer(1)
    n0 = LA.fallback_calls
    with pytest.raises(ValueError):
        m(x)  # CPU tensors: the binding rejects them, nothing computes them behind its back
    assert LA.fallback_calls == n0
