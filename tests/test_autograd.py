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


def _coded_inputs(kind, d_out=40, d_in=128, seed=7):
    import numpy as np
    from rank_linear_lora_b200 import inputs
    spec = inputs.LayerSpec("coded", 8, d_in, d_out, 8, alpha=16.0, q4=kind == "q4", fp8=kind == "fp8",
                            nf4=kind == "nf4", seed=seed)
    return spec, inputs.make_inputs(spec)


@pytest.mark.parametrize("kind", ["q4", "fp8", "nf4"])
def test_frozen_weight_decode_matches_the_oracle(kind):
    """The unfused composition's decoded weight (torch operators) against the oracle's
    decode of the same codes: FP8 exactly, the 4-bit formats to one fp32 rounding."""
    import numpy as np
    import oracle
    spec, inp = _coded_inputs(kind)
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    b16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    if kind == "fp8":
        wt = LA.FrozenWeight("fp8", (u8(inp.W8), b16(inp.W8scale)))
        want = oracle.weight(spec.d_out, spec.d_in, W8=inp.W8, W8scale=inp.W8scale)
    else:
        cb = None if kind == "q4" else np.asarray(inp.codebook, dtype=np.float32)
        wt = LA.FrozenWeight(kind, (u8(inp.Wq), b16(inp.Wscale)), codebook=cb)
        kw = dict(Wq=inp.Wq, Wscale=inp.Wscale)
        if cb is not None:
            kw["codebook"] = cb.astype(np.float64)
        want = oracle.weight(spec.d_out, spec.d_in, **kw)
    got = wt.dense().double().numpy()
    assert (wt.d_out, wt.d_in) == (spec.d_out, spec.d_in)
    if kind == "fp8":
        np.testing.assert_array_equal(got, want)
    else:
        np.testing.assert_allclose(got, want, rtol=2 ** -23, atol=0)


def test_coded_module_unfused_composition(monkeypatch):
    """A module over a 4-bit weight with the fused path off: forward and backward through
    torch's autograd on the decoded weight, and the merged weight of the same terms."""
    import numpy as np
    monkeypatch.setenv("LORA_LINEAR_FUSED", "0")
    spec, inp = _coded_inputs("q4")
    m = LA.LoraLinear.from_q4(torch.from_numpy(np.ascontiguousarray(inp.Wq)),
                              torch.from_numpy(np.ascontiguousarray(inp.Wscale).view(np.int16)).view(torch.bfloat16),
                              r=8, alpha=16.0)
    with torch.no_grad():
        m.lora_B.copy_(torch.randn(spec.d_out, 8, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16) * 0.02)
    x = torch.randn(3, spec.d_in, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16).requires_grad_(True)
    with warnings.catch_warnings(record=True):
        warnings.simplefilter("always")
        h = m(x)
    W = m._frozen().dense().double()
    s = 16.0 / 8
    want = x.detach().double() @ W.t() + s * (x.detach().double() @ m.lora_A.double().t()) @ m.lora_B.double().t()
    torch.testing.assert_close(h.double(), want, rtol=2e-2, atol=2e-2)
    h.float().sum().backward()
    assert x.grad is not None and m.lora_A.grad is not None and m.lora_B.grad is not None
    merged = m.merged_weight().double()
    torch.testing.assert_close(merged, W + s * m.lora_B.double() @ m.lora_A.double(), rtol=1e-2, atol=1e-3)
    with pytest.raises(ValueError):
        LA.LoraLinear(r=8, alpha=16.0)  # neither a weight nor a frozen one
