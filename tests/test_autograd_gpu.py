"""The framework shim on the GPU: the module runs the library's kernels (five launches
per forward + backward, no fallback) and its outputs and gradients match the oracle;
with LORA_LINEAR_FUSED=0 it computes the unfused composition instead, to the same
bounds."""
import numpy as np
import pytest
import torch

from lora_cases import TOL_AB, TOL_HX, assert_close, oracle_ref
from rank_linear_lora_b200 import autograd as LA
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200 import lora_linear as L

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "unfused"])
def test_module_matches_oracle(fused, monkeypatch):
    monkeypatch.setenv("LORA_LINEAR_FUSED", "1" if fused else "0")
    spec = inputs.LayerSpec("shim", 2 * 160, 384, 320, 16, alpha=32.0, seed=0x5A1)
    inp = inputs.make_inputs(spec)
    m = LA.LoraLinear(_dev(inp.W), r=spec.r, alpha=spec.alpha)
    with torch.no_grad():
        m.lora_A.copy_(_dev(inp.A))
        m.lora_B.copy_(_dev(inp.B))
    x = _dev(inp.x).reshape(2, 160, 384).requires_grad_(True)
    dY = _dev(inp.dY).reshape(2, 160, 320)
    n0, f0 = L.lora_linear_launch_count(), LA.fallback_calls
    h = m(x)
    h.backward(dY)
    torch.cuda.synchronize()
    if fused:
        assert L.lora_linear_launch_count() - n0 == 5 and LA.fallback_calls == f0
    else:
        assert L.lora_linear_launch_count() == n0 and LA.fallback_calls == f0 + 1
    ref = oracle_ref(inp)
    f64 = lambda t: t.detach().double().cpu().numpy()
    assert_close("h", f64(h).reshape(spec.M, -1), ref["h"], TOL_HX)
    assert_close("dX", f64(x.grad).reshape(spec.M, -1), ref["dX"], TOL_HX)
    assert_close("dA", f64(m.lora_A.grad), ref["dA"], TOL_AB)
    assert_close("dB", f64(m.lora_B.grad), ref["dB"], TOL_AB)


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("kind", ["q4", "fp8", "nf4"])
def test_coded_module_matches_oracle(kind):
    """Modules over a 4-bit, FP8 and NF4 frozen weight: the fused layer's outputs and
    gradients against the oracle, and the merged weight against the oracle's."""
    import oracle
    spec = inputs.LayerSpec("shim-" + kind, 2 * 160, 384, 320, 16, alpha=32.0, seed=0x5A2,
                            q4=kind == "q4", fp8=kind == "fp8", nf4=kind == "nf4")
    inp = inputs.make_inputs(spec)
    if kind == "q4":
        m = LA.LoraLinear.from_q4(_u8(inp.Wq), _dev(inp.Wscale), r=spec.r, alpha=spec.alpha)
        wkw = dict(Wq=inp.Wq, Wscale=inp.Wscale)
    elif kind == "fp8":
        m = LA.LoraLinear.from_fp8(_u8(inp.W8), _dev(inp.W8scale), r=spec.r, alpha=spec.alpha)
        wkw = dict(W8=inp.W8, W8scale=inp.W8scale)
    else:
        m = LA.LoraLinear.from_nf4(_u8(inp.Wq), _dev(inp.Wscale), inp.codebook, r=spec.r, alpha=spec.alpha)
        wkw = dict(Wq=inp.Wq, Wscale=inp.Wscale, codebook=np.asarray(inp.codebook, np.float32).astype(np.float64))
    with torch.no_grad():
        m.lora_A.copy_(_dev(inp.A))
        m.lora_B.copy_(_dev(inp.B))
    x = _dev(inp.x).reshape(2, 160, 384).requires_grad_(True)
    dY = _dev(inp.dY).reshape(2, 160, 320)
    n0, f0 = L.lora_linear_launch_count(), LA.fallback_calls
    h = m(x)
    h.backward(dY)
    torch.cuda.synchronize()
    assert L.lora_linear_launch_count() - n0 == 5 and LA.fallback_calls == f0
    ref = oracle_ref(inp)
    f64 = lambda t: t.detach().double().cpu().numpy()
    assert_close("h", f64(h).reshape(spec.M, -1), ref["h"], TOL_HX)
    assert_close("dX", f64(x.grad).reshape(spec.M, -1), ref["dX"], TOL_HX)
    assert_close("dA", f64(m.lora_A.grad), ref["dA"], TOL_AB)
    assert_close("dB", f64(m.lora_B.grad), ref["dB"], TOL_AB)
    merged = f64(m.merged_weight())
    want = oracle.merged_weight(inp.A, inp.B, spec.s, **wkw)
    # one bf16 rounding of the exact merged value (plus fp32 sums): 2^-8 relative
    assert np.all(np.abs(merged - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)
