"""The every-element checker the full-size GPU tests use, exercised on the CPU: fed the
oracle's own results rounded to bf16 (what a correct GPU path returns) it passes; one
corrupted element anywhere in h or dX, a few times the per-element bound, fails it.
That single-element case is exactly what a projection check cannot see."""
import numpy as np
import pytest
import torch

from lora_cases import compare_every_element
import oracle
from rank_linear_lora_b200 import inputs


class _HostLayer:
    """Stands in for the device layer: bf16 results of the oracle on the host."""

    def __init__(self, inp):
        sp = inp.spec
        ref_h, xa_ = oracle.forward(inp.x, inp.A, inp.B, sp.s, W=inp.W)
        bw = oracle.backward(inp.dY, inp.x, inp.A, inp.B, sp.s, W=inp.W, xa_=xa_)
        self.h = torch.from_numpy(ref_h).to(torch.bfloat16)
        self.dX = torch.from_numpy(bw["dX"]).to(torch.bfloat16)
        self.xa = torch.from_numpy(sp.s * xa_).to(torch.bfloat16)
        self.dA = torch.from_numpy(bw["dA"]).to(torch.float32)
        self.dB = torch.from_numpy(bw["dB"]).to(torch.float32)


@pytest.fixture(scope="module")
def layer():
    spec = inputs.LayerSpec("checker", 300, 192, 136, 8, alpha=16.0, seed=0xC4)
    inp = inputs.make_inputs(spec)
    return inp, _HostLayer(inp)


def test_rounded_oracle_passes(layer):
    inp, hl = layer
    res = compare_every_element(hl, inp, block_rows=64)
    assert res["elements"] == 300 * 136 + 300 * 192 + 300 * 8 + 8 * 192 + 136 * 8
    assert all(v <= 1.0 for v in res["worst"].values())


@pytest.mark.parametrize("name,where", [("h", (0, 0)), ("h", (299, 135)), ("dX", (150, 77)), ("dX", (64, 191))])
def test_one_bad_element_fails(layer, name, where):
    inp, hl = layer
    t = getattr(hl, name)
    saved = t[where].clone()
    bound = 1e-2 * float(t.float().abs().max()) + 1e-3
    t[where] = saved + 3.0 * bound
    try:
        with pytest.raises(AssertionError, match=name):
            compare_every_element(hl, inp, block_rows=64)
    finally:
        t[where] = saved
