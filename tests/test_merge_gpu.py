"""Deploy-time merge W' = W + s.B.A (lora_linear_merge / _q4) against the oracle, on
every element.  The kernel forms the exact bf16 products, sums them in fp32 and rounds
once to bf16, so each element is within one bf16 ulp of the exact merged value and
nearly all are its correctly rounded value."""
import numpy as np
import pytest
import torch

import oracle
from lora_cases import dev_bf16, dev_u8
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200 import lora_linear as L

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _check(got_bits: np.ndarray, ref: np.ndarray, absmag: np.ndarray, r: int, min_exact: float = 0.99):
    """Within one bf16 ulp of the exact value, plus the fp32 error of an r-term sum and
    the final fused multiply-add, (r + 2) * 2^-24 * (|w| + s * sum_j |B||A|), which only
    matters where w and the update nearly cancel."""
    got = inputs.bf16_bits_to_f32(got_bits).astype(np.float64)
    mag = np.maximum(np.abs(ref), np.finfo(np.float32).tiny)
    ulp = np.exp2(np.floor(np.log2(mag)) - 7)  # bf16: 7 fraction bits
    err = np.abs(got - ref)
    bad = err > ulp + (r + 2) * 2.0 ** -24 * absmag
    assert not bad.any(), (f"{int(bad.sum())} elements off by more than one bf16 ulp; first at "
                           f"{np.argwhere(bad)[0]}: got {got[bad][0]:.8g}, exact {ref[bad][0]:.8g}")
    exact = np.mean(got_bits == inputs.to_bf16_bits(ref))
    assert exact >= min_exact, f"only {exact:.4f} of the elements are the correctly rounded value"


def _merge(inp, spec, in_place=False):
    A, B = dev_bf16(inp.A), dev_bf16(inp.B)
    if spec.q4:
        out = torch.empty(spec.d_out, spec.d_in, dtype=torch.bfloat16, device="cuda")
        L.lora_linear_merge_q4(dev_u8(inp.Wq), dev_bf16(inp.Wscale), A, B, out, spec.alpha)
    else:
        W = dev_bf16(inp.W)
        out = W if in_place else torch.empty_like(W)
        L.lora_linear_merge(W, A, B, out, spec.alpha)
    L.lora_linear_merge_check()
    return _bits(out)


def _ref(inp, spec, r0=0, r1=None):
    """Oracle merged weight of rows r0..r1, and the magnitude sum behind the tolerance."""
    r1 = spec.d_out if r1 is None else r1
    if spec.q4:
        wkw = dict(Wq=inp.Wq[r0:r1], Wscale=inp.Wscale[r0:r1])
    else:
        wkw = dict(W=inp.W[r0:r1])
    ref = oracle.merged_weight(inp.A, inp.B[r0:r1], spec.s, **wkw)
    w = oracle.weight(r1 - r0, spec.d_in, **wkw)
    A = np.abs(inputs.bf16_bits_to_f32(inp.A).astype(np.float64))
    B = np.abs(inputs.bf16_bits_to_f32(inp.B[r0:r1]).astype(np.float64))
    return ref, np.abs(w) + abs(spec.s) * (B @ A)


SHAPES = [  # d_out, d_in, r, q4
    # r <= 64: tensor-core kernel, 128 x 128 tiles
    (200, 320, 8, False),     # ragged last tile: its second 64-column chunk lies past d_in
    (333, 520, 24, False),    # ragged rows; K = 32 with ranks 24..31 zero-filled
    (129, 136, 16, False),    # one row and 8 columns into the last tiles
    (1, 64, 8, False),        # one row, one chunk
    (1000, 4104, 40, False),  # 264 tiles: two per CTA on most SMs
    (1200, 6000, 64, False),  # 470 tiles: the three stages and two accumulators wrap
    (256, 384, 48, False),
    (64, 1024, 56, False),
    (200, 320, 16, True),
    (300, 1216, 64, True),    # 4-bit: a last tile half past d_in
    (520, 4160, 32, True),
    # r > 64: CUDA-core kernel
    (64, 264, 72, False),     # r crosses the 64-rank staging chunk
    (40, 512, 256, False),
    (96, 512, 72, True),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "out%d_in%d_r%d%s" % (s[0], s[1], s[2], "_q4" if s[3] else ""))
def test_merge_matches_oracle(shape):
    d_out, d_in, r, q4 = shape
    spec = inputs.LayerSpec("merge", 8, d_in, d_out, r, alpha=2.0 * r, q4=q4, seed=0x3F + d_out)
    inp = inputs.make_inputs(spec)
    _check(_merge(inp, spec), *_ref(inp, spec), r)


def test_merge_in_place_and_zero_adapter():
    spec = inputs.LayerSpec("merge", 8, 320, 200, 16, alpha=32.0, seed=0x40)
    inp = inputs.make_inputs(spec)
    _check(_merge(inp, spec, in_place=True), *_ref(inp, spec), spec.r)
    inp0 = inputs.make_inputs(spec, zero_B=True)
    assert np.array_equal(_merge(inp0, spec), inp0.W)  # nothing to add: W' is W bitwise


@pytest.mark.parametrize("idx", [1, 4], ids=["attn-proj", "q4-up-proj"])
def test_merge_full_size(idx):
    """The full weights of the attention-projection (4096 x 4096, r=8) and 4-bit up-
    projection (28672 x 8192, r=16) workloads, every element, oracle in row blocks."""
    spec = inputs.workload(idx).layers[0]
    inp = inputs.make_inputs(spec)
    got = _merge(inp, spec)
    for r0 in range(0, spec.d_out, 4096):
        r1 = min(spec.d_out, r0 + 4096)
        _check(got[r0:r1], *_ref(inp, spec, r0, r1), spec.r)


def test_merge_rejects_bad_arguments():
    W = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(8, 256, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(64, 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_merge(W, A, B, W, float("nan"))
    assert e.value.status == 1
    with pytest.raises(L.LoraError) as e:  # 4-bit base needs d_in % 64 == 0
        L.lora_linear_merge_q4(torch.zeros(64, 100, dtype=torch.uint8, device="cuda"),
                               torch.zeros(64, 3, dtype=torch.bfloat16, device="cuda"),
                               torch.zeros(8, 200, dtype=torch.bfloat16, device="cuda"), B,
                               torch.zeros(64, 200, dtype=torch.bfloat16, device="cuda"), 1.0)
    assert e.value.status == 1
