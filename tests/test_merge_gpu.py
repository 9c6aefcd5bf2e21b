"""Deploy-time merge W' = W + s.B.A (lora_linear_merge / _q4) against the oracle, on
every element, for each stored weight format.  The kernel forms the exact bf16
products, sums them in fp32 on the tensor cores, adds the decoded weight in fp32 and
rounds once to bf16, so each element is within one bf16 ulp of the exact merged value
and nearly all are its correctly rounded value."""
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
    out = torch.empty(spec.d_out, spec.d_in, dtype=torch.bfloat16, device="cuda")
    if spec.q4:
        L.lora_linear_merge_q4(dev_u8(inp.Wq), dev_bf16(inp.Wscale), A, B, out, spec.alpha)
    elif spec.nf4:
        L.lora_linear_merge_nf4(dev_u8(inp.Wq), dev_bf16(inp.Wscale), inp.codebook, A, B, out, spec.alpha)
    elif spec.fp8:
        L.lora_linear_merge_fp8(dev_u8(inp.W8), dev_bf16(inp.W8scale), A, B, out, spec.alpha)
    else:
        W = dev_bf16(inp.W)
        out = W if in_place else out
        L.lora_linear_merge(W, A, B, out, spec.alpha)
    L.lora_linear_merge_check()
    return _bits(out)


def _ref(inp, spec, r0=0, r1=None):
    """Oracle merged weight of rows r0..r1, and the magnitude sum behind the tolerance.
    The codebook reaches the library as fp32, so the oracle takes the same fp32 values."""
    r1 = spec.d_out if r1 is None else r1
    if spec.q4:
        wkw = dict(Wq=inp.Wq[r0:r1], Wscale=inp.Wscale[r0:r1])
    elif spec.nf4:
        wkw = dict(Wq=inp.Wq[r0:r1], Wscale=inp.Wscale[r0:r1],
                   codebook=np.asarray(inp.codebook, dtype=np.float32).astype(np.float64))
    elif spec.fp8:
        wkw = dict(W8=inp.W8[r0:r1], W8scale=inp.W8scale[r0:r1])
    else:
        wkw = dict(W=inp.W[r0:r1])
    ref = oracle.merged_weight(inp.A, inp.B[r0:r1], spec.s, **wkw)
    w = oracle.weight(r1 - r0, spec.d_in, **wkw)
    A = np.abs(inputs.bf16_bits_to_f32(inp.A).astype(np.float64))
    B = np.abs(inputs.bf16_bits_to_f32(inp.B[r0:r1]).astype(np.float64))
    return ref, np.abs(w) + abs(spec.s) * (B @ A)


FMT = {"bf16": {}, "q4": dict(q4=True), "fp8": dict(fp8=True), "nf4": dict(nf4=True)}

SHAPES = [  # d_out, d_in, r, weight format
    (200, 320, 8, "bf16"),      # ragged last tile: its second 64-column box lies past d_in
    (333, 520, 24, "bf16"),     # ragged rows; K = 32 with ranks 24..31 zero-filled
    (129, 136, 16, "bf16"),     # one row and 8 columns into the last tiles
    (1, 64, 8, "bf16"),         # one row, one box
    (1000, 4104, 40, "bf16"),   # 264 tiles: two per CTA on most SMs
    (1200, 6000, 64, "bf16"),   # 470 tiles: the rings and both accumulators wrap
    (256, 384, 48, "bf16"),
    (64, 1024, 56, "bf16"),
    (64, 264, 72, "bf16"),      # two rank chunks, the second 8 ranks wide
    (40, 512, 256, "bf16"),     # four full rank chunks
    (700, 2048, 136, "bf16"),   # three rank chunks over several tiles per CTA
    (200, 320, 16, "q4"),
    (300, 1216, 64, "q4"),      # 4-bit: a last tile half past d_in
    (520, 4160, 32, "q4"),
    (96, 512, 72, "q4"),
    (200, 320, 16, "fp8"),
    (333, 1040, 24, "fp8"),     # FP8: d_in % 16 == 0 with a ragged last tile
    (1500, 4096, 128, "fp8"),
    (200, 320, 8, "nf4"),
    (333, 1216, 32, "nf4"),
    (1100, 4160, 96, "nf4"),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "out%d_in%d_r%d_%s" % s)
def test_merge_matches_oracle(shape):
    d_out, d_in, r, fmt = shape
    spec = inputs.LayerSpec("merge", 8, d_in, d_out, r, alpha=2.0 * r, seed=0x3F + d_out, **FMT[fmt])
    inp = inputs.make_inputs(spec)
    _check(_merge(inp, spec), *_ref(inp, spec), r)


def test_merge_in_place_and_zero_adapter():
    spec = inputs.LayerSpec("merge", 8, 320, 200, 16, alpha=32.0, seed=0x40)
    inp = inputs.make_inputs(spec)
    _check(_merge(inp, spec, in_place=True), *_ref(inp, spec), spec.r)
    inp0 = inputs.make_inputs(spec, zero_B=True)
    assert np.array_equal(_merge(inp0, spec), inp0.W)  # nothing to add: W' is W bitwise


@pytest.mark.parametrize("case", [(1, "bf16"), (4, "q4"), (1, "fp8"), (4, "nf4")],
                         ids=["attn-proj", "q4-up-proj", "attn-proj-fp8", "up-proj-nf4"])
def test_merge_full_size(case):
    """The full weights of the attention-projection (4096 x 4096, r=8) and up-projection
    (28672 x 8192, r=16) workloads in the bench's formats, every element, oracle in row
    blocks."""
    idx, fmt = case
    spec = inputs.workload(idx).layers[0].with_(**{"q4": False, **FMT[fmt]})
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
