"""Several projections of one x stacked into one layer (rank_linear_lora_b200.multi):
host-side layout and the stacking identity, checked through the oracle on the CPU.

P projections h_p = x W_p^T + s (x A_p^T) B_p^T of one x, with the gradient of x summed
over them, are what the stacked layer must give.  The oracle run on the stacked
tensors (W, A by rows, B block-diagonal, alpha and r both times P) must reproduce
the oracle run on each projection alone.
"""
import numpy as np
import pytest
import torch

import oracle
from lora_cases import shared_input_projections
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200.multi import SharedInputProjections


def _bits(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.uint8:
        return t.numpy().copy()
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def _t16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _wkw(inp):
    return dict(Wq=inp.Wq, Wscale=inp.Wscale) if inp.spec.q4 else dict(W=inp.W)


CASES = [  # M, d_in, d_outs, r, alpha, q4
    (7, 24, (16, 8, 24), 8, 16.0, False),     # q/k/v-like, unequal widths
    (5, 128, (24, 40), 16, 32.0, True),       # gate/up-like, 4-bit weight
    (3, 16, (8,), 8, 8.0, False),             # one projection: the stack is the layer
]


@pytest.mark.parametrize("case", CASES, ids=["qkv", "gate_up_q4", "single"])
def test_stacked_layer_equals_the_separate_projections(case):
    M, d_in, d_outs, r, alpha, q4 = case
    layers = shared_input_projections(M, d_in, d_outs, r, alpha, q4, seed=0x5AE + M)
    st = SharedInputProjections(d_in, d_outs, r, alpha, q4=q4)
    for p, inp in enumerate(layers):
        if q4:
            st.load(p, Wq=torch.from_numpy(inp.Wq), Wscale=_t16(inp.Wscale), A=_t16(inp.A), B=_t16(inp.B))
        else:
            st.load(p, W=_t16(inp.W), A=_t16(inp.A), B=_t16(inp.B))
    P = len(d_outs)
    assert st.r_call == P * r and st.alpha_call == P * alpha
    assert st.alpha_call / st.r_call == alpha / r

    # the stacked B is block-diagonal: nothing outside projection p's block
    Bs = _bits(st.B)
    for p in range(P):
        assert np.array_equal(Bs[st.rows(p), st.ranks(p)], layers[p].B)
    off = np.ones_like(Bs, dtype=bool)
    for p in range(P):
        off[st.rows(p), st.ranks(p)] = False
    assert not Bs[off].any()

    x = layers[0].x
    dY = np.concatenate([inp.dY for inp in layers], axis=1)
    wkw = dict(Wq=_bits(st.Wq), Wscale=_bits(st.Wscale)) if q4 else dict(W=_bits(st.W))
    s_call = st.alpha_call / st.r_call
    h_all, xa_all = oracle.forward(x, _bits(st.A), Bs, s_call, **wkw)
    bw = oracle.backward(dY, x, _bits(st.A), Bs, s_call, xa_=xa_all, **wkw)

    dX_sum = np.zeros((M, d_in))
    dA_views = [v[0] for v in st.split_grads(torch.from_numpy(bw["dA"]), torch.from_numpy(bw["dB"]))]
    dB_views = [v[1] for v in st.split_grads(torch.from_numpy(bw["dA"]), torch.from_numpy(bw["dB"]))]
    h_views = st.split_h(torch.from_numpy(h_all))
    xa_views = st.split_xa(torch.from_numpy(xa_all))
    for p, inp in enumerate(layers):
        s = inp.spec.s
        h_p, xa_p = oracle.forward(x, inp.A, inp.B, s, **_wkw(inp))
        b_p = oracle.backward(inp.dY, x, inp.A, inp.B, s, xa_=xa_p, **_wkw(inp))
        dX_sum += b_p["dX"]
        np.testing.assert_allclose(h_views[p].numpy(), h_p, rtol=1e-12, atol=1e-12 * np.abs(h_p).max())
        np.testing.assert_array_equal(xa_views[p].numpy(), xa_p)
        np.testing.assert_allclose(dA_views[p].numpy(), b_p["dA"], rtol=1e-12, atol=1e-12 * np.abs(b_p["dA"]).max())
        np.testing.assert_allclose(dB_views[p].numpy(), b_p["dB"], rtol=1e-12, atol=1e-12 * np.abs(b_p["dB"]).max())
    np.testing.assert_allclose(bw["dX"], dX_sum, rtol=1e-12, atol=1e-12 * np.abs(dX_sum).max())


def test_views_alias_the_stacked_storage():
    st = SharedInputProjections(32, (16, 8), 8, 16.0)
    st.B_p(1).fill_(1.0)
    st.A_p(0).fill_(2.0)
    assert float(st.B[16:24, 8:16].sum()) == 64.0 and float(st.B.sum()) == 64.0
    assert float(st.A[:8].sum()) == 2.0 * 8 * 32 and float(st.A[8:].sum()) == 0.0
    (dA0, dB0), (dA1, dB1) = st.split_grads()
    st.grads.zero_()
    dB1.fill_(3.0)
    dA0.fill_(1.0)
    buf = st.grads.buf
    assert float(buf[: 16 * 32].sum()) == 8 * 32  # dA occupies the head: projection 0's rows
    assert float(st.grads.dB[16:24, 8:16].sum()) == 3.0 * 64 and float(st.grads.dB.sum()) == 3.0 * 64
    assert st.W_p(1).shape == (8, 32) and st.W_p(1).data_ptr() == st.W[16:].data_ptr()


@pytest.mark.parametrize("kw,msg", [
    (dict(d_outs=(16, 12), r=8, alpha=16.0), "multiple of 8"),
    (dict(d_outs=(16, 16), r=12, alpha=16.0), "r % 8"),
    (dict(d_outs=(16,) * 3, r=96, alpha=16.0), "P\\*r <= 256"),
    (dict(d_outs=(16, 16, 16), r=8, alpha=1.0 / 3.0), "exact in fp32"),
    (dict(d_outs=(), r=8, alpha=16.0), "at least one"),
    (dict(d_outs=(16, 16), r=8, alpha=3e38), "exact in fp32"),          # 2*alpha overflows fp32
    (dict(d_outs=(16, 16), r=8, alpha=float("nan")), "exact in fp32"),
])
def test_rejects_stacks_the_layer_cannot_take(kw, msg):
    with pytest.raises(ValueError, match=msg):
        SharedInputProjections(64, kw["d_outs"], kw["r"], kw["alpha"])


def test_alpha_rounded_to_fp32_as_the_single_call_does():
    """alpha = 0.1 is not an fp32 value; the library takes it as fp32(0.1), and so does
    the stack: 2 * fp32(0.1) / 16 is fp32(0.1) / 8 exactly."""
    st = SharedInputProjections(64, (16, 16), 8, 0.1)
    a32 = np.float32(0.1)
    assert np.float32(st.alpha_call) / np.float32(st.r_call) == a32 / np.float32(8)


def test_stacked_workload_spec():
    """The gate+up workload stacked on one x: B drawn block-diagonal, and the FLOPs
    are those of the two projections (the zero blocks are no work)."""
    spec = inputs.workload(2).layers[3]
    assert (spec.proj, spec.d_out, spec.r, spec.s) == (2, 22016, 32, 2.0)
    one = inputs.workload(2).layers[0]
    assert spec.flops == 2 * one.flops
    small = spec.with_(M=4, d_in=64, d_out=48, r=16, alpha=32.0)
    inp = inputs.make_inputs(small)
    B = inp.B
    assert not B[:24, 8:].any() and not B[24:, :8].any()
    assert B[:24, :8].all() and B[24:, 8:].all()  # N(0, 0.02^2) draws are nonzero
