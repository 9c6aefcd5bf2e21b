"""Several projections of one x run as one stacked layer on the GPU, against the oracle
run on each projection alone: h_p, s.xa_p, dA_p and dB_p per projection, and dX against
the sum of the projections' dX (the gradient of the shared x)."""
import numpy as np
import pytest
import torch

import oracle
from lora_cases import (RMS_AB, RMS_HX, TOL_AB, TOL_HX, assert_close, dev_bf16, dev_u8, host_f64,
                        shared_input_projections)
from rank_linear_lora_b200 import lora_linear as L
from rank_linear_lora_b200.multi import SharedInputProjections

pytestmark = pytest.mark.gpu

CASES = [  # M, d_in, d_outs, r, alpha, q4
    (200, 320, (264, 64, 64), 8, 16.0, False),   # q/k/v-like: unequal widths, ragged tiles
    (136, 512, (200, 136), 16, 32.0, True),      # gate/up-like on the 4-bit weight
    (129, 256, (128, 256, 72, 64), 32, 64.0, False),  # four projections, r_call = 128
]


@pytest.mark.parametrize("case", CASES, ids=["qkv", "gate_up_q4", "four_r32"])
def test_stacked_projections_match_the_oracle(case):
    M, d_in, d_outs, r, alpha, q4 = case
    layers = shared_input_projections(M, d_in, d_outs, r, alpha, q4, seed=0x3A1 + M)
    st = SharedInputProjections(d_in, d_outs, r, alpha, q4=q4, device="cuda")
    for p, inp in enumerate(layers):
        if q4:
            st.load(p, Wq=dev_u8(inp.Wq), Wscale=dev_bf16(inp.Wscale), A=dev_bf16(inp.A), B=dev_bf16(inp.B))
        else:
            st.load(p, W=dev_bf16(inp.W), A=dev_bf16(inp.A), B=dev_bf16(inp.B))
    x = dev_bf16(layers[0].x)
    dY = dev_bf16(np.concatenate([inp.dY for inp in layers], axis=1))
    h = torch.empty(M, st.d_out, dtype=torch.bfloat16, device="cuda")
    xa = torch.empty(M, st.r_call, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(M, d_in, dtype=torch.bfloat16, device="cuda")
    ws_f, ws_b = st.workspaces(M, device="cuda")
    st.forward(x, h, xa, ws_f)
    st.backward(dY, x, xa, dX, ws_b)
    L.lora_linear_check(ws_f)
    L.lora_linear_check(ws_b)
    torch.cuda.synchronize()

    dX_ref = np.zeros((M, d_in))
    grads = st.split_grads()
    for p, inp in enumerate(layers):
        s = inp.spec.s
        wkw = dict(Wq=inp.Wq, Wscale=inp.Wscale) if q4 else dict(W=inp.W)
        h_p, xa_p = oracle.forward(inp.x, inp.A, inp.B, s, **wkw)
        b_p = oracle.backward(inp.dY, inp.x, inp.A, inp.B, s, xa_=xa_p, **wkw)
        dX_ref += b_p["dX"]
        assert_close(f"h_{p}", host_f64(st.split_h(h)[p]), h_p, TOL_HX, RMS_HX)
        assert_close(f"xa_{p}", host_f64(st.split_xa(xa)[p]), s * xa_p, (2 ** -8, 1e-6), RMS_HX)
        assert_close(f"dA_{p}", host_f64(grads[p][0]), b_p["dA"], TOL_AB, RMS_AB)
        assert_close(f"dB_{p}", host_f64(grads[p][1]), b_p["dB"], TOL_AB, RMS_AB)
    assert_close("dX", host_f64(dX), dX_ref, TOL_HX, RMS_HX)
