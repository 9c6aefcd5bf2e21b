"""The workspace-free forward (lora_linear_fwd_noalloc), for callers that cannot
allocate device memory: a plugin whose host framework owns every allocation, or a
service whose device-memory budget is fixed at start-up.  It must give the same h and
s.xa as the ordinary forward, call after call, using only the library's fixed 4 MiB
device scratch.  This file is collected last so a stop-at-first-failure run has
already run every other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from lora_cases import TOL_HX, RMS_HX, assert_close, dev_bf16
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200 import lora_linear as L

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("shape", [(520, 640, 768, 16), (4096, 4096, 4096, 8)], ids=["ragged", "attn-proj"])
def test_fwd_noalloc_matches_fwd_on_two_calls(shape):
    M, d_in, d_out, r = shape
    spec = inputs.LayerSpec("noalloc", M, d_in, d_out, r, alpha=2.0 * r, seed=0xA110C + M)
    inp = inputs.make_inputs(spec)
    x, W, A, B = (dev_bf16(a) for a in (inp.x, inp.W, inp.A, inp.B))
    h_ref = torch.empty(M, d_out, dtype=torch.bfloat16, device="cuda")
    xa_ref = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    ws = L.workspace(L.OP_FWD, M, d_in, d_out, r)
    L.lora_linear_fwd(x, W, A, B, h_ref, xa_ref, spec.alpha, ws)
    L.lora_linear_check(ws)
    for _ in range(2):
        h = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
        xa = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.lora_linear_fwd_noalloc(x, W, A, B, h, xa, spec.alpha)
        torch.cuda.synchronize()
        assert_close("h", _f64(h), _f64(h_ref), TOL_HX, RMS_HX)
        assert_close("xa_save", _f64(xa), _f64(xa_ref), TOL_HX, RMS_HX)


def test_fwd_noalloc_rejects_problems_beyond_its_scratch():
    M, d_in, d_out, r = 16384, 4096, 4096, 128   # needs ~12 MiB of scratch > 4 MiB
    assert L.lora_linear_workspace_size(L.OP_FWD, M, d_in, d_out, r) > 4 << 20
    x = torch.zeros(M, d_in, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(d_out, d_in, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(r, d_in, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(d_out, r, dtype=torch.bfloat16, device="cuda")
    h = torch.zeros(M, d_out, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_fwd_noalloc(x, W, A, B, h, None, 256.0)
    assert e.value.status == 4
