"""The workspace-free forward (lora_linear_fwd_noalloc), for callers that cannot
allocate device memory: a plugin whose host framework owns every allocation, or a
service whose device-memory budget is fixed at start-up.  It runs the ordinary
forward's kernels on the library's fixed 4 MiB device scratch, so its h and s.xa must
be bit for bit those of lora_linear_fwd, call after call, and match the oracle.  A
bounded wait that runs out inside it must be reported by lora_linear_noalloc_check.
This file is collected last so a stop-at-first-failure run has already run every
other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import oracle
from lora_cases import TOL_HX, RMS_HX, ErrorTally, dev_bf16, host_f64
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200 import lora_linear as L

pytestmark = pytest.mark.gpu


def _oracle_check(inp, h, xa):
    """Every element of h and s.xa against the oracle (dense steps for the rows of h)."""
    sp = inp.spec
    xa_ = oracle.xa(inp.x, inp.A)
    Wf = oracle.weight(sp.d_out, sp.d_in, W=inp.W)
    th, tx = ErrorTally("h"), ErrorTally("xa_save")
    for r0 in range(0, sp.M, 1024):
        r1 = min(sp.M, r0 + 1024)
        th.add(host_f64(h[r0:r1]), oracle.h_dense(inp.x[r0:r1], inp.B, xa_[r0:r1], sp.s, Wf), r0)
    tx.add(host_f64(xa), sp.s * xa_)
    th.check(TOL_HX, RMS_HX)
    tx.check((2 ** -8, 1e-6), RMS_HX)


@pytest.mark.parametrize("shape", [(520, 640, 768, 16), (4096, 4096, 4096, 8)], ids=["ragged", "attn-proj"])
def test_fwd_noalloc_matches_fwd_on_two_calls(shape):
    M, d_in, d_out, r = shape
    spec = inputs.LayerSpec("noalloc", M, d_in, d_out, r, alpha=2.0 * r, seed=0xA110C + M)
    inp = inputs.make_inputs(spec)
    x, W, A, B = (dev_bf16(a) for a in (inp.x, inp.W, inp.A, inp.B))
    h_ref = torch.empty(M, d_out, dtype=torch.bfloat16, device="cuda")
    xa_ref = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    # The ordinary forward on a workspace of the scratch's 4 MiB: the same plan as the
    # workspace-free call (the full workspace may add the K-split hand-over buffer, whose
    # last-wave tiles sum in another order).
    ws = torch.zeros(4 << 20, dtype=torch.uint8, device="cuda")
    L.lora_linear_fwd(x, W, A, B, h_ref, xa_ref, spec.alpha, ws)
    L.lora_linear_check(ws)
    _oracle_check(inp, h_ref, xa_ref)
    # and on the full workspace (K-split tail where the shape has one), against the oracle
    h_full = torch.empty_like(h_ref)
    ws_full = L.workspace(L.OP_FWD, M, d_in, d_out, r)
    L.lora_linear_fwd(x, W, A, B, h_full, None, spec.alpha, ws_full)
    L.lora_linear_check(ws_full)
    _oracle_check(inp, h_full, xa_ref)
    for call in range(2):
        h = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
        xa = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda")
        L.lora_linear_fwd_noalloc(x, W, A, B, h, xa, spec.alpha)
        L.lora_linear_noalloc_check()
        assert torch.equal(h.view(torch.int16), h_ref.view(torch.int16)), f"call {call}: h differs"
        assert torch.equal(xa.view(torch.int16), xa_ref.view(torch.int16)), f"call {call}: s.xa differs"
    # without xa_save the scratch itself holds s.xa between the two kernels
    h = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.lora_linear_fwd_noalloc(x, W, A, B, h, None, spec.alpha)
    L.lora_linear_noalloc_check()
    assert torch.equal(h.view(torch.int16), h_ref.view(torch.int16)), "h differs without xa_save"


def test_fwd_noalloc_timeout_is_reported_and_kept_until_checked():
    """A bounded wait that runs out on the scratch's error word (the self-test's wait on
    a barrier nothing arrives on) is reported by lora_linear_noalloc_check even after a
    later forward call, then cleared; the scratch then serves a correct forward."""
    M, d_in, d_out, r = 200, 256, 192, 8
    spec = inputs.LayerSpec("noalloc-timeout", M, d_in, d_out, r, alpha=16.0, seed=0xA11)
    inp = inputs.make_inputs(spec)
    x, W, A, B = (dev_bf16(a) for a in (inp.x, inp.W, inp.A, inp.B))
    h = torch.empty(M, d_out, dtype=torch.bfloat16, device="cuda")
    xa = torch.empty(M, r, dtype=torch.bfloat16, device="cuda")
    L.lora_linear_noalloc_check()  # nothing recorded yet
    L.lora_linear_noalloc_selftest_timeout(2000)  # 2 ms
    L.lora_linear_fwd_noalloc(x, W, A, B, h, xa, spec.alpha)  # must not clear the record
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_noalloc_check()
    assert e.value.status == 6  # LORA_ERR_TIMEOUT
    L.lora_linear_noalloc_check()  # cleared
    L.lora_linear_fwd_noalloc(x, W, A, B, h, xa, spec.alpha)
    L.lora_linear_noalloc_check()
    _oracle_check(inp, h, xa)


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
    L.lora_linear_noalloc_check()
