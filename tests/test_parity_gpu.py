"""GPU path against the fp64 oracle, element by element, through the C ABI.

Every test compares every output element.  Small and ragged shapes use the oracle's
plain loops; the full-size workloads, in the launch configuration the benchmark times,
use the oracle's dense steps for the rows of h and dX, and also check all row and
column projections of h and dX.
"""
import numpy as np
import pytest
import torch

from lora_cases import (DeviceLayer, assert_close, check_projections, compare_all, compare_every_element, oracle_ref,
                        sample_rows, TOL_AB, TOL_HX, RMS_AB, RMS_HX)
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200 import lora_linear as L

pytestmark = pytest.mark.gpu


def _run_full(spec, **mk):
    inp = inputs.make_inputs(spec, **mk)
    dl = DeviceLayer(inp)
    dl.forward()
    dl.backward()
    dl.check()
    return inp, dl


def test_config0_tiny_full():
    spec = inputs.workload(0).layers[0]
    inp, dl = _run_full(spec)
    compare_all(dl.results(), oracle_ref(inp), spec.s)


RAGGED = [
    # (M, d_in, d_out, r): token tails, K tails (d % 64 != 0), N tails, rank tails (r % 16 != 0)
    (200, 328, 200, 8),
    (129, 64, 72, 16),
    (1, 8, 8, 8),
    (300, 520, 264, 24),
    (77, 256, 512, 64),
    (160, 192, 128, 128),
    (130, 136, 520, 256),
    (513, 1032, 776, 40),
]


@pytest.mark.parametrize("shape", RAGGED, ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_ragged_full(shape):
    M, di, do, r = shape
    spec = inputs.LayerSpec("ragged", M, di, do, r, alpha=2.0 * r, seed=0xBEEF + M)
    inp, dl = _run_full(spec)
    compare_all(dl.results(), oracle_ref(inp), spec.s)


def test_lora_dominant():
    """B drawn 50x larger than the workloads' init so the rank-r term dominates h and dX:
    any dropped or mis-indexed piece of the K tail shows up far outside tolerance."""
    spec = inputs.LayerSpec("dominant", 192, 320, 448, 24, alpha=48.0, seed=77)
    inp = inputs.make_inputs(spec)
    inp.B = inputs.to_bf16_bits(inputs.bf16_bits_to_f32(inp.B).astype(np.float64) * 50.0)
    dl = DeviceLayer(inp)
    dl.forward()
    dl.backward()
    dl.check()
    compare_all(dl.results(), oracle_ref(inp), spec.s)


def test_zero_B_gives_zero_dA_exactly():
    spec = inputs.workload(0).layers[0].with_(M=200)
    inp, dl = _run_full(spec, zero_B=True)
    got = dl.results()
    assert np.all(got["dA"] == 0.0)
    compare_all(got, oracle_ref(inp), spec.s)


def test_zero_A_gives_zero_dB_exactly():
    spec = inputs.workload(0).layers[0].with_(M=136)
    inp, dl = _run_full(spec, zero_A=True)
    got = dl.results()
    assert np.all(got["dB"] == 0.0) and np.all(got["xa"] == 0.0)
    compare_all(got, oracle_ref(inp), spec.s)


def test_recompute_xa_and_skip_dx():
    """Backward without the saved s.xa recomputes it (same dB); dX = NULL skips dX only."""
    spec = inputs.LayerSpec("opt", 264, 384, 320, 16, alpha=32.0, seed=5)
    inp = inputs.make_inputs(spec)
    dl = DeviceLayer(inp)
    dl.forward()
    dl.backward(use_xa=True)
    torch.cuda.synchronize()
    dA1, dB1, dX1 = dl.dA.clone(), dl.dB.clone(), dl.dX.clone()
    dl.dA.fill_(float("nan"))
    dl.dB.fill_(float("nan"))
    dl.dX.fill_(7.0)
    dl.backward(use_xa=False, want_dx=False)
    dl.check()
    assert torch.equal(dl.dA, dA1) and torch.equal(dl.dB, dB1)
    assert torch.all(dl.dX == 7.0)
    ref = oracle_ref(inp)
    assert_close("dX", dX1.double().cpu().numpy(), ref["dX"], TOL_HX, RMS_HX)


def test_deterministic():
    spec = inputs.LayerSpec("det", 384, 512, 384, 8, alpha=16.0, seed=9)
    dl = DeviceLayer(inputs.make_inputs(spec))
    outs = []
    for _ in range(2):
        dl.forward()
        dl.backward()
        torch.cuda.synchronize()
        outs.append([t.clone() for t in (dl.h, dl.xa, dl.dX, dl.dA, dl.dB)])
    dl.check()
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.uint8) if b.dtype == torch.bfloat16 else b)


def test_outputs_stay_in_bounds():
    """Guard bands after every output: the kernels write exactly the declared extents."""
    spec = inputs.LayerSpec("guard", 200, 328, 200, 8, alpha=16.0, seed=11)
    inp = inputs.make_inputs(spec)
    dl = DeviceLayer(inp)
    M, di, do, r = spec.M, spec.d_in, spec.d_out, spec.r
    pad = 4096
    hb = torch.full((M * do + pad,), 3.0, dtype=torch.bfloat16, device="cuda")
    xb = torch.full((M * r + pad,), 3.0, dtype=torch.bfloat16, device="cuda")
    dxb = torch.full((M * di + pad,), 3.0, dtype=torch.bfloat16, device="cuda")
    dab = torch.full((r * di + pad,), 3.0, dtype=torch.float32, device="cuda")
    dbb = torch.full((do * r + pad,), 3.0, dtype=torch.float32, device="cuda")
    dl.h, dl.xa, dl.dX = hb[:M * do].view(M, do), xb[:M * r].view(M, r), dxb[:M * di].view(M, di)
    dl.dA, dl.dB = dab[:r * di].view(r, di), dbb[:do * r].view(do, r)
    dl.forward()
    dl.backward()
    dl.check()
    for buf, n in ((hb, M * do), (xb, M * r), (dxb, M * di), (dab, r * di), (dbb, do * r)):
        assert torch.all(buf[n:] == 3.0)
    compare_all(dl.results(), oracle_ref(inp), spec.s)


def test_status_codes_on_device():
    spec = inputs.workload(0).layers[0]
    dl = DeviceLayer(inputs.make_inputs(spec))
    small = dl.ws_f[: dl.ws_f.numel() // 2]
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_fwd(dl.x, dl.W, dl.A, dl.B, dl.h, dl.xa, spec.alpha, small)
    assert e.value.status == 4
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_fwd(dl.x, dl.W, dl.A, dl.B, dl.h, dl.xa, spec.alpha, dl.ws_f[16:])
    assert e.value.status == 2
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_fwd(dl.x, dl.W, dl.A, dl.B, dl.h, dl.xa, float("inf"), dl.ws_f)
    assert e.value.status == 1
    dl.check()


def test_timing_hooks_count_launches():
    spec = inputs.workload(0).layers[0]
    dl = DeviceLayer(inputs.make_inputs(spec))
    L.lora_linear_timing_read()
    n0 = L.lora_linear_launch_count()
    L.lora_linear_timing_enable(True)
    try:
        dl.forward()
        dl.backward()
        rec = L.lora_linear_timing_read()
    finally:
        L.lora_linear_timing_enable(False)
    assert L.lora_linear_launch_count() - n0 == 5
    assert all(rec[k][1] == 1 and rec[k][0] > 0 for k in L.KERNEL_KINDS)


# Shapes whose main-GEMM tile count leaves a partial last wave on 148 SMs, so the
# last-wave 128 x 256 tiles are cut along N into 128 x 128 or 128 x 64 tiles.
TAIL_WAVE = [
    (2560, 1024, 2048, 8),    # forward: 160 tiles -> 12 tail tiles x 4 (K-major B, narrow maps)
    (2560, 2048, 1024, 16),   # dX: 160 tiles -> 12 tail tiles x 4 (MN-major B)
    (2304, 512, 2816, 16),    # forward: 198 tiles -> 50 tail tiles x 2
    (2304, 2816, 512, 8),     # dX: 198 tiles -> 50 tail tiles x 2
    (1920, 2048, 2560, 24),   # forward: 150 tiles -> 2 tail tiles x 4, rank tail r % 16 != 0
]


@pytest.mark.parametrize("shape", TAIL_WAVE, ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_tail_wave_split(shape):
    M, di, do, r = shape
    spec = inputs.LayerSpec("streamk", M, di, do, r, alpha=2.0 * r, seed=0x51 + M + di)
    inp, dl = _run_full(spec)
    compare_all(dl.results(), oracle_ref(inp), spec.s)


# Forward shapes whose CTA-pair GEMM (256 x 256 tiles on 74 pairs) leaves a last wave of
# at most 37 tiles: each is cut along K into two items on two pairs (the library's
# choice for the bf16 weight), the first handing its fp32 accumulator to the second.
KSPLIT = [
    (1280, 4096, 4096, 8),    # 80 tiles: 6 tail tiles, 32 + 33 K blocks
    (1200, 2040, 4000, 24),   # ragged M, K and N; the rank-r block in the second half
    (1280, 2048, 4096, 136),  # three rank-r blocks, all in the second half
    (2304, 3072, 2816, 16),   # 99 tiles: 25 tail tiles on 50 pairs
]


def _check_forward(dl, ref, s):
    got = dl.results()
    assert_close("h", got["h"], ref["h"], TOL_HX, RMS_HX)
    assert_close("xa_save", got["xa"], s * ref["xa"], (2 ** -8, 1e-6), RMS_HX)


@pytest.mark.parametrize("shape", KSPLIT, ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_forward_last_wave_cut_along_k(shape):
    """Every element against the oracle with the K-split tail and with the N-split one
    (plan override), and the K-split result the same bit for bit on a second call."""
    M, di, do, r = shape
    assert L.lora_linear_get_plan(L.OP_FWD, M, di, do, r)["fwd_tail"] == 3
    assert L.lora_linear_get_plan(L.OP_FWD, M, 1024, do, r)["fwd_tail"] == 1  # short K: cut along N
    spec = inputs.LayerSpec("ksplit", M, di, do, r, alpha=2.0 * r, seed=0x4B + M + di)
    inp = inputs.make_inputs(spec)
    ref = oracle_ref(inp)
    dl = DeviceLayer(inp)
    dl.forward()
    dl.check()
    h1 = dl.h.clone()
    _check_forward(dl, ref, spec.s)
    dl.forward()
    dl.check()
    assert torch.equal(h1.view(torch.int16), dl.h.view(torch.int16)), "K-split tail not deterministic"
    plan = L.lora_linear_get_plan(L.OP_FWD, M, di, do, r)
    plan["fwd_tail"] = 1
    try:
        L.lora_linear_set_plan(M, di, do, r, plan)
        dn = DeviceLayer(inp)
        dn.forward()
        dn.check()
        _check_forward(dn, ref, spec.s)
    finally:
        L.lora_linear_set_plan(M, di, do, r, None)


@pytest.mark.parametrize("shape", [(1280, 4096, 4096, 8), (1200, 4000, 2040, 24)], ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_dx_last_wave_cut_along_k(shape):
    """The backward with the dX GEMM's last wave cut along K (plan dx_overlap 3; dA and
    dB after it): every output against the oracle, dX the same bit for bit twice."""
    M, di, do, r = shape
    spec = inputs.LayerSpec("dxksplit", M, di, do, r, alpha=2.0 * r, seed=0xD5 + M + do)
    inp = inputs.make_inputs(spec)
    plan = L.lora_linear_get_plan(L.OP_BWD, M, di, do, r)
    plan["dx_overlap"] = 3
    try:
        L.lora_linear_set_plan(M, di, do, r, plan)
        assert L.lora_linear_get_plan(L.OP_BWD, M, di, do, r)["dx_overlap"] == 3
        dl = DeviceLayer(inp)
        dl.forward()
        dl.backward()
        dl.check()
        dx1 = dl.dX.clone()
        compare_all(dl.results(), oracle_ref(inp), spec.s)
        dl.backward()
        dl.check()
        assert torch.equal(dx1.view(torch.int16), dl.dX.view(torch.int16)), "K-split dX not deterministic"
    finally:
        L.lora_linear_set_plan(M, di, do, r, None)


@pytest.mark.parametrize("shape", [(1280, 4096, 4096, 8), (1280, 4032, 2040, 16), (1200, 4000, 2040, 24)],
                         ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_dx_last_wave_cut_along_n(shape):
    """The backward with the dX GEMM's last wave cut along N (plan dx_overlap 2): its
    tail tiles stage 64 weight columns per CTA by 2D copies while whole tiles take the
    3D column-chunk copy (d_in a multiple of 64; the last shape only 2D copies).  Every
    output against the oracle."""
    M, di, do, r = shape
    spec = inputs.LayerSpec("dxnsplit", M, di, do, r, alpha=2.0 * r, seed=0xD6 + M + di)
    inp = inputs.make_inputs(spec)
    plan = L.lora_linear_get_plan(L.OP_BWD, M, di, do, r)
    plan["dx_overlap"] = 2
    try:
        L.lora_linear_set_plan(M, di, do, r, plan)
        assert L.lora_linear_get_plan(L.OP_BWD, M, di, do, r)["dx_overlap"] == 2
        dl = DeviceLayer(inp)
        dl.forward()
        dl.backward()
        dl.check()
        compare_all(dl.results(), oracle_ref(inp), spec.s)
    finally:
        L.lora_linear_set_plan(M, di, do, r, None)


@pytest.mark.parametrize("shape", [TAIL_WAVE[0], TAIL_WAVE[1], TAIL_WAVE[2]], ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_single_sm_main_gemm(shape, monkeypatch):
    """The single-SM main-GEMM kernel (chosen when CTA pairs are unavailable) on the
    same tail-wave shapes, including its 2-way and 4-way N splits."""
    monkeypatch.setenv("LORA_LINEAR_PAIR", "0")
    M, di, do, r = shape
    spec = inputs.LayerSpec("single", M, di, do, r, alpha=2.0 * r, seed=0x77 + M + di)
    inp, dl = _run_full(spec)
    compare_all(dl.results(), oracle_ref(inp), spec.s)


@pytest.mark.parametrize("shape", [(520, 640, 768, 16), (1280, 4096, 4096, 8)], ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_without_programmatic_launch(shape, monkeypatch):
    """Every launch without programmatic dependent launch.  The second shape has a
    partial last wave: dA + dB then run after the dX GEMM, whose tail tiles are cut
    along N (2D weight copies beside the 3D ones of whole tiles)."""
    monkeypatch.setenv("LORA_LINEAR_PDL", "0")
    M, di, do, r = shape
    spec = inputs.LayerSpec("nopdl", M, di, do, r, alpha=2.0 * r, seed=0x99 + M)
    inp, dl = _run_full(spec)
    compare_all(dl.results(), oracle_ref(inp), spec.s)


# 4-bit frozen weight: codes dequantised in shared memory inside both main GEMMs.
Q4_SHAPES = [
    (200, 320, 200, 16),     # ragged M and d_out (out-of-range rows and K rows of the codes)
    (520, 512, 768, 24),     # rank tail r % 16 != 0
    (129, 1024, 1536, 8),
    # more 256 x 256 tiles than CTA pairs, so CTAs take several work items; K blocks per
    # item (11 and 17, incl. the rank-r block) are not a multiple of the stage count, so
    # the rank-r block falls on a different stage in each item
    (1100, 640, 4000, 16),   # forward: 5 x 16 tiles
    (1100, 4096, 1000, 16),  # dX: 5 x 16 tiles, K = d_out ragged
]


@pytest.mark.parametrize("shape", Q4_SHAPES, ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_q4_full(shape):
    M, di, do, r = shape
    spec = inputs.LayerSpec("q4", M, di, do, r, alpha=2.0 * r, q4=True, seed=0x44 + M)
    inp, dl = _run_full(spec)
    compare_all(dl.results(), oracle_ref(inp), spec.s)


def test_q4_lora_dominant():
    """Large B so the rank-r tail (bf16, not dequantised) dominates: the tail blocks pass
    through the dequant stage untouched."""
    spec = inputs.LayerSpec("q4dom", 264, 384, 320, 16, alpha=32.0, q4=True, seed=0x45)
    inp = inputs.make_inputs(spec)
    inp.B = inputs.to_bf16_bits(inputs.bf16_bits_to_f32(inp.B).astype(np.float64) * 50.0)
    dl = DeviceLayer(inp)
    dl.forward()
    dl.backward()
    dl.check()
    compare_all(dl.results(), oracle_ref(inp), spec.s)


# ------------------------------------------------------------------ full sizes
FULL = [(1, None, 0), (2, None, 0), (2, None, 1), (2, None, 2), (2, None, 3), (3, 8, 0), (3, 16, 0), (3, 64, 0),
        (3, 128, 0), (4, None, 0)]


@pytest.mark.parametrize("cfg", FULL, ids=lambda c: f"cfg{c[0]}_r{c[1]}_layer{c[2]}")
def test_full_size_every_element(cfg):
    """The full-size workloads in the launch configuration the benchmark times: every
    element of h, dX, s.xa, dA and dB against the oracle's whole tensors, plus every
    row and column projection of h and dX as a second, independent check."""
    idx, r, layer = cfg
    spec = inputs.workload(idx, r=r).layers[layer]
    inp = inputs.make_inputs(spec)
    dl = DeviceLayer(inp)
    dl.forward()
    dl.backward()
    dl.check()
    res = compare_every_element(dl, inp)
    rows = sample_rows(spec.M, seed=idx * 10 + layer)
    ref = oracle_ref(inp, rows=rows)
    worst_proj = check_projections(dl, inp, ref, seed=idx * 10 + layer)
    print(f"{spec.name}: {res['elements']} elements compared, oracle {res['oracle_s']:.1f} s; worst error / bound "
          + ", ".join(f"{k} {v:.3f}" for k, v in res["worst"].items())
          + f"; projection residual / allowance {worst_proj:.3f}")


def test_data_parallel_shards_sum_to_full_batch():
    """Data parallel over tokens on one GPU: the layer run on two token shards, each
    backward writing into its own packed [dA | dB] buffer, sums (what the all-reduce
    does across ranks) to the whole batch's dA and dB; every shard's buffer is bitwise
    what the backward writes into separately allocated dA and dB."""
    from rank_linear_lora_b200.dp import PackedGrads, token_shard
    spec = inputs.LayerSpec("dp", 645, 512, 320, 16, alpha=32.0, seed=0xDB)
    inp = inputs.make_inputs(spec)
    total = PackedGrads(spec.r, spec.d_in, spec.d_out, device="cuda").zero_()
    for rank in range(2):
        start, count = token_shard(spec.M, 2, rank)
        sp = spec.with_(M=count)
        shard = inputs.LayerInputs(sp, inp.x[start:start + count], inp.A, inp.B, inp.dY[start:start + count], inp.W,
                                   None, None)
        dl = DeviceLayer(shard)
        dl.forward()
        dl.backward()
        packed = PackedGrads(spec.r, spec.d_in, spec.d_out, device="cuda")
        L.lora_linear_bwd(dl.dY, dl.x, dl.W, dl.A, dl.B, dl.xa, dl.dX, packed.dA, packed.dB, spec.alpha, dl.ws_b)
        dl.check()
        torch.cuda.synchronize()
        assert torch.equal(packed.dA, dl.dA) and torch.equal(packed.dB, dl.dB)
        total.buf += packed.buf
    ref = oracle_ref(inp)
    assert_close("dA", total.dA.cpu().numpy().astype(np.float64), ref["dA"], TOL_AB, RMS_AB)
    assert_close("dB", total.dB.cpu().numpy().astype(np.float64), ref["dB"], TOL_AB, RMS_AB)


def test_bounded_wait_timeout_is_reported_and_recoverable():
    """A device wait that can never complete (nothing arrives on its barrier) runs out,
    records LORA_ERR_TIMEOUT in the workspace error word, and returns: the check reports
    it once, clears it, and the same workspace and context then run a layer correctly."""
    spec = inputs.LayerSpec("after-timeout", 200, 256, 192, 8, alpha=16.0, seed=0x7E)
    inp = inputs.make_inputs(spec)
    dl = DeviceLayer(inp)
    L.lora_linear_selftest_timeout(dl.ws_f, 2000)  # 2 ms
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_check(dl.ws_f)
    assert e.value.status == 6  # LORA_ERR_TIMEOUT
    L.lora_linear_check(dl.ws_f)  # cleared
    dl.forward()
    dl.backward()
    dl.check()
    compare_all(dl.results(), oracle_ref(inp), spec.s)


# Rank-r side kernels (r <= 64): clusters of 1 to 8 CTAs reduce over distributed shared
# memory; these shapes reach several rounds per cluster (more 128-row output blocks
# than CTAs), s.g + dB rounds of 1 to 5 token blocks, clusters in which some CTAs hold
# no share of the reduction, and every rank width the MMA pads (r % 16 != 0, r = 64).
SIDE = [
    (40000, 64, 64, 8),       # s.xa: 313 token blocks on 148 CTAs (3 rounds); dA on an 8-CTA cluster
    (40000, 192, 1000, 16),   # s.g + dB: 5 token blocks per round, 2-CTA clusters
    (2048, 2048, 2048, 32),
    (1024, 512, 3000, 48),    # ragged d_out (partial last column block), r = 48
    (4500, 4160, 1800, 56),   # ragged M, d_in, d_out
    (384, 320, 8, 64),        # d_out = 8: one column block; d_in = 320: CTAs with no reduction share
]


@pytest.mark.parametrize("shape", SIDE, ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_side_kernels_every_element(shape):
    M, di, do, r = shape
    spec = inputs.LayerSpec("side", M, di, do, r, alpha=2.0 * r, seed=0x51DE + M + do)
    inp, dl = _run_full(spec)
    compare_every_element(dl, inp)


@pytest.mark.parametrize("shape", [(200, 328, 200, 8), (1024, 512, 3000, 48), (2048, 2048, 2048, 32)],
                         ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_split_k_side_products_for_narrow_ranks(shape, monkeypatch):
    """The split-K kernels (used above r = 64) on ranks the side kernels take by default."""
    monkeypatch.setenv("LORA_LINEAR_SIDE", "0")
    M, di, do, r = shape
    spec = inputs.LayerSpec("splitk", M, di, do, r, alpha=2.0 * r, seed=0x5B1 + M)
    inp, dl = _run_full(spec)
    compare_every_element(dl, inp)


# FP8 (E4M3) frozen weight with one bf16 scale per row, decoded in shared memory inside
# both main GEMMs: every element against the oracle's weight format 2.
FP8_SHAPES = [
    (200, 320, 200, 16),     # ragged M and d_out
    (520, 512, 768, 24),     # rank tail r % 16 != 0
    (129, 1040, 1536, 8),    # d_in % 64 != 0 (a partial last K block of codes)
    (1100, 640, 4000, 16),   # forward: 5 x 16 tiles, several work items per CTA pair
    (1100, 4096, 1000, 16),  # dX: 5 x 16 tiles, K = d_out ragged
]


@pytest.mark.parametrize("shape", FP8_SHAPES, ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_fp8_every_element(shape):
    M, di, do, r = shape
    spec = inputs.LayerSpec("fp8", M, di, do, r, alpha=2.0 * r, fp8=True, seed=0xF8 + M)
    inp, dl = _run_full(spec)
    compare_every_element(dl, inp)


def test_fp8_code_order_dominant_weight():
    """B = 0, so h and dX are the decoded weight's products alone: any swapped code
    pair, wrong scale row or chunk order shows far outside the bound."""
    spec = inputs.LayerSpec("fp8w", 256, 192, 320, 8, alpha=16.0, fp8=True, seed=0xF9)
    inp, dl = _run_full(spec, zero_B=True)
    compare_every_element(dl, inp)


@pytest.mark.parametrize("idx", [1, 4], ids=["attn_proj", "up_proj"])
def test_fp8_full_size_every_element(idx):
    """The attention projection and the up projection's sizes with the FP8 weight."""
    spec = inputs.workload(idx).layers[0].with_(q4=False, fp8=True)
    inp, dl = _run_full(spec)
    res = compare_every_element(dl, inp)
    print(f"{spec.name} fp8: {res['elements']} elements, oracle {res['oracle_s']:.1f} s; worst error / bound "
          + ", ".join(f"{k} {v:.3f}" for k, v in res["worst"].items()))


# 4-bit codebook weight (NF4 codebook): codes decoded through the 16-value table in
# shared memory inside both main GEMMs; every element against the oracle's format 3.
NF4_SHAPES = [
    (200, 320, 200, 16),     # ragged M and d_out
    (520, 512, 768, 24),     # rank tail r % 16 != 0
    (1100, 640, 4000, 16),   # forward: several work items per CTA pair
    (1100, 4096, 1000, 16),  # dX: K = d_out ragged
]


@pytest.mark.parametrize("shape", NF4_SHAPES, ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_nf4_every_element(shape):
    M, di, do, r = shape
    spec = inputs.LayerSpec("nf4", M, di, do, r, alpha=2.0 * r, nf4=True, seed=0x4F4 + M)
    inp, dl = _run_full(spec)
    compare_every_element(dl, inp)


def test_nf4_weight_dominated_every_code():
    """B = 0: h and dX are the decoded weight's products alone, and the weight uses all
    16 codes, so a wrong table entry, byte order or half-table choice shows."""
    spec = inputs.LayerSpec("nf4w", 256, 192, 320, 8, alpha=16.0, nf4=True, seed=0x4F5)
    inp, dl = _run_full(spec, zero_B=True)
    assert len(np.unique(inputs.unpack_q4_codes(inp.Wq))) == 16
    compare_every_element(dl, inp)


def test_nf4_full_size_every_element():
    """The up projection's size (M=4096, 8192 -> 28672, r=16) with the NF4 weight."""
    spec = inputs.workload(4).layers[0].with_(q4=False, nf4=True)
    inp, dl = _run_full(spec)
    res = compare_every_element(dl, inp)
    print(f"{spec.name} nf4: {res['elements']} elements, oracle {res['oracle_s']:.1f} s; worst error / bound "
          + ", ".join(f"{k} {v:.3f}" for k, v in res["worst"].items()))


@pytest.mark.parametrize("shape", [(1024, 512, 3000, 32), (520, 640, 768, 24), (2048, 2048, 2048, 32)],
                         ids=lambda s: "M%d_in%d_out%d_r%d" % s)
def test_one_pass_backward_at_ranks_above_the_default(shape):
    """s.g + dB in one pass over dY, and dA, at r = 24 and 32 (64-byte swizzled narrow
    operands, N = 32), which a plan selects (the library's own choice is split-K there)."""
    M, di, do, r = shape
    L.lora_linear_set_plan(M, di, do, r, dict(side_bwd=1))
    try:
        assert L.lora_linear_get_plan(L.OP_BWD, M, di, do, r)["side_bwd"] == 1
        spec = inputs.LayerSpec("onepass", M, di, do, r, alpha=2.0 * r, seed=0x1BA + M)
        inp, dl = _run_full(spec)
        compare_every_element(dl, inp)
    finally:
        L.lora_linear_set_plan(M, di, do, r, None)
