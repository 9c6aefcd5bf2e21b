"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test ties one or more of the oracle's six steps to a hand-worked value, a
closed form, an invariance of the layer, brute force in pure Python, finite
differences of the forward, or a library matmul on a case the definition reduces to.
A dropped term, a wrong sign, a transposed operand or a swapped gradient fails at
least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from rank_linear_lora_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(a):
    """Exact bf16 bit patterns of small dyadic values (asserts exact representability)."""
    a = np.asarray(a, dtype=np.float64)
    bits = inputs.to_bf16_bits(a)
    assert np.array_equal(inputs.bf16_bits_to_f32(bits).astype(np.float64), a), "not bf16-exact"
    return bits


def f64(bits):
    return inputs.bf16_bits_to_f32(bits).astype(np.float64)


def run_all(x, W, A, B, dY, alpha):
    r = A.shape[0]
    s = alpha / r
    h, xa = oracle.forward(x, A, B, s, W=W)
    bw = oracle.backward(dY, x, A, B, s, W=W)
    return dict(h=h, xa=xa, **{k: bw[k] for k in ("dX", "dA", "dB", "g")})


@pytest.mark.parametrize("name", ["rank1_hand.json", "rank2_hand.json"])
def test_hand_worked_cases(name):
    c = json.load(open(os.path.join(GOLDEN, name)))
    out = run_all(bf(c["x"]), bf(c["W"]), bf(c["A"]), bf(c["B"]), bf(c["dY"]), c["alpha"])
    for key in ("xa", "g", "h", "dX", "dA", "dB"):
        np.testing.assert_array_equal(out[key], np.array(c[key], dtype=np.float64), err_msg=key)
    assert float((f64(bf(c["dY"])) * out["h"]).sum()) == c["L"]


def _rand_bits(rng, shape, scale=1.0):
    return inputs.to_bf16_bits(rng.standard_normal(shape) * scale)


def _py_xwT(x, W):
    """Brute force x.W^T in pure Python, summing k in increasing order."""
    M, d_in = x.shape
    d_out = W.shape[0]
    out = np.zeros((M, d_out))
    for m in range(M):
        for n in range(d_out):
            acc = 0.0
            for k in range(d_in):
                acc += float(x[m, k]) * float(W[n, k])
            out[m, n] = acc
    return out


def _py_dyW(dY, W):
    """Brute force dY.W in pure Python, summing n in increasing order."""
    M, d_out = dY.shape
    d_in = W.shape[1]
    out = np.zeros((M, d_in))
    for m in range(M):
        for k in range(d_in):
            acc = 0.0
            for n in range(d_out):
                acc += float(dY[m, n]) * float(W[n, k])
            out[m, k] = acc
    return out


def test_zero_B_is_the_frozen_linear():
    """Delta W = 0: h = x.W^T and dX = dY.W exactly, dA = 0 exactly, dB stays nonzero."""
    rng = np.random.default_rng(1)
    M, d_in, d_out, r = 5, 7, 6, 3
    x, W, A, dY = (_rand_bits(rng, s) for s in [(M, d_in), (d_out, d_in), (r, d_in), (M, d_out)])
    B = np.zeros((d_out, r), dtype=np.uint16)
    out = run_all(x, W, A, B, dY, alpha=6.0)
    np.testing.assert_array_equal(out["h"], _py_xwT(f64(x), f64(W)))
    np.testing.assert_array_equal(out["dX"], _py_dyW(f64(dY), f64(W)))
    assert np.all(out["g"] == 0) and np.all(out["dA"] == 0)
    assert np.abs(out["dB"]).max() > 0


def test_zero_A_is_the_frozen_linear():
    """A = 0: xa = 0, so h = x.W^T, dB = 0 exactly and dX = dY.W exactly; dA stays nonzero."""
    rng = np.random.default_rng(2)
    M, d_in, d_out, r = 4, 6, 5, 2
    x, W, B, dY = (_rand_bits(rng, s) for s in [(M, d_in), (d_out, d_in), (d_out, r), (M, d_out)])
    A = np.zeros((r, d_in), dtype=np.uint16)
    out = run_all(x, W, A, B, dY, alpha=4.0)
    assert np.all(out["xa"] == 0) and np.all(out["dB"] == 0)
    np.testing.assert_array_equal(out["h"], _py_xwT(f64(x), f64(W)))
    np.testing.assert_array_equal(out["dX"], _py_dyW(f64(dY), f64(W)))
    assert np.abs(out["dA"]).max() > 0


@pytest.mark.parametrize("shape", [(64, 256, 256, 8), (37, 48, 80, 16), (9, 120, 24, 1)])
def test_merged_weight_identity(shape):
    """x.(W + s.B.A)^T = h and dY.(W + s.B.A) = dX with the d_out x d_in update formed
    explicitly: the merged weight of deployment, and (B.A)^T.dY = A^T.(B^T.dY), the
    reassociation the backward relies on."""
    M, d_in, d_out, r = shape
    rng = np.random.default_rng(3)
    x, W, A, B, dY = (_rand_bits(rng, s, sc) for s, sc in
                      [((M, d_in), 1), ((d_out, d_in), d_in ** -0.5), ((r, d_in), d_in ** -0.5),
                       ((d_out, r), 0.5), ((M, d_out), 1)])
    alpha = 2.0 * r
    s = alpha / r
    out = run_all(x, W, A, B, dY, alpha)
    merged = f64(W) + s * (f64(B) @ f64(A))
    h_ref = f64(x) @ merged.T
    dx_ref = f64(dY) @ merged
    np.testing.assert_allclose(out["h"], h_ref, rtol=0, atol=1e-12 * np.abs(h_ref).max())
    np.testing.assert_allclose(out["dX"], dx_ref, rtol=0, atol=1e-12 * np.abs(dx_ref).max())


@pytest.mark.parametrize("shape", [(64, 256, 256, 8), (23, 72, 40, 16)])
def test_matches_library_matmul(shape):
    """Every output against numpy fp64 matmuls of the same definition."""
    M, d_in, d_out, r = shape
    rng = np.random.default_rng(4)
    x, W, A, B, dY = (_rand_bits(rng, s, sc) for s, sc in
                      [((M, d_in), 1), ((d_out, d_in), d_in ** -0.5), ((r, d_in), d_in ** -0.5),
                       ((d_out, r), 0.02), ((M, d_out), 1)])
    alpha = 16.0
    s = alpha / r
    out = run_all(x, W, A, B, dY, alpha)
    X, Wd, Ad, Bd, dYd = map(f64, (x, W, A, B, dY))
    ref = {
        "xa": X @ Ad.T,
        "h": X @ Wd.T + s * (X @ Ad.T) @ Bd.T,
        "g": dYd @ Bd,
        "dX": dYd @ Wd + s * (dYd @ Bd) @ Ad,
        "dB": s * dYd.T @ (X @ Ad.T),
        "dA": s * (dYd @ Bd).T @ X,
    }
    for key, want in ref.items():
        np.testing.assert_allclose(out[key], want, rtol=0, atol=1e-12 * np.abs(want).max(), err_msg=key)


def _dyadic(rng, shape):
    """Multiples of 1/8 in [-2, 2]: with eps = 1/16 every perturbed value stays bf16-exact."""
    return rng.integers(-16, 17, size=shape).astype(np.float64) / 8.0


@pytest.mark.parametrize("r", [1, 2])
def test_central_differences(r):
    """dX, dA, dB are the derivatives of L = sum(dY * h).  L is affine in every single
    entry of x, A and B, so the central difference is exact up to rounding."""
    M, d_in, d_out = 3, 5, 4
    rng = np.random.default_rng(10 + r)
    vals = {k: _dyadic(rng, s) for k, s in
            [("x", (M, d_in)), ("W", (d_out, d_in)), ("A", (r, d_in)), ("B", (d_out, r)), ("dY", (M, d_out))]}
    alpha = 2.0 * r
    s = alpha / r
    eps = 1.0 / 16.0

    def loss(v):
        h, _ = oracle.forward(bf(v["x"]), bf(v["A"]), bf(v["B"]), s, W=bf(v["W"]))
        return float((v["dY"] * h).sum())

    grads = oracle.backward(bf(vals["dY"]), bf(vals["x"]), bf(vals["A"]), bf(vals["B"]), s, W=bf(vals["W"]))
    for name, gname in (("x", "dX"), ("A", "dA"), ("B", "dB")):
        fd = np.zeros_like(vals[name])
        for idx in np.ndindex(vals[name].shape):
            vp = {k: v.copy() for k, v in vals.items()}
            vm = {k: v.copy() for k, v in vals.items()}
            vp[name][idx] += eps
            vm[name][idx] -= eps
            fd[idx] = (loss(vp) - loss(vm)) / (2 * eps)
        scale = max(1.0, np.abs(fd).max())
        np.testing.assert_allclose(grads[gname], fd, rtol=0, atol=1e-10 * scale, err_msg=gname)


def test_rescaling_and_alpha():
    """(A*c, B/c) leaves h and dX unchanged (c a power of two: exact); doubling alpha
    doubles the low-rank term of h."""
    rng = np.random.default_rng(5)
    M, d_in, d_out, r = 6, 16, 12, 4
    x, W, A, B, dY = (_rand_bits(rng, s, 0.5) for s in
                      [(M, d_in), (d_out, d_in), (r, d_in), (d_out, r), (M, d_out)])
    base = run_all(x, W, A, B, dY, 8.0)
    resc = run_all(x, W, bf(f64(A) * 2.0), bf(f64(B) / 2.0), dY, 8.0)
    np.testing.assert_array_equal(base["h"], resc["h"])
    np.testing.assert_array_equal(base["dX"], resc["dX"])
    h0 = run_all(x, W, A, np.zeros_like(B), dY, 8.0)["h"]
    h2 = run_all(x, W, A, B, dY, 16.0)["h"]
    np.testing.assert_allclose(h2 - h0, 2.0 * (base["h"] - h0), rtol=0, atol=1e-12 * np.abs(h2).max())


def test_q4_code_pins():
    """The 4-bit code of a block [a, -a, 0, a/2, ...] is [15, 1, 8, 12, ...] and
    decodes to [a, -a, 0, 4a/7, ...]; low nibble = even index; a zero block codes 8."""
    a = 0.75  # bf16-exact, so the stored scale is exactly a
    w = np.zeros((2, 128), dtype=np.float32)
    w[0, :4] = [a, -a, 0.0, a / 2]
    w[0, 4:64] = np.linspace(-a / 2, a / 2, 60, dtype=np.float32)
    q, sc = inputs.quantise_q4(w)
    codes = inputs.unpack_q4_codes(q)
    assert list(codes[0, :4]) == [15, 1, 8, 12]
    assert q[0, 0] == (15 | (1 << 4)) and q[0, 1] == (8 | (12 << 4))
    assert np.all(codes[1] == 8) and np.all(codes[0, 64:] == 8)
    assert inputs.bf16_bits_to_f32(sc)[0, 0] == np.float32(a)
    assert np.all(sc[1] == 0)
    wd = oracle.weight(2, 128, Wq=q, Wscale=sc)
    np.testing.assert_array_equal(wd[0, :4], [a, -a, 0.0, 4 * a / 7])
    assert np.all(wd[1] == 0) and np.all(wd[0, 64:] == 0)


def test_q4_forward_reads_dequantised_columns():
    """With B = 0 and x = e_k, row h[k] of the q4 oracle is column k of the decoded weight
    (q - 8) * scale / 7 computed here from the codes and scales by hand."""
    d_in, d_out, r = 128, 3, 2
    rng = np.random.default_rng(6)
    q = rng.integers(0, 256, size=(d_out, d_in // 2), dtype=np.uint8)
    sc = inputs.to_bf16_bits(rng.uniform(0.1, 1.0, size=(d_out, d_in // 64)))
    x = inputs.to_bf16_bits(np.eye(d_in))
    A = np.zeros((r, d_in), dtype=np.uint16)
    B = np.zeros((d_out, r), dtype=np.uint16)
    h, _ = oracle.forward(x, A, B, 1.0, Wq=q, Wscale=sc)
    codes = inputs.unpack_q4_codes(q).astype(np.float64)
    scale = np.repeat(inputs.bf16_bits_to_f32(sc).astype(np.float64), 64, axis=1)
    np.testing.assert_array_equal(h.T, (codes - 8.0) * scale / 7.0)


def _e4m3_library_values() -> np.ndarray:
    """All 256 FP8 E4M3 codes decoded by torch's float8_e4m3fn (a library routine)."""
    import torch
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_fp8_decode_matches_library_for_every_code():
    """The oracle's E4M3 decode of all 256 codes (scale 1) equals the library's, NaN
    codes and the sign of zero included."""
    codes = np.arange(256, dtype=np.uint8).reshape(1, 256)
    got = oracle.weight(1, 256, W8=codes, W8scale=bf([1.0]))[0]
    ref = _e4m3_library_values()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    np.testing.assert_array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def test_fp8_hand_values():
    """Codes decoded by hand from the E4M3 layout (sign | 4-bit exponent, bias 7 |
    3-bit mantissa): 0x01 is the smallest subnormal 2^-9, 0x08 the smallest normal
    2^-6, 0x38 = 0.0111.000 is 1, 0x3C = 1 + 4/8, 0x7E = 0.1111.110 is 1.75 * 2^8 = 448
    (0x7F is NaN, not a number above it); the row scale multiplies every code."""
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0x38: 1.0,
             0x3C: 1.5, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0}
    codes = np.array([list(table)], dtype=np.uint8)
    got = oracle.weight(1, len(table), W8=codes, W8scale=bf([1.0]))[0]
    np.testing.assert_array_equal(got, list(table.values()))
    got = oracle.weight(2, len(table), W8=np.repeat(codes, 2, axis=0), W8scale=bf([0.375, -2.0]))
    np.testing.assert_array_equal(got, np.outer([0.375, -2.0], list(table.values())))
    assert np.isnan(oracle.weight(1, 2, W8=np.array([[0x7F, 0xFF]], np.uint8), W8scale=bf([1.0]))).all()


def test_fp8_quantiser_pins():
    """Row absmax 28 gives the bf16-exact scale 28/448 = 1/16, so w/scale is exact:
    [28, -28, 14, 0] code to [0x7E, 0xFE, 0x76, 0x00] and decode back exactly; the
    midpoints 1.0625/16 and 1.1875/16 round to the even mantissa (1/16, 1.25/16); a zero
    row gets scale 0.  A row whose rounded scale sits below absmax/448 saturates at 448."""
    w = np.zeros((3, 8), dtype=np.float32)
    w[0, :6] = [28.0, -28.0, 14.0, 0.0, 1.0625 / 16, 1.1875 / 16]
    w[2, :2] = [3.0, -3.0]  # bf16(3/448) < 3/448: w / scale > 448, clamped
    q, sc = inputs.quantise_fp8(w)
    assert list(q[0, :6]) == [0x7E, 0xFE, 0x76, 0x00, 0x38, 0x3A]
    assert inputs.bf16_bits_to_f32(sc)[0] == np.float32(1 / 16)
    assert sc[1] == 0 and not q[1].any()
    assert list(q[2, :2]) == [0x7E, 0xFE]
    wd = oracle.weight(3, 8, W8=q, W8scale=sc)
    np.testing.assert_array_equal(wd[0, :6], [28.0, -28.0, 14.0, 0.0, 1 / 16, 1.25 / 16])
    assert abs(wd[2, 0] - 3.0) <= 3.0 * 2.0 ** -8  # within the bf16 rounding of the scale


def test_fp8_forward_reads_decoded_columns():
    """With B = 0 and x = e_k, row h[k] of the fp8 oracle is column k of the decoded
    weight, decoded here through the library table times each row's scale."""
    d_in, d_out, r = 64, 5, 2
    rng = np.random.default_rng(16)
    q = rng.integers(0, 256, size=(d_out, d_in), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x3F  # no NaN codes
    sc = inputs.to_bf16_bits(rng.uniform(0.01, 1.0, size=d_out))
    x = inputs.to_bf16_bits(np.eye(d_in))
    A = np.zeros((r, d_in), dtype=np.uint16)
    B = np.zeros((d_out, r), dtype=np.uint16)
    h, _ = oracle.forward(x, A, B, 1.0, W8=q, W8scale=sc)
    want = _e4m3_library_values()[q] * inputs.bf16_bits_to_f32(sc).astype(np.float64)[:, None]
    np.testing.assert_array_equal(h.T, want)


def test_fp8_matches_library_matmul():
    """Every output with an FP8 weight against numpy fp64 matmuls of the same definition,
    the weight decoded through the library table."""
    M, d_in, d_out, r = 19, 96, 40, 8
    rng = np.random.default_rng(17)
    w32 = (rng.standard_normal((d_out, d_in)) / np.sqrt(d_in)).astype(np.float32)
    q, sc = inputs.quantise_fp8(w32)
    x, A, B, dY = (_rand_bits(rng, s_, c) for s_, c in
                   [((M, d_in), 1), ((r, d_in), d_in ** -0.5), ((d_out, r), 0.02), ((M, d_out), 1)])
    s = 2.0
    h, xa = oracle.forward(x, A, B, s, W8=q, W8scale=sc)
    bw = oracle.backward(dY, x, A, B, s, W8=q, W8scale=sc)
    Wd = _e4m3_library_values()[q] * inputs.bf16_bits_to_f32(sc).astype(np.float64)[:, None]
    X, Ad, Bd, dYd = map(f64, (x, A, B, dY))
    ref = {"h": X @ Wd.T + s * (X @ Ad.T) @ Bd.T, "dX": dYd @ Wd + s * (dYd @ Bd) @ Ad,
           "dA": s * (dYd @ Bd).T @ X, "dB": s * dYd.T @ (X @ Ad.T)}
    got = {"h": h, "dX": bw["dX"], "dA": bw["dA"], "dB": bw["dB"]}
    for key, want in ref.items():
        np.testing.assert_allclose(got[key], want, rtol=0, atol=1e-12 * np.abs(want).max(), err_msg=key)
    # the quantised weight is close to the draws it codes (3 mantissa bits: 2^-4 relative)
    np.testing.assert_allclose(Wd, w32, rtol=0, atol=2.0 ** -4 * np.abs(w32).max())


def test_row_selection_matches_full():
    """The sampled-row mode used at full sizes returns exactly the full rows."""
    rng = np.random.default_rng(7)
    M, d_in, d_out, r = 20, 24, 16, 8
    x, W, A, B, dY = (_rand_bits(rng, s) for s in [(M, d_in), (d_out, d_in), (r, d_in), (d_out, r), (M, d_out)])
    rows = np.array([19, 0, 7])
    full = run_all(x, W, A, B, dY, 16.0)
    hs, _ = oracle.forward(x, A, B, 2.0, W=W, rows=rows)
    dxs = oracle.backward(dY, x, A, B, 2.0, W=W, rows=rows)["dX"]
    np.testing.assert_array_equal(hs, full["h"][rows])
    np.testing.assert_array_equal(dxs, full["dX"][rows])


@pytest.mark.parametrize("q4", [False, True], ids=["bf16", "q4"])
def test_projections_match_full_outputs(q4):
    """The row/column projections used to cover every element at full sizes equal the
    projections of the oracle's full h and dX (associativity, fp64 rounding only), also
    when the weight is taken in several row blocks."""
    spec = inputs.LayerSpec("proj", 37, 128, 80, 8, alpha=16.0, q4=q4, seed=0x9E)
    inp = inputs.make_inputs(spec)
    wkw = dict(Wq=inp.Wq, Wscale=inp.Wscale) if q4 else dict(W=inp.W)
    h_full, xa_ = oracle.forward(inp.x, inp.A, inp.B, spec.s, **wkw)
    bwd = oracle.backward(inp.dY, inp.x, inp.A, inp.B, spec.s, **wkw)
    rng = np.random.default_rng(3)
    v_h, u = rng.choice([-1.0, 1.0], 80), rng.choice([-1.0, 1.0], 37)
    v_x = rng.choice([-1.0, 1.0], 128)
    for blk in (2048, 24):
        row, col = oracle.h_projections(inp.x, inp.A, inp.B, spec.s, v_h, u, block_rows=blk, **wkw)
        np.testing.assert_allclose(row, h_full @ v_h, rtol=0, atol=1e-12 * np.abs(h_full).sum(1).max())
        np.testing.assert_allclose(col, u @ h_full, rtol=0, atol=1e-12 * np.abs(h_full).sum(0).max())
        row, col = oracle.dx_projections(inp.dY, inp.A, inp.B, spec.s, v_x, u, block_rows=blk, **wkw)
        np.testing.assert_allclose(row, bwd["dX"] @ v_x, rtol=0, atol=1e-12 * np.abs(bwd["dX"]).sum(1).max())
        np.testing.assert_allclose(col, u @ bwd["dX"], rtol=0, atol=1e-12 * np.abs(bwd["dX"]).sum(0).max())


def test_matches_library_matmul_at_attention_projection_size():
    """The oracle at the attention-projection size (M=4096, 4096x4096, r=8, its seeded
    inputs) against numpy fp64: every element of xa, g, dA, dB, and 16 token rows of h
    and dX (the oracle's row mode, which the full-size GPU tests use)."""
    spec = inputs.workload(1).layers[0]
    inp = inputs.make_inputs(spec)
    s = spec.s
    rows = np.array([0, 1, 127, 128, 255, 1000, 2047, 2048, 2049, 3000, 3967, 3968, 4000, 4094, 4095, 511])
    h_rows, xa_ = oracle.forward(inp.x, inp.A, inp.B, s, W=inp.W, rows=rows)
    bwd = oracle.backward(inp.dY, inp.x, inp.A, inp.B, s, W=inp.W, rows=rows, xa_=xa_)
    X, Wd, Ad, Bd, dYd = map(f64, (inp.x, inp.W, inp.A, inp.B, inp.dY))
    xa_ref = X @ Ad.T
    g_ref = dYd @ Bd
    ref = {
        "xa": (xa_, xa_ref),
        "g": (bwd["g"], g_ref),
        "dB": (bwd["dB"], s * dYd.T @ xa_ref),
        "dA": (bwd["dA"], s * g_ref.T @ X),
        "h": (h_rows, X[rows] @ Wd.T + s * xa_ref[rows] @ Bd.T),
        "dX": (bwd["dX"], dYd[rows] @ Wd + s * g_ref[rows] @ Ad),
    }
    for key, (got, want) in ref.items():
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12 * np.abs(want).max(), err_msg=key)


@pytest.mark.parametrize("q4", [False, True], ids=["bf16", "q4"])
def test_merged_weight_reproduces_the_forward(q4):
    """The merged weight the deploy-time merge is checked against gives the oracle's own
    forward: x . merged^T = h (steps 1-2), for the bf16 and the 4-bit weight."""
    spec = inputs.LayerSpec("merge", 29, 128, 72, 16, alpha=24.0, q4=q4, seed=0x3E)
    inp = inputs.make_inputs(spec)
    wkw = dict(Wq=inp.Wq, Wscale=inp.Wscale) if q4 else dict(W=inp.W)
    merged = oracle.merged_weight(inp.A, inp.B, spec.s, **wkw)
    h, _ = oracle.forward(inp.x, inp.A, inp.B, spec.s, **wkw)
    np.testing.assert_allclose(f64(inp.x) @ merged.T, h, rtol=0, atol=1e-12 * np.abs(h).max())


@pytest.mark.parametrize("fmt", ["bf16", "q4", "fp8"])
def test_dense_steps_match_the_loops(fmt):
    """The dense steps 2 and 4 (numpy's fp64 product as the summation primitive, used for
    whole tensors at full size) equal oracle.c's loops up to fp64 summation order, for
    every weight format, whole and a block of rows at a time."""
    spec = inputs.LayerSpec("dense", 70, 192, 136, 16, alpha=32.0, q4=(fmt == "q4"), seed=0xD5)
    inp = inputs.make_inputs(spec)
    if fmt == "q4":
        wkw = dict(Wq=inp.Wq, Wscale=inp.Wscale)
    elif fmt == "fp8":
        W8, W8scale = inputs.quantise_fp8(inputs.bf16_bits_to_f32(inp.W))
        wkw = dict(W8=W8, W8scale=W8scale)
    else:
        wkw = dict(W=inp.W)
    h, xa_ = oracle.forward(inp.x, inp.A, inp.B, spec.s, **wkw)
    bwd = oracle.backward(inp.dY, inp.x, inp.A, inp.B, spec.s, xa_=xa_, **wkw)
    Wf = oracle.weight(spec.d_out, spec.d_in, **wkw)
    hd = oracle.h_dense(inp.x, inp.B, xa_, spec.s, Wf)
    dd = oracle.dx_dense(inp.dY, inp.A, bwd["g"], spec.s, Wf)
    np.testing.assert_allclose(hd, h, rtol=0, atol=1e-13 * np.abs(h).max())
    np.testing.assert_allclose(dd, bwd["dX"], rtol=0, atol=1e-13 * np.abs(bwd["dX"]).max())
    # a block of rows (BLAS may take another kernel, e.g. for one row: same sums, other order)
    for r0, r1 in ((0, 32), (32, 33), (33, 70)):
        np.testing.assert_allclose(oracle.h_dense(inp.x[r0:r1], inp.B, xa_[r0:r1], spec.s, Wf), h[r0:r1],
                                   rtol=0, atol=1e-13 * np.abs(h).max())
        np.testing.assert_allclose(oracle.dx_dense(inp.dY[r0:r1], inp.A, bwd["g"][r0:r1], spec.s, Wf),
                                   bwd["dX"][r0:r1], rtol=0, atol=1e-13 * np.abs(bwd["dX"]).max())


def test_codebook_format_with_the_linear_codebook_is_the_4bit_format():
    """Weight format 3 (codebook[q] * scale) with codebook (i - 8) / 7 decodes exactly as
    format 1 ((q - 8) * scale / 7) through other code: every output agrees."""
    spec = inputs.LayerSpec("cb", 40, 192, 72, 16, alpha=32.0, q4=True, seed=0xCB)
    inp = inputs.make_inputs(spec)
    lin = (np.arange(16) - 8) / 7.0
    w1 = oracle.weight(72, 192, Wq=inp.Wq, Wscale=inp.Wscale)
    w3 = oracle.weight(72, 192, Wq=inp.Wq, Wscale=inp.Wscale, codebook=lin)
    np.testing.assert_allclose(w3, w1, rtol=0, atol=1e-15 * np.abs(w1).max())
    h1, xa1 = oracle.forward(inp.x, inp.A, inp.B, spec.s, Wq=inp.Wq, Wscale=inp.Wscale)
    h3, _ = oracle.forward(inp.x, inp.A, inp.B, spec.s, Wq=inp.Wq, Wscale=inp.Wscale, codebook=lin)
    np.testing.assert_allclose(h3, h1, rtol=0, atol=1e-13 * np.abs(h1).max())
    b1 = oracle.backward(inp.dY, inp.x, inp.A, inp.B, spec.s, Wq=inp.Wq, Wscale=inp.Wscale, xa_=xa1)
    b3 = oracle.backward(inp.dY, inp.x, inp.A, inp.B, spec.s, Wq=inp.Wq, Wscale=inp.Wscale, codebook=lin, xa_=xa1)
    np.testing.assert_allclose(b3["dX"], b1["dX"], rtol=0, atol=1e-13 * np.abs(b1["dX"]).max())


def test_nf4_forward_reads_decoded_columns():
    """With x = e_k the forward returns column k of the decoded weight: codebook[q] *
    scale of the code's 64-block, for every code value the NF4 weight uses."""
    spec = inputs.LayerSpec("nf4", 192, 192, 40, 8, alpha=16.0, nf4=True, seed=0x4F)
    inp = inputs.make_inputs(spec)
    x = np.zeros((192, 192), dtype=np.uint16)
    x[np.arange(192), np.arange(192)] = 0x3F80  # bf16 1.0
    zeroB = np.zeros_like(inp.B)
    h, _ = oracle.forward(x, inp.A, zeroB, spec.s, Wq=inp.Wq, Wscale=inp.Wscale, codebook=inp.codebook)
    q = inputs.unpack_q4_codes(inp.Wq)
    sc = inputs.bf16_bits_to_f32(inp.Wscale).astype(np.float64)
    want = inp.codebook[q] * np.repeat(sc, 64, axis=1)
    np.testing.assert_array_equal(h, want.T)
    assert len(np.unique(q)) == 16
