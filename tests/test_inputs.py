"""The seeded input generator: published test values, determinism, distributions."""
import math

import numpy as np
import pytest

from rank_linear_lora_b200 import inputs


def test_splitmix64_published_sequence():
    """splitmix64 from state 0: the first three outputs of the published generator."""
    words = inputs._words(np.uint64(0), np.arange(3, dtype=np.uint64))
    assert [int(w) for w in words] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_round_to_nearest_even():
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 3.0e-3, 1.0 + 2.0 ** -8 + 2.0 ** -20],
                    dtype=np.float32)
    bits = inputs.f32_to_bf16_bits(vals)
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 is a tie -> even (1+2^-6); just above a tie rounds up
    assert list(bits[:4]) == [0x3F80, 0x3F80, 0x3F82, 0xC020]
    assert bits[5] == 0x3F81
    back = inputs.bf16_bits_to_f32(bits[4:5])[0]
    assert abs(back - 3.0e-3) <= 3.0e-3 * 2.0 ** -8


def test_streams_are_deterministic_and_shape_independent():
    a = inputs.LayerSpec("t", 16, 64, 32, 8, 16.0, seed=123)
    b = a.with_(d_out=48)
    ia, ib = inputs.make_inputs(a), inputs.make_inputs(b)
    np.testing.assert_array_equal(ia.x, ib.x)
    np.testing.assert_array_equal(ia.A, ib.A)
    ia2 = inputs.make_inputs(a)
    for k in ("x", "W", "A", "B", "dY"):
        np.testing.assert_array_equal(getattr(ia, k), getattr(ia2, k))
    assert not np.array_equal(ia.x[:, :32], ia.dY)


def test_chunked_draws_match_single_pass():
    n = inputs._CHUNK + 12345
    big = inputs.draw("normal", 7, 1, n, 1.0)
    head = inputs._draw_chunk("normal", inputs.stream_key(7, 1), 0, 1000, 1.0)
    tail = inputs._draw_chunk("normal", inputs.stream_key(7, 1), n - 1000, n, 1.0)
    np.testing.assert_array_equal(big[:1000], head)
    np.testing.assert_array_equal(big[-1000:], tail)


def test_distributions():
    n = 1 << 20
    z = inputs.draw("normal", 99, 1, n, 0.02)
    assert abs(z.mean()) < 4 * 0.02 / math.sqrt(n) * 1.5
    assert abs(z.std() / 0.02 - 1.0) < 5e-3
    u = inputs.draw("uniform", 99, 2, n, 0.25)
    assert u.min() > -0.25 and u.max() < 0.25
    assert abs(u.std() - 0.25 / math.sqrt(3)) < 1e-3


def test_e4m3_encoder_matches_library_cast():
    """The FP8 E4M3 encoder rounds like torch's float32 -> float8_e4m3fn cast (nearest,
    ties to even, subnormals included) over every binade and both signs."""
    import torch
    rng = np.random.default_rng(11)
    mag = rng.choice([1e-4, 3e-3, 0.05, 1.0, 20.0, 200.0], size=100_000)
    v = np.clip(rng.standard_normal(100_000) * mag, -448, 448).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(inputs.e4m3_encode(v), ref)


def test_e4m3_encoder_exact_values_and_ties():
    """Every representable value encodes to its own code; midpoints go to the even
    mantissa (1.0625 -> 1.0, 1.1875 -> 1.25); the top value is 448."""
    import torch
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(inputs.e4m3_encode(vals), codes)
    assert list(inputs.e4m3_encode(np.array([1.0625, 1.1875, -1.0625, 448.0]))) == [0x38, 0x3A, 0xB8, 0x7E]
    with pytest.raises(ValueError):
        inputs.e4m3_encode(np.array([449.0]))


def test_nf4_codebook_construction():
    """16 increasing values with an exact zero at code 7 and +-1 at the ends; each side
    holds standard-normal quantiles at evenly spaced probabilities (the NormalFloat
    construction), and the published values of the format come out."""
    from scipy.special import ndtr
    cb = inputs.nf4_codebook()
    assert cb.shape == (16,) and np.all(np.diff(cb) > 0)
    assert cb[0] == -1.0 and cb[7] == 0.0 and cb[15] == 1.0
    delta = 0.5 * (1 / 30 + 1 / 32)
    from scipy.special import ndtri
    top = ndtri(1 - delta)
    p_pos = ndtr(cb[8:] * top)          # 8 probabilities, 1/2 excluded, evenly spaced up to 1 - delta
    p_neg = ndtr(-cb[:7] * top)         # 7 probabilities on the negative side
    np.testing.assert_allclose(np.diff(p_pos), (0.5 - delta) / 8, rtol=1e-12)
    np.testing.assert_allclose(np.diff(p_neg[::-1]), (0.5 - delta) / 7, rtol=1e-12)
    # values of the NormalFloat-4 table as printed with 7 digits
    np.testing.assert_allclose(cb[[1, 6, 8, 14]], [-0.6961928, -0.0910500, 0.0795803, 0.7229568], atol=2e-7)


def test_codebook_quantiser_picks_the_nearest_value():
    cb = inputs.nf4_codebook()
    rng = np.random.default_rng(5)
    w = rng.standard_normal((6, 192)).astype(np.float32)
    w[0, :4] = [np.abs(w[0, :64]).max(), -np.abs(w[0, :64]).max(), 0.0, 0.0]
    w[1, 64:128] = 0.0                   # a block of zeros: scale 0, code of 0
    packed, scales = inputs.quantise_codebook(w, cb)
    q = inputs.unpack_q4_codes(packed)
    sc = inputs.bf16_bits_to_f32(scales).astype(np.float64)
    assert sc[1, 1] == 0.0 and np.all(q[1, 64:128] == 7)
    for n in range(6):
        for k in range(192):
            s = sc[n, k // 64]
            if s == 0:
                continue
            t = float(w[n, k]) / s
            best = int(np.argmin(np.abs(cb - t)))
            assert q[n, k] == best or abs(abs(cb[q[n, k]] - t) - abs(cb[best] - t)) < 1e-15, (n, k)
    amax = np.abs(w[0, :64]).max()
    assert q[0, 2] == 7 and q[0, 3] == 7
    if inputs.bf16_bits_to_f32(scales)[0, 0] <= amax:  # rounding of the scale may put w/scale a hair above 1
        assert q[0, 0] == 15 and q[0, 1] == 0
