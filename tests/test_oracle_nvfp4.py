"""Pins of the oracle's NVFP4 weight format (CPU).

The references:
- the E2M1 definition (sign, 2 exponent bits with bias 1, 1 mantissa bit);
- brute force over its 8 magnitudes;
- a block worked by hand;
- the scale rules stated in the oracle, with the error bounds they imply;
- a brute-force GEMV.
"""
import math

import numpy as np
import pytest

import synth
from oracle import mxfp8 as MX
from oracle import nvfp4 as F


def test_e2m1_table():
    t = F.e2m1_table()
    assert t[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert t[8:].tolist() == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    assert math.copysign(1.0, t[8]) == -1.0


def brute_e2m1(y: float) -> int:
    """Nearest magnitude by search, ties to the even code, clamp at 6, sign kept."""
    mags = F.e2m1_table()[:8]
    a = min(abs(y), 6.0)
    best = min(range(8), key=lambda c: (abs(mags[c] - a), c % 2))
    return best | (0x8 if math.copysign(1.0, y) < 0 else 0)


def test_e2m1_rounding_matches_brute_force():
    mags = F.e2m1_table()[:8]
    mids = (mags[1:] + mags[:-1]) / 2  # every tie
    rng = np.random.default_rng(0)
    vals = np.concatenate([mids, -mids, mags, -mags, rng.uniform(-7, 7, 2000), [6.5, 100.0, -1e9, 1e-9, -1e-9]])
    got = F.e2m1_encode(vals)
    want = np.array([brute_e2m1(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)
    # the ties by hand: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    assert F.e2m1_decode(F.e2m1_encode(mids)).tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def test_e2m1_round_trip():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(F.e2m1_encode(F.e2m1_decode(codes)), codes)


@pytest.mark.parametrize("amax,g", [(2688.0, 1.0), (2689.0, 2.0), (1.0, 2.0 ** -11), (1344.0, 0.5),
                                    (0.0, 1.0)])
def test_tensor_scale(amax, g):
    assert F.tensor_scale(np.array([[amax, -amax / 3]])) == g


def test_worked_blocks():
    # tensor max 1.3125 = 2688 * 2^-11 -> g = 2^-11; block 0 scale E4M3(1.3125 / (6 g)) = 448 (0x7E),
    # so one step of the block is 448 * 2^-11 = 0.21875
    row = np.zeros((1, 32))
    row[0, :10] = [1.3125, 0.5, -0.1, 0.05, -0.01, 0.9, 1.1, 0.65625, 0.765625, 0.0]
    # block 1: amax 0.01 -> 0.01 / (6 g) = 3.41 -> E4M3 3.5 (0x46); 0.01 / (3.5 g) = 5.85 -> 6
    row[0, 16] = 0.01
    codes, s, g = F.quantize(row)
    assert g == 2.0 ** -11 and s.tolist() == [[0x7E, 0x46]]
    # 6 | 2.29 -> 2 | -0.457 -> -0.5 | 0.229 -> 0 | -0.046 -> -0 | 4.11 -> 4 | 5.03 -> 6 | 3 | 3.5 (tie) -> 4 | 0
    assert codes[0, :10].tolist() == [7, 4, 9, 0, 8, 6, 7, 5, 6, 0] and codes[0, 16] == 7
    deq = F.dequantize(codes, s, g)
    assert deq[0, :9].tolist() == [1.3125, 0.4375, -0.109375, 0.0, 0.0, 0.875, 1.3125, 0.65625, 0.875]
    assert deq[0, 16] == 6 * 3.5 * 2.0 ** -11


def test_error_bounds_and_exactness_on_normalised_rows():
    rng = np.random.default_rng(1)
    w = rng.standard_normal((48, 256))
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    w = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w.astype(np.float32))).astype(np.float64)
    codes, s, g = F.quantize(w)
    deq = F.dequantize(codes, s, g)
    amax = np.abs(w).max()
    assert 6 * 448 * g >= amax > 6 * 448 * g / 2
    sv = MX.e4m3_decode(s)
    assert sv.max() <= 448 and sv.max() > 224
    for n in range(0, 48, 7):
        for k in range(256):
            b = k // 16
            assert abs(w[n, k] - deq[n, k]) <= F.element_error_bound(w[n, k], g, sv[n, b]) * (1 + 1e-12)
    # every dequantised weight is a bf16 value (short mantissas times a power of two)
    f32 = deq.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), deq)
    assert np.array_equal(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(f32)), f32)


def test_gemv_matches_brute_force_sum():
    rng = np.random.default_rng(2)
    w = rng.standard_normal((3, 32)) * 0.05
    x = rng.standard_normal((2, 32))
    codes, s, g = F.quantize(w)
    t, st = F.e2m1_table(), MX.e4m3_table()
    want = np.zeros((2, 3))
    for m in range(2):
        for n in range(3):
            want[m, n] = sum(g * st[s[n, k // 16]] * t[codes[n, k]] * x[m, k] for k in range(32))
    assert np.allclose(F.gemv(x, codes, s, g), want, rtol=1e-12, atol=1e-15)


def test_quantized_weights_keep_the_embedding():
    w = synth.make_weights(synth.TINY_BF16, 3)
    q = F.quantized_weights(w)
    assert q["embed"] is w["embed"]
    f = (w["L1.wdown"].astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(q["L1.wdown"].astype(np.float64), F.dequantize(*F.quantize(f)))
