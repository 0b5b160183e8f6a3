"""Pins of the oracle's MXFP8 weight format (CPU).

The references are the E4M3 definition (the OCP 8-bit floating point
specification, also the OCP MX v1.0 element format), PyTorch's float8_e4m3fn
conversions (a library routine), brute force over the 254 finite codes, and
hand-worked blocks."""
import math

import numpy as np
import pytest
import torch

from oracle import mxfp8 as MX


def test_decode_known_codes():
    t = MX.e4m3_table()
    assert t[0x00] == 0.0 and t[0x80] == 0.0 and math.copysign(1, t[0x80]) == -1
    assert t[0x38] == 1.0  # exponent field 7 = bias
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0  # largest finite
    assert t[0x01] == 2.0 ** -9  # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9  # largest subnormal
    assert t[0x08] == 2.0 ** -6  # smallest normal
    assert t[0x3C] == 1.5 and t[0x40] == 2.0 and t[0x6A] == 80.0
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    assert np.sum(np.isnan(t)) == 2


def test_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    t = MX.e4m3_table()
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(t), np.isnan(ref))
    assert np.array_equal(t[fin], ref[fin])


def brute_encode(y: float) -> int:
    """Nearest finite code by exhaustive search; ties to the even code (the
    mantissa's last bit); clamp beyond 448; the sign of y kept on zero."""
    t = MX.e4m3_table()
    a = min(abs(y), 448.0)
    best, bd = None, None
    for c in range(0x7F):  # non-negative finite codes 0x00..0x7E
        d = abs(t[c] - a)
        if bd is None or d < bd or (d == bd and c % 2 == 0 and best % 2 == 1):
            best, bd = c, d
    return best | (0x80 if math.copysign(1.0, y) < 0 else 0)


def test_encode_matches_brute_force_on_midpoints_and_random_values():
    t = MX.e4m3_table()
    pos = np.sort(t[:0x7F])
    mids = (pos[1:] + pos[:-1]) / 2  # every exact tie between neighbours
    rng = np.random.default_rng(0)
    vals = np.concatenate([mids, -mids, pos, -pos, rng.standard_normal(400) * 100,
                           rng.uniform(-2 ** -6, 2 ** -6, 100), [449.0, 464.0, 470.0, 1e6, -1e6, 2.0 ** -11, -2.0 ** -11]])
    got = MX.e4m3_encode(vals)
    want = np.array([brute_encode(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_encode_matches_torch_cast_within_range():
    rng = np.random.default_rng(1)
    y = np.concatenate([rng.standard_normal(5000) * 50, rng.uniform(-448, 448, 5000),
                        rng.uniform(-0.02, 0.02, 2000)]).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(MX.e4m3_encode(y), ref)


def test_finite_codes_round_trip():
    t = MX.e4m3_table()
    fin = [c for c in range(256) if not math.isnan(t[c])]
    assert np.array_equal(MX.e4m3_encode(t[fin]), np.array(fin, dtype=np.uint8))


@pytest.mark.parametrize("amax,shared", [(1.0, -8), (448.0, 0), (0.75, -9), (511.9, 0), (512.0, 1),
                                         (0.0, -127), (2.0 ** -140, -127), (2.0 ** -118, -126)])
def test_block_exponent(amax, shared):
    assert int(MX.block_exponent(amax)) == shared


def test_worked_block():
    # amax 1.0 -> shared -8 (scale byte 119); 0.3 * 256 = 76.8 lies in [64, 128)
    # where E4M3 steps by 8: 76.8 -> 80 (code 0x6A), dequantised 80 / 256.
    row = np.zeros((1, 32))
    row[0, :4] = [1.0, 0.3, -0.3, 0.0]
    row[0, 4] = 0.001  # 0.256 in [1/4, 1/2), step 1/32: 8.19 steps -> 0.25 (exponent field 5: code 0x28)
    row[0, 5] = 0.00003  # 0.00768 < 2^-6, subnormal step 2^-9: 3.93 -> 4 (code 0x04)
    row[0, 6] = -1e-7  # rounds to zero and keeps its sign (code 0x80)
    codes, scales = MX.quantize(row)
    assert scales.tolist() == [[119]]
    assert codes[0, :7].tolist() == [0x78, 0x6A, 0xEA, 0x00, 0x28, 0x04, 0x80]
    deq = MX.dequantize(codes, scales)
    assert deq[0, :6].tolist() == [1.0, 0.3125, -0.3125, 0.0, 0.25 / 256, 2.0 ** -15]


def test_clamp_in_a_block():
    # amax 1.9 -> shared -8; 1.9 * 256 = 486.4 > 448: clamped to 448
    row = np.zeros((1, 32))
    row[0, 0], row[0, 1] = 1.9, -1.9
    codes, scales = MX.quantize(row)
    assert scales[0, 0] == 119 and codes[0, 0] == 0x7E and codes[0, 1] == 0xFE


def test_quantisation_error_bounds_on_normalised_rows():
    rng = np.random.default_rng(2)
    w = rng.standard_normal((64, 256))
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    codes, scales = MX.quantize(w)
    deq = MX.dequantize(codes, scales)
    X = np.ldexp(1.0, scales.astype(np.int64) - 127)  # [64, 8]
    amax = np.abs(w).reshape(64, 8, 32).max(-1)
    s = amax / X
    assert np.all((s >= 256) & (s < 512))  # the scale puts the block maximum in [2^8, 2^9)
    assert not np.any((codes & 0x7F) == 0x7F)  # never NaN
    err = np.abs(w - deq).reshape(64, 8, 32)
    y = np.abs(w).reshape(64, 8, 32) / X[..., None]
    # half a step of E4M3 in the element's binade (2^(e-4) of the scaled value), 2^-10 below 2^-6,
    # and the clamp above 448 (at most 512 - 448)
    e = np.floor(np.log2(np.maximum(y, 2.0 ** -6)))
    bound = np.where(y > 448, y - 448, np.ldexp(1.0, (e - 4).astype(int))) * X[..., None]
    assert np.all(err <= bound * (1 + 1e-12))


def test_gemv_matches_brute_force_sum():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((3, 64)) * 0.05
    x = rng.standard_normal((2, 64))
    codes, scales = MX.quantize(w)
    t = MX.e4m3_table()
    want = np.zeros((2, 3))
    for m in range(2):
        for n in range(3):
            acc = 0.0
            for b in range(2):
                part = sum(t[codes[n, 32 * b + i]] * x[m, 32 * b + i] for i in range(32))
                acc += 2.0 ** (int(scales[n, b]) - 127) * part
            want[m, n] = acc
    assert np.allclose(MX.gemv(x, codes, scales), want, rtol=1e-12, atol=1e-15)


def test_quantized_weights_keep_the_embedding_and_are_exact_in_float32():
    import synth
    w = synth.make_weights(synth.TINY_BF16, 5)
    q = MX.quantized_weights(w)
    assert q["embed"] is w["embed"]
    f = (w["L1.wg"].astype(np.uint32) << 16).view(np.float32)
    deq64 = MX.dequantize(*MX.quantize(f))
    assert np.array_equal(q["L1.wg"].astype(np.float64), deq64)
    assert q["lm_head"].dtype == np.float32 and q["lm_head"].shape == w["lm_head"].shape
