"""MXFP8 weights, the oracle's plain restatement (test infrastructure: only
tests/, the smoke check and the bench's CPU legs use this package).

The pages list MXFP8 among the released weight formats and measure its batch-1
decode speed against BF16 ("NVIDIA, 반복 연산형 4B 언어 모델 Dory 공개",
section "KV 캐시와 실행 환경"; the lucasainews formats article, section
"학습 방식과 변형"), but do not define the format.  The
reading taken here is the OCP Microscaling Formats (MX) Specification v1.0
with FP8 E4M3 elements:

* A block is 32 consecutive elements of one weight row (along the reduction
  dimension K).  It shares one E8M0 scale X = 2^(byte - 127).
* E4M3 has 1 sign bit, 4 exponent bits (bias 7) and 3 mantissa bits.  Its
  subnormals are m/8 * 2^-6, and its largest finite value is 448
  (S.1111.110).  S.1111.111 is NaN.  There is no infinity.
* Quantising a block, per section 6.3 of the specification:
  shared = floor(log2(max |v|)) - 8, since 8 is the exponent of E4M3's
  largest normal.  Each element becomes P_i = E4M3(v_i / 2^shared), rounded
  to nearest-even, with magnitudes above 448 clamped to 448.
* Dequantising: w_i = 2^shared * P_i.

Readings where the specification leaves a choice:

* shared is clamped to [-127, 127].  A block of zeros takes -127 (byte 0).
* A value that rounds to zero keeps its sign, so a negative one becomes code
  0x80.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
E4M3_MAX = 448.0
EMAX_ELEM = 8  # exponent of the largest normal E4M3 value (448 = 1.75 * 2^8)
SCALE_BIAS = 127


def e4m3_value(code: int) -> float:
    """The real number an E4M3 byte encodes (NaN for S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """All 256 codes decoded (float64, NaN at 0x7F and 0xFF)."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(y) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to the even mantissa, clamping
    finite magnitudes above 448 to 448.  Returns uint8 codes."""
    y = np.asarray(y, dtype=np.float64)
    neg = np.signbit(y)
    a = np.minimum(np.abs(y), E4M3_MAX)
    # exponent of the binade holding a (subnormal binade for a < 2^-6)
    _, ex = np.frexp(a)  # a = f * 2^ex with f in [0.5, 1), ex = floor(log2 a) + 1
    e = np.maximum(ex - 1, -6)
    quantum = np.ldexp(1.0, e - 3)  # spacing of E4M3 values in that binade
    n = np.rint(a / quantum)  # integer multiple of the spacing, ties to even
    v = n * quantum  # the rounded magnitude (may be 2^(e+1): next binade)
    # encode the magnitude v
    _, vx = np.frexp(v)
    ve = vx - 1  # floor(log2 v) for v > 0
    sub = v < 2.0 ** -6
    code = np.where(
        v == 0,
        0,
        np.where(sub, np.rint(v / 2.0 ** -9), ((ve + 7) << 3) + np.rint(v / np.ldexp(1.0, ve - 3)) - 8),
    ).astype(np.int64)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, dtype=np.int64)]


def block_exponent(amax) -> np.ndarray:
    """shared = floor(log2(amax)) - 8, clamped to [-127, 127]; -127 for amax == 0."""
    amax = np.asarray(amax, dtype=np.float64)
    _, ex = np.frexp(amax)
    shared = np.where(amax > 0, ex - 1 - EMAX_ELEM, -SCALE_BIAS)
    return np.clip(shared, -SCALE_BIAS, SCALE_BIAS).astype(np.int64)


def quantize(w) -> tuple[np.ndarray, np.ndarray]:
    """MXFP8 copy of a [N, K] matrix (K % 32 == 0): E4M3 codes uint8 [N, K]
    and E8M0 scale bytes uint8 [N, K/32] (the block of element (n, k) is
    k // 32)."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    assert K % BLOCK == 0
    blocks = w.reshape(N, K // BLOCK, BLOCK)
    shared = block_exponent(np.max(np.abs(blocks), axis=-1))
    scaled = blocks / np.ldexp(1.0, shared)[..., None]  # exact: a power of two
    codes = e4m3_encode(scaled).reshape(N, K)
    return codes, (shared + SCALE_BIAS).astype(np.uint8)


def dequantize(codes, scales) -> np.ndarray:
    """w[n, k] = 2^(scales[n, k // 32] - 127) * E4M3(codes[n, k]) (float64)."""
    codes = np.asarray(codes)
    N, K = codes.shape
    X = np.ldexp(1.0, np.asarray(scales, dtype=np.int64) - SCALE_BIAS)
    return (e4m3_decode(codes).reshape(N, K // BLOCK, BLOCK) * X[..., None]).reshape(N, K)


def gemv(x, codes, scales) -> np.ndarray:
    """y = x . dequantize(codes, scales)^T for x [M, K] (float64)."""
    return np.asarray(x, dtype=np.float64) @ dequantize(codes, scales).T


def quantized_weights(weights: dict) -> dict:
    """The model's weights with every projection matrix and the LM head
    replaced by its MXFP8 dequantisation (float32: exact, each value is a
    3-bit-mantissa multiple of a power of two).  The embedding, a gather, keeps
    its original values."""
    out = {}
    for name, a in weights.items():
        if name == "embed":
            out[name] = a
            continue
        f = a
        if a.dtype == np.uint16:  # bf16 bit patterns: widen exactly
            f = (a.astype(np.uint32) << 16).view(np.float32)
        out[name] = dequantize(*quantize(f)).astype(np.float32)
    return out
