"""NVFP4 weights, the oracle's plain restatement (test infrastructure: only
tests/, the smoke check and the bench's CPU legs use this package).

The pages list NVFP4 among the released weight formats and give its batch-1
decode speed over BF16, 2.17x to 2.44x ("NVIDIA, 반복 연산형 4B 언어 모델 Dory
공개", section "KV 캐시와 실행 환경"; the lucasainews formats article, section
"학습 방식과 변형"), but do not define the format.  The reading taken here is
NVIDIA's published NVFP4 format:

* Elements are FP4 E2M1: 1 sign bit, 2 exponent bits (bias 1) and 1 mantissa
  bit.  The magnitudes are 0, 0.5 (the only subnormal), 1, 1.5, 2, 3, 4 and
  6.  There is no infinity and no NaN.
* 16 consecutive elements of a weight row (along K) share one scale stored
  as FP8 E4M3.  One FP32 scale covers the whole tensor.
* w = E2M1(code) * E4M3(block scale) * tensor scale.

The quantisation recipe is the plainest one consistent with the format:

* tensor scale g = the smallest power of two with 6 * 448 * g >= max |w|.
  The largest block scale is then at most 448, the E4M3 maximum, and above
  224.  g = 1 for an all-zero tensor.  A power of two, rather than max |w| /
  2688 itself, keeps every dequantised weight exact in bf16: an E2M1 value
  (2 significant bits) times an E4M3 value (4 bits) times 2^k.
* block scale s_b = E4M3(amax_b / (6 * g)), rounded to nearest-even
  (oracle.mxfp8.e4m3_encode).
* code = E2M1(w / (s_b * g)), rounded to nearest-even, with magnitudes
  above 6 clamped to 6 and codes 0 for a block whose scale rounds to 0.  A
  value that rounds to zero keeps its sign.
"""
from __future__ import annotations

import math

import numpy as np

from . import mxfp8 as MX

BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def e2m1_value(code: int) -> float:
    """The number a 4-bit E2M1 code encodes."""
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * 0.5 * m  # subnormal: m/2 * 2^(1-1)
    return s * (1.0 + 0.5 * m) * 2.0 ** (e - 1)


def e2m1_table() -> np.ndarray:
    return np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def e2m1_encode(y) -> np.ndarray:
    """Round to the nearest E2M1 value, ties to the even mantissa (even code),
    magnitudes above 6 clamped to 6; the sign is kept on zero.  uint8 codes
    0..15."""
    y = np.asarray(y, dtype=np.float64)
    neg = np.signbit(y)
    a = np.minimum(np.abs(y), E2M1_MAX)
    # binade exponent: spacing 0.5 below 2, 1 in [2, 4), 2 in [4, 6]
    _, ex = np.frexp(a)
    e = np.maximum(ex - 1, 0)  # floor(log2 a), at least 0 (the subnormal binade [0, 1) steps by 0.5)
    quantum = np.ldexp(0.5, e)
    v = np.rint(a / quantum) * quantum  # nearest multiple, ties to even multiple
    mags = e2m1_table()[:8]
    code = np.searchsorted(mags, v)  # exact: v is one of the magnitudes
    return (code | np.where(neg, 0x8, 0)).astype(np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    return e2m1_table()[np.asarray(codes, dtype=np.int64)]


def tensor_scale(w) -> float:
    """The smallest power of two g with 6 * 448 * g >= max |w|; 1 for an
    all-zero tensor.  Found by exact comparisons (6 * 448 * 2^k is exact)."""
    amax = float(np.max(np.abs(np.asarray(w, dtype=np.float64))))
    if amax == 0:
        return 1.0
    top = E2M1_MAX * E4M3_MAX
    _, ex = math.frexp(amax / top)
    k = ex
    while math.ldexp(top, k) < amax:
        k += 1
    while math.ldexp(top, k - 1) >= amax:
        k -= 1
    return math.ldexp(1.0, k)


def quantize(w) -> tuple[np.ndarray, np.ndarray, float]:
    """NVFP4 copy of a [N, K] matrix (K % 16 == 0): E2M1 codes uint8 [N, K]
    (one code per byte here; packing two per byte is a storage matter), E4M3
    block-scale codes uint8 [N, K/16], and the power-of-two tensor scale."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    assert K % BLOCK == 0
    g = tensor_scale(w)
    blocks = w.reshape(N, K // BLOCK, BLOCK)
    amax = np.max(np.abs(blocks), axis=-1)
    s_codes = MX.e4m3_encode(amax / (E2M1_MAX * g))
    s = MX.e4m3_decode(s_codes)  # the block scales as numbers
    denom = (s * g)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        scaled = np.where(denom > 0, blocks / np.where(denom > 0, denom, 1.0), 0.0 * blocks)
    codes = e2m1_encode(scaled).reshape(N, K)
    return codes, s_codes, g


def dequantize(codes, s_codes, g: float) -> np.ndarray:
    """w[n, k] = E2M1(codes[n, k]) * E4M3(s_codes[n, k // 16]) * g (float64)."""
    codes = np.asarray(codes)
    N, K = codes.shape
    s = MX.e4m3_decode(s_codes) * float(g)
    return (e2m1_decode(codes).reshape(N, K // BLOCK, BLOCK) * s[..., None]).reshape(N, K)


def gemv(x, codes, s_codes, g: float) -> np.ndarray:
    """y = x . dequantize(codes, s_codes, g)^T for x [M, K] (float64)."""
    return np.asarray(x, dtype=np.float64) @ dequantize(codes, s_codes, g).T


def quantized_weights(weights: dict) -> dict:
    """Every projection matrix and the LM head replaced by its NVFP4
    dequantisation as float32 (exact: at most 6 significant bits times a
    power of two).  The embedding, a gather, keeps its values."""
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


def element_error_bound(w, g: float, s: float) -> float:
    """Half the E2M1 spacing at |w| in a block with scale s (times g), or the
    clamp loss above 6: the largest error the rounding may make."""
    a = abs(float(w)) / (s * g)
    if a > E2M1_MAX:
        return (a - E2M1_MAX) * s * g
    e = max(math.floor(math.log2(a)) if a > 0 else 0, 0)
    return 0.5 * math.ldexp(0.5, e) * s * g
