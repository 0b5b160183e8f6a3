"""The online softmax of the tcgen05 prefill attention kernels
(csrc/attn_prefill_ws.cu, csrc/attn_prefill_tc.cu), restated for one query
row in numpy and checked against the exact softmax-weighted sum in float64.

What the kernels do per row: scores arrive in log2 units (the queries are
pre-scaled by log2(e)/sqrt(head_dim)) one 128-key tile at a time; masked
keys are -inf; the running maximum used for the exponentials moves only
when a tile's maximum exceeds it by more than 8 (then O and the row sum are
rescaled by 2^(old - new)); P = 2^(s - m) is summed into the row sum in
fp32 and rounded to bf16 for the P V product, which accumulates in fp32; the
output is O / sum.  The lazy maximum bounds every P by 2^8, so nothing
overflows, and the result must stay within the bf16 rounding of P of the
exact answer, whatever the score pattern: slow drifts just under the
threshold, long fully masked prefixes, huge ranges, ties.
"""
import numpy as np
import pytest

TK = 128
LAZY = 8.0


def bf16(x):
    """Round float32 values to bf16 (nearest, ties to even), back as float32."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def kernel_row(s, v, lazy=LAZY):
    """s: scores in log2 units (float32, -inf where masked); v: [keys, d]."""
    s = s.astype(np.float32)
    m_used, l = np.float32(-1e30), np.float32(0)
    o = np.zeros(v.shape[1], np.float32)
    p_max = 0.0
    for t0 in range(0, len(s), TK):
        st = s[t0:t0 + TK]
        mt = np.float32(st.max())
        factor = np.float32(1)
        if mt > m_used + np.float32(lazy):
            factor = np.float32(np.exp2(np.float32(m_used - mt)))
            m_used = mt
        o *= factor
        l *= factor
        p = np.exp2((st - m_used).astype(np.float32)).astype(np.float32)
        p_max = max(p_max, float(p.max()))
        l += np.float32(p.sum(dtype=np.float32))
        o += bf16(p) @ v[t0:t0 + TK].astype(np.float32)
    return o / l, p_max


def exact_row(s, v):
    s64 = s.astype(np.float64)
    w = np.exp2(s64 - s64[np.isfinite(s64)].max())
    w[~np.isfinite(s64)] = 0.0
    return (w @ v.astype(np.float64)) / w.sum()


def scores(kind, n, rng):
    if kind == "random":
        return rng.normal(0, 3, n)
    if kind == "drift_under_threshold":  # each tile's maximum 7.9 above the last
        return np.repeat(np.arange(n // TK + 1) * 7.9, TK)[:n] + rng.uniform(-1, 0, n)
    if kind == "drift_over_threshold":
        return np.repeat(np.arange(n // TK + 1) * 8.1, TK)[:n] + rng.uniform(-1, 0, n)
    if kind == "masked_prefix":  # a window: the first tiles see nothing
        s = rng.normal(0, 2, n)
        s[: n - 200] = -np.inf
        return s
    if kind == "huge_range":
        return rng.uniform(-1000, 1000, n)
    if kind == "ties":
        return np.full(n, 3.25)
    if kind == "falling":
        return np.linspace(50, -50, n)
    if kind == "one_key":
        s = np.full(n, -np.inf)
        s[n // 2] = 0.0
        return s
    raise ValueError(kind)


KINDS = ["random", "drift_under_threshold", "drift_over_threshold", "masked_prefix", "huge_range", "ties",
         "falling", "one_key"]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("n", [1, 128, 300, 4096])
def test_lazy_online_softmax_within_bf16_of_exact(kind, n):
    rng = np.random.default_rng(n)
    s = scores(kind, n, rng).astype(np.float32)
    if not np.isfinite(s).any():
        s[-1] = 0.0  # every real query row sees at least itself
    v = rng.normal(0, 1, (n, 128)).astype(np.float32)
    got, p_max = kernel_row(s, v)
    want = exact_row(s, v)
    assert np.all(np.isfinite(got))
    assert p_max <= 2.0 ** LAZY
    # each P carries a bf16 rounding (relative <= 2^-9) into the numerator
    # only, so the output moves by at most 2^-9 max|V| (+1% for fp32 sums)
    assert np.abs(got - want).max() <= 1.01 * 2.0 ** -9 * np.abs(v).max()


def test_lazy_maximum_changes_results_only_by_rounding():
    """Threshold 0 (a rescale at every new maximum) and threshold 8 agree to
    within the bf16 rounding of P."""
    rng = np.random.default_rng(5)
    s = (np.repeat(np.arange(32) * 3.0, TK) + rng.normal(0, 2, 32 * TK)).astype(np.float32)
    v = rng.normal(0, 1, (32 * TK, 128)).astype(np.float32)
    a, _ = kernel_row(s, v, lazy=0.0)
    b, pb = kernel_row(s, v)
    assert pb > 1.0  # the lazy maximum did lag behind the true one
    assert np.abs(a - b).max() <= 2 * 1.01 * 2.0 ** -9 * np.abs(v).max()  # each within the bound of exact


def test_a_dropped_rescale_is_caught():
    """The check has teeth: not rescaling O when the maximum moves (a plausible
    kernel mistake) fails the bound on a drifting row."""
    rng = np.random.default_rng(1)
    n = 1024
    s = scores("drift_over_threshold", n, rng).astype(np.float32)
    v = rng.normal(0, 1, (n, 128)).astype(np.float32)
    m_used, l, o = np.float32(-1e30), np.float32(0), np.zeros(128, np.float32)
    for t0 in range(0, n, TK):
        st = s[t0:t0 + TK]
        mt = np.float32(st.max())
        if mt > m_used + LAZY:
            l *= np.float32(np.exp2(np.float32(m_used - mt)))  # O is not rescaled
            m_used = mt
        p = np.exp2(st - m_used).astype(np.float32)
        l += p.sum(dtype=np.float32)
        o += bf16(p) @ v[t0:t0 + TK]
    assert np.abs(o / l - exact_row(s, v)).max() > 1.01 * 2.0 ** -9 * np.abs(v).max()
