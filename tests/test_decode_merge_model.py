"""The decode attention's split-KV merge (csrc/attn_decode.cu,
k_attn_decode_tc), restated for one query row in numpy and checked against
the exact softmax-weighted sum in float64.

The kernel: the visible keys are split over the CTAs of a cluster, and each
CTA's keys over its warps; a warp runs a base-2 online softmax over its keys
(max m, sum l, accumulator a); a CTA merges its warps with weights
2^(m_w - M) (0 for a warp that saw no key, whose m is -FLT_MAX), then the
cluster merges its CTAs the same way in rank order and divides by the total
sum.  Ranks and warps without keys are the normal case at short context
(16 CTAs x 8 warps for a handful of keys); they must drop out exactly, and a
row's result must not depend on how its keys are split.
"""
import numpy as np
import pytest

NEG = np.float32(-np.finfo(np.float32).max)


def warp_partial(s, v):
    """Online softmax of one warp over its keys, in key order (fp32)."""
    m, l, a = NEG, np.float32(0), np.zeros(v.shape[1], np.float32)
    for j in range(len(s)):
        mn = max(m, s[j])
        c = np.float32(np.exp2(np.float32(m - mn))) if m != NEG else np.float32(0)
        p = np.float32(np.exp2(np.float32(s[j] - mn)))
        l = np.float32(l * c + p)
        a = (a * c + p * v[j]).astype(np.float32)
        m = mn
    return m, l, a


def merge(parts):
    """(m, l, a) of several partials -> one, empty partials weighted 0."""
    M = max(p[0] for p in parts)
    L, A = np.float32(0), np.zeros_like(parts[0][2])
    for m, l, a in parts:
        w = np.float32(0) if m == NEG else np.float32(np.exp2(np.float32(m - M)))
        L = np.float32(L + l * w)
        A = (A + a * w).astype(np.float32)
    return M, L, A


def kernel_row(s, v, ranks, warps, rng):
    """Keys split into contiguous ranges over ranks, each range over warps
    (some ranges empty), merged warp -> rank -> cluster."""
    n = len(s)
    cuts = np.sort(rng.integers(0, n + 1, ranks - 1))
    bounds = np.concatenate([[0], cuts, [n]])
    rank_parts = []
    for r in range(ranks):
        lo, hi = bounds[r], bounds[r + 1]
        wc = np.sort(rng.integers(lo, hi + 1, warps - 1))
        wb = np.concatenate([[lo], wc, [hi]])
        rank_parts.append(merge([warp_partial(s[wb[w]:wb[w + 1]], v[wb[w]:wb[w + 1]]) for w in range(warps)]))
    _, L, A = merge(rank_parts)
    return A / L


def exact_row(s, v):
    w = np.exp2(s.astype(np.float64) - s.max())
    return (w @ v.astype(np.float64)) / w.sum()


@pytest.mark.parametrize("n", [1, 2, 5, 37, 300, 2600])
@pytest.mark.parametrize("ranks", [4, 8, 16])
def test_split_merge_matches_exact(n, ranks):
    rng = np.random.default_rng(n * 31 + ranks)
    s = rng.normal(0, 4, n).astype(np.float32)
    v = rng.normal(0, 1, (n, 16)).astype(np.float32)
    got = kernel_row(s, v, ranks, 8, rng)
    assert np.all(np.isfinite(got))
    assert np.abs(got - exact_row(s, v)).max() <= 1e-5 * np.abs(v).max()


def test_every_key_on_one_rank_and_one_warp():
    """All other ranks and warps empty: their -FLT_MAX maxima drop out."""
    rng = np.random.default_rng(2)
    s = rng.normal(0, 3, 9).astype(np.float32)
    v = rng.normal(0, 1, (9, 16)).astype(np.float32)
    parts = [warp_partial(s[:0], v[:0])] * 15 + [warp_partial(s, v)]
    _, L, A = merge(parts)
    assert np.abs(A / L - exact_row(s, v)).max() <= 1e-5


def test_large_score_ranges_do_not_overflow():
    rng = np.random.default_rng(3)
    s = rng.uniform(-500, 500, 1000).astype(np.float32)
    v = rng.normal(0, 1, (1000, 16)).astype(np.float32)
    got = kernel_row(s, v, 16, 8, rng)
    assert np.all(np.isfinite(got)) and np.abs(got - exact_row(s, v)).max() <= 1e-5


def test_an_empty_partial_weighted_by_its_sentinel_is_caught():
    """The check has teeth: weighting an empty partial by 2^(m - M) with a
    finite stand-in maximum of 0 instead of dropping it moves the result
    when every score is negative (the empty partial then claims weight)."""
    s = np.array([-30.0, -31.0], np.float32)
    v = np.array([[1.0], [-1.0]], np.float32)
    good = merge([warp_partial(s, v), warp_partial(s[:0], v[:0])])
    bad_empty = (np.float32(0), np.float32(1), np.zeros(1, np.float32))  # a stand-in with l = 1
    bad = merge([warp_partial(s, v), bad_empty])
    want = exact_row(s, v)
    assert np.abs(good[2] / good[1] - want).max() <= 1e-6
    assert np.abs(bad[2] / bad[1] - want).max() > 1e-3
