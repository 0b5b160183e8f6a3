"""Pins of the oracle's temperature / top-p sampler (CPU)."""
import math

import numpy as np
import pytest

from oracle import sampling as S


@pytest.mark.parametrize("counter,key,expect", [
    # known-answer vectors published with the Philox reference implementation
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
])
def test_philox_known_answers(counter, key, expect):
    assert S.philox4x32_10(counter, key) == expect


def test_tiny_top_p_is_greedy():
    rng = np.random.default_rng(3)
    for trial in range(20):
        l = rng.standard_normal(1000).astype(np.float32)
        l[rng.integers(0, 1000)] += 0.0  # keep a unique max in general
        best = int(np.argmax(l))
        for pos in range(5):
            assert S.sample(l, 1.0, 1e-9, seed=trial, seq=0, pos=pos) == best


def test_tiny_top_p_keeps_lowest_index_on_ties():
    l = np.zeros(16, np.float32)
    l[[3, 9]] = 2.0
    # both maxima are in the nucleus (ties at the threshold are kept); the draw picks between them
    got = {S.sample(l, 1.0, 1e-9, seed=s, seq=0, pos=0) for s in range(64)}
    assert got == {3, 9}


def test_full_top_p_follows_softmax():
    l = np.array([0.0, 1.0, -0.5, 2.0, 0.3, -2.0], np.float32)
    p = np.exp(l - l.max())
    p /= p.sum()
    n = 20000
    counts = np.bincount([S.sample(l, 1.0, 1.0, seed=11, seq=0, pos=i) for i in range(n)], minlength=len(l))
    sd = np.sqrt(n * p * (1 - p))
    assert np.all(np.abs(counts - n * p) <= 5 * sd + 1), (counts, n * p)


def test_top_p_cut_excludes_the_tail():
    # masses 0.5, 0.3, 0.15, 0.05 (by construction): top_p = 0.7 keeps the first two
    probs = np.array([0.15, 0.5, 0.05, 0.3])
    l = np.log(probs).astype(np.float32)
    n = 6000
    draws = [S.sample(l, 1.0, 0.7, seed=5, seq=1, pos=i) for i in range(n)]
    counts = np.bincount(draws, minlength=4)
    assert counts[0] == 0 and counts[2] == 0
    frac = counts[1] / n  # 0.5 / 0.8 within the nucleus
    assert abs(frac - 0.625) < 5 * math.sqrt(0.625 * 0.375 / n)


def test_threshold_keeps_ties_and_reaches_the_mass():
    q = np.array([5, 5, 5, 5], np.int64)
    assert S.nucleus_threshold(q, 0.5) == 5  # all four tie at the threshold
    q = np.array([10, 4, 4, 1], np.int64)
    assert S.nucleus_threshold(q, 0.5) == 10
    assert S.nucleus_threshold(q, 0.6) == 4  # 10 < ceil(0.6 * 19) = 12 <= 18
    assert S.nucleus_threshold(q, 1.0) == 1


def test_draws_depend_only_on_seed_sequence_and_position():
    l = np.random.default_rng(0).standard_normal(500).astype(np.float32)
    a = [S.sample(l, 1.0, 0.95, seed=7, seq=2, pos=i) for i in range(50)]
    b = [S.sample(l, 1.0, 0.95, seed=7, seq=2, pos=i) for i in range(50)]
    c = [S.sample(l, 1.0, 0.95, seed=8, seq=2, pos=i) for i in range(50)]
    assert a == b and a != c


@pytest.mark.parametrize("T", [0.5, 2.0])
def test_temperature_frequencies_follow_softmax_of_scaled_logits(T):
    l = np.array([0.0, 1.0, -0.5, 2.0, 0.3], np.float32)
    p = np.exp(l / T - (l / T).max())
    p /= p.sum()
    n = 20000
    counts = np.bincount([S.sample(l, T, 1.0, seed=21, seq=3, pos=i) for i in range(n)], minlength=len(l))
    sd = np.sqrt(n * p * (1 - p))
    assert np.all(np.abs(counts - n * p) <= 5 * sd + 1), (counts, n * p)


def test_masses_closed_forms():
    # the largest logit has mass 2^31; one T * ln 2 below it, exactly half (exp2(-1) = 0.5)
    for T in (1.0, 0.5, 2.0):
        l = np.array([3.0, 3.0 - T * math.log(2.0), -50.0], np.float32)
        q = S.masses(l, T)
        assert q[0] == 2 ** 31 and abs(int(q[1]) - 2 ** 30) <= 2 ** 31 * 2e-7 and q[2] >= 0


def test_nucleus_mass_is_rounded_up():
    # top_p * Q = 0.55 * 19 = 10.45: the nucleus must reach 10.45, so {10} (mass 10) is not enough
    assert S.nucleus_threshold(np.array([10, 4, 4, 1], np.int64), 0.55) == 4


def test_choice_rule_at_boundaries():
    mass = np.array([5, 0, 3], np.int64)  # running sums 5, 5, 8
    assert [S.choose(mass, r) for r in range(8)] == [0, 0, 0, 0, 0, 2, 2, 2]


def test_worked_draw_from_the_philox_known_answer():
    # seed 0, sequence 0, position 0: counter and key all zero, first output word 0x6627E8D5
    # (the published known answer), so u = 0x6627E8 / 2^24 and r = floor(u * M)
    assert S.draw(0, 0, 0, 2 ** 24) == 0x6627E8
    assert S.draw(0, 0, 0, 1000) == (0x6627E8 * 1000) >> 24  # 399
