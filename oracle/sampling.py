"""Temperature / top-p sampling, the oracle's plain restatement (test
infrastructure: only tests/, the smoke check and the bench's CPU baseline use
this package).

The pages name the sampling settings of the released model (temperature 1.0,
top-p 0.95: news, "How to run") but no procedure; the reading taken here
(see the repository's design notes) is:

1. A seeded counter-based generator gives one uniform draw per generated
   token: Philox4x32 with 10 rounds (Salmon, Moraes, Dror and Shaw, "Parallel
   random numbers: as easy as 1, 2, 3", SC 2011), key = (seed low 32 bits,
   seed high 32 bits), counter = (sequence id, position of the new token, 0,
   0); u = (first output word >> 8) / 2^24.
2. e_i = exp2((l_i - max l) * log2(e) / T) in float32, and the integer masses
   q_i = floor(e_i * 2^31).
3. Q = sum q_i; P = ceil(top_p * Q).  The nucleus is {i : q_i >= tau} with
   tau the largest value such that sum_{q_i >= tau} q_i >= P (ties at the
   threshold are all kept).
4. M = sum of the nucleus masses; r = floor(u * M), computed exactly as
   ((word >> 8) * M) >> 24; the token is the first index j, in token order,
   at which the running sum of nucleus masses exceeds r.

Steps 3 and 4 are integer work; only step 2 depends on how exp2 is rounded.
"""
from __future__ import annotations

import math

import numpy as np

M0, M1 = 0xD2511F53, 0xCD9E8D57  # round multipliers
W0, W1 = 0x9E3779B9, 0xBB67AE85  # key increments (golden ratio, sqrt(3) - 1)
MASK = 0xFFFFFFFF


def philox4x32_10(counter, key):
    """Philox4x32 with 10 rounds: four 32-bit counter words, two key words."""
    c0, c1, c2, c3 = (int(v) & MASK for v in counter)
    k0, k1 = (int(v) & MASK for v in key)
    for r in range(10):
        if r:
            k0, k1 = (k0 + W0) & MASK, (k1 + W1) & MASK
        p0, p1 = M0 * c0, M1 * c2
        c0, c1, c2, c3 = ((p1 >> 32) ^ c1 ^ k0), p1 & MASK, ((p0 >> 32) ^ c3 ^ k1), p0 & MASK
    return c0, c1, c2, c3


def uniform_word(seed: int, seq: int, pos: int) -> int:
    """The first output word of the draw for (sequence, position)."""
    return philox4x32_10((seq, pos, 0, 0), (seed & MASK, (seed >> 32) & MASK))[0]


def masses(logits: np.ndarray, temperature: float) -> np.ndarray:
    """Integer masses q_i = floor(exp2((l_i - max) * log2(e) / T) * 2^31)."""
    l = np.asarray(logits, dtype=np.float32)
    scale = np.float32(1.4426950408889634 / temperature)
    e = np.exp2((l - l.max()) * scale, dtype=np.float32)
    return np.floor(e.astype(np.float64) * 2.0 ** 31).astype(np.int64)


def nucleus_threshold(q: np.ndarray, top_p: float) -> int:
    """Largest tau with sum(q[q >= tau]) >= ceil(top_p * sum(q))."""
    P = math.ceil(float(top_p) * int(q.sum()))
    desc = np.sort(q)[::-1]
    cum = np.cumsum(desc)
    idx = int(np.searchsorted(cum, P, side="left"))
    return int(desc[min(idx, len(desc) - 1)])


def draw(seed: int, seq: int, pos: int, M: int) -> int:
    """r = floor(u * M) for the draw u = (word >> 8) / 2^24 of (seq, pos)."""
    return ((uniform_word(seed, seq, pos) >> 8) * int(M)) >> 24


def choose(mass, r: int) -> int:
    """The first index at which the running sum of `mass` exceeds r."""
    return int(np.searchsorted(np.cumsum(mass), r, side="right"))


def sample(logits, temperature: float, top_p: float, seed: int, seq: int, pos: int) -> int:
    """The token drawn for sequence `seq` at position `pos`.  Temperature and
    top_p are float32 parameters (rounded to float32 first)."""
    temperature, top_p = float(np.float32(temperature)), float(np.float32(top_p))
    q = masses(logits, temperature)
    tau = nucleus_threshold(q, top_p)
    mass = np.where(q >= tau, q, 0)
    return choose(mass, draw(seed, seq, pos, int(mass.sum())))
