"""Host-side work planning of the prefill attention (CPU): the row tiles a
ragged batch is cut into, and the work items of the warp-specialised
tcgen05 kernel, called in libdory.so directly (they touch no device).

Tiles: every row of every sequence in exactly one tile, tiles never span two
sequences, at most `rows` rows each, in row order; too small a capacity is
an error (-1), not a truncation.

Items: every (row tile, query head) pair in exactly one slot of one item;
two slots of one item share one K/V stream: either two consecutive heads of
one KV group on the same tile, or the group's last head (when the group has
an odd number of heads) on two consecutive tiles of the same sequence; items
are ordered by their key-tile count, largest first (the hardware hands
blocks to SMs in index order, so the long items start first).
"""
import ctypes

import numpy as np
import pytest

import looped_ngpt_lm_b200 as dory

lib = dory.lib
INT = ctypes.c_int
_tiles = getattr(lib, "_ZN4dory13prefill_tilesEiPKiP4int2ii")
_tiles.argtypes = [INT, ctypes.POINTER(INT), ctypes.c_void_p, INT, INT]
_tiles.restype = INT
_items = getattr(lib, "_ZN4dory16prefill_ws_itemsEiPKiS1_iiP4int4i")
_items.argtypes = [INT, ctypes.POINTER(INT), ctypes.POINTER(INT), INT, INT, ctypes.c_void_p, INT]
_items.restype = INT
TK = 128


def ints(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.POINTER(INT))


def tiles_of(lens, rows=128, cap=None):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    n_max = sum((n + rows - 1) // rows for n in lens)
    cap = n_max if cap is None else cap
    out = np.zeros((max(cap, 1), 2), np.int32)
    cu_a, cu_p = ints(cu)
    n = _tiles(len(lens), cu_p, out.ctypes.data, cap, rows)
    return n, out[:max(n, 0)], cu


def items_of(last_pos, seq, H, KV, cap=None):
    n = len(last_pos)
    cap = n * H if cap is None else cap
    out = np.zeros((max(cap, 1), 4), np.int32)
    lp, lp_p = ints(last_pos)
    sq, sq_p = ints(seq)
    k = _items(n, lp_p, sq_p, H, KV, out.ctypes.data, cap)
    return k, out[:max(k, 0)]


@pytest.mark.parametrize("lens", [[1], [128], [129], [2560], [300, 5, 260], [128, 128, 1, 255], [700] * 7])
@pytest.mark.parametrize("rows", [64, 128])
def test_tiles_cover_each_sequence_in_order(lens, rows):
    n, t, cu = tiles_of(lens, rows)
    assert n == sum((x + rows - 1) // rows for x in lens)
    covered = np.zeros(cu[-1], np.int32)
    for a, b in t:
        assert 0 < b - a <= rows
        s = np.searchsorted(cu, a, side="right") - 1
        assert b <= cu[s + 1]  # inside one sequence
        covered[a:b] += 1
    assert np.all(covered == 1)
    assert np.all(t[1:, 0] == t[:-1, 1])  # in row order, no gaps


def test_tiles_capacity_is_an_error():
    n, _, _ = tiles_of([300, 300], 128, cap=5)
    assert n == -1


def plan(lens, positions0, H, KV):
    """Tiles of a ragged batch whose sequence b starts at position
    positions0[b] (a later chunk), with each tile's last position and
    sequence."""
    n, t, cu = tiles_of(lens)
    seq = np.searchsorted(cu, t[:, 0], side="right") - 1
    last = np.array([positions0[s] + (b - 1 - cu[s]) for (a, b), s in zip(t, seq)], np.int32)
    k, it = items_of(last, seq, H, KV)
    return n, last, seq, k, it


CASES = [
    ([2560], [0], 20, 4),          # the 4B shape: 5 heads per KV group
    ([300, 5, 260], [0, 0, 0], 5, 1),
    ([400], [4096], 20, 4),        # a later chunk: long key ranges
    ([640, 129, 1], [0, 640, 77], 20, 4),
    ([1000], [0], 4, 1),           # 4 heads per group: no cross-tile pairs
    ([130, 130], [0, 0], 6, 2),    # 3 heads per group
    ([128] * 5, [0, 0, 0, 0, 0], 20, 4),  # one tile per sequence: the odd head runs alone
]


@pytest.mark.parametrize("lens,pos0,H,KV", CASES)
def test_items_cover_every_tile_and_head_once(lens, pos0, H, KV):
    n, last, seq, k, it = plan(lens, pos0, H, KV)
    G = H // KV
    seen = np.zeros((n, H), np.int32)
    for x, y, z, w in it:
        seen[x, y] += 1
        if z >= 0:
            seen[z, w] += 1
            if x == z:  # two heads of one group on the same rows
                assert w == y + 1 and y // G == w // G and (y % G) % 2 == 0
            else:  # the group's odd head on consecutive tiles of one sequence
                assert G % 2 == 1 and y == w and y % G == G - 1
                assert z == x + 1 and seq[x] == seq[z]
        else:
            assert w == -1 and G % 2 == 1 and y % G == G - 1
    assert np.all(seen == 1)


@pytest.mark.parametrize("lens,pos0,H,KV", CASES)
def test_items_run_longest_first(lens, pos0, H, KV):
    _, last, _, _, it = plan(lens, pos0, H, KV)
    cost = [last[z if z >= 0 else x] // TK + 1 for x, _, z, _ in it]
    assert all(a >= b for a, b in zip(cost, cost[1:]))


def test_odd_heads_pair_greedily_within_a_sequence():
    """Three tiles of one sequence: tiles 0 and 1 share an item for the odd
    head, tile 2 runs alone; a tile of the next sequence never joins it."""
    _, _, _, _, it = plan([384, 128], [0, 0], 5, 1)
    odd = sorted((x, z) for x, y, z, w in it if y == 4)
    assert odd == [(0, 1), (2, -1), (3, -1)]


def test_items_capacity_is_an_error():
    k, _ = items_of(np.array([127, 255], np.int32), np.array([0, 0], np.int32), 20, 4, cap=10)
    assert k == -1
