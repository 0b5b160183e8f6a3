"""The barrier protocol of the TMA-fed low-bit GEMM (csrc/mx_gemm_tc.cu, MXFP8 and NVFP4), model-checked on
the CPU.

The kernel's roles, each restated as a state machine:
- the TMA producer (pre-issue of the first ring stages, main loop, drain);
- four converter warps;
- the MMA issuer;
- four epilogue warps.

The rings are the raw tiles (depth RS), the converted tiles (CS) and the TMEM block
slots (TS).

The mbarrier model: a phase completes after `count` arrivals (a TMA fill is the
producer's arrival), and try_wait.parity(p) succeeds when the current phase's parity
differs from p.

Random schedules must finish without deadlock, and every stage or slot a role reads
must hold the chunk that role expects.  Planted protocol mistakes must be caught.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.arrived, self.phase = count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count
        if self.arrived == self.count:
            self.arrived, self.phase = 0, self.phase + 1

    def try_wait(self, parity):
        return (self.phase & 1) != parity


def simulate(units, RS=7, CS=2, TS=4, seed=0, bug=None):
    chunks = [(u, c) for u, n in enumerate(units) for c in range(n)]
    raw_full, raw_empty = [Bar(1) for _ in range(RS)], [Bar(3 if bug == "count" else 4) for _ in range(RS)]
    conv_full, conv_empty = [Bar(4) for _ in range(CS)], [Bar(1) for _ in range(CS)]
    tfull, tempty = [Bar(1) for _ in range(TS)], [Bar(4) for _ in range(TS)]
    raw_slot, conv_slot, tmem, seen = [None] * RS, [None] * CS, [None] * TS, []

    def producer():
        npre = min(RS, len(chunks))
        for i in range(npre):  # codes before the predecessor is waited for, activations after
            raw_slot[i] = chunks[i]
            raw_full[i].arrive()
            yield ("step",)
        stage, phase = npre % RS, (0 if bug == "phase" else (1 if npre == RS else 0))
        issued = npre
        for ch in chunks[npre:]:
            yield ("wait", raw_empty[stage], phase ^ 1)
            raw_slot[stage] = ch
            raw_full[stage].arrive()
            issued += 1
            stage += 1
            if stage == RS:
                stage, phase = 0, phase ^ 1
        st, ph = stage, phase  # drain: the last min(issued, RS) fills must have landed
        for _ in range(min(RS, issued)):
            if st == 0:
                st, ph = RS, ph ^ 1
            st -= 1
            yield ("wait", raw_full[st], ph)

    def converter(w):
        rst = cst = rph = cph = 0
        for ch in chunks:
            yield ("wait", raw_full[rst], rph)
            yield ("wait", conv_empty[cst], cph if bug == "conv_parity" else cph ^ 1)
            if bug == "early_release":
                raw_empty[rst].arrive()
                yield ("step",)
            assert raw_slot[rst] == ch
            if w == 0:
                conv_slot[cst] = ch
            yield ("step",)
            if bug != "early_release":
                raw_empty[rst].arrive()
            conv_full[cst].arrive()
            rst, cst = rst + 1, cst + 1
            if rst == RS:
                rst, rph = 0, rph ^ 1
            if cst == CS:
                cst, cph = 0, cph ^ 1

    def mma():
        cst = tsl = cph = tph = 0
        for ch in chunks:
            yield ("wait", conv_full[cst], cph)
            yield ("wait", tempty[tsl], tph if bug == "tmem_parity" else tph ^ 1)
            assert conv_slot[cst] == ch
            tmem[tsl] = ch
            conv_empty[cst].arrive()
            tfull[tsl].arrive()
            cst, tsl = cst + 1, tsl + 1
            if cst == CS:
                cst, cph = 0, cph ^ 1
            if tsl == TS:
                tsl, tph = 0, tph ^ 1

    def epilogue(w):
        tsl = tph = 0
        for ch in chunks:
            if bug != "no_wait":
                yield ("wait", tfull[tsl], tph)
            assert tmem[tsl] == ch
            if w == 0:
                seen.append(ch)
            yield ("step",)
            tempty[tsl].arrive()
            tsl += 1
            if tsl == TS:
                tsl, tph = 0, tph ^ 1

    roles = [producer()] + [converter(w) for w in range(4)] + [mma()] + [epilogue(w) for w in range(4)]
    pending, done = [None] * len(roles), [False] * len(roles)
    rng = random.Random(seed)
    idle = 0
    while not all(done):
        order = list(range(len(roles)))
        rng.shuffle(order)
        moved = False
        for i in order:
            if done[i] or (pending[i] is not None and not pending[i][1].try_wait(pending[i][2])):
                continue
            pending[i] = None
            try:
                op = next(roles[i])
            except StopIteration:
                done[i] = True
                moved = True
                continue
            moved = True
            if op[0] == "wait":
                pending[i] = op
        idle = 0 if moved else idle + 1
        if idle > 3:
            raise RuntimeError("deadlock")
    assert seen == chunks


CASES = [[1], [3], [7], [8], [20], [3, 5], [7, 7, 7], [1] * 9, [20, 20, 20, 20], [80], [2, 13, 1, 6, 29]]


@pytest.mark.parametrize("units", CASES, ids=str)
def test_protocol_completes_and_every_read_sees_its_chunk(units):
    for seed in range(25):
        simulate(units, seed=seed)


@pytest.mark.parametrize("RS,CS,TS", [(1, 1, 1), (2, 1, 4), (7, 2, 1), (7, 2, 4), (3, 2, 2)])
def test_protocol_at_other_ring_depths(RS, CS, TS):
    for seed in range(10):
        simulate([5, 9, 1], RS, CS, TS, seed)


@pytest.mark.parametrize("bug", ["count", "phase", "conv_parity", "early_release", "tmem_parity", "no_wait"])
def test_planted_protocol_mistakes_are_caught(bug):
    caught = False
    for units in ([20], [3, 5], [80], [7, 7, 7]):
        for seed in range(30):
            try:
                simulate(units, seed=seed, bug=bug)
            except (AssertionError, RuntimeError):
                caught = True
                break
        if caught:
            break
    assert caught, bug


def test_converter_addressing_builds_the_swizzled_k_major_tile():
    """The converters' shared-memory writes, restated: lane l of converter warp w, pass it,
    takes raw row r = 32w + 4it + l/8, codes 16j..16j+15 with j = l % 8, and stores them as
    f16 chunks 2(j%4), 2(j%4)+1 of sub-tile j/4 at r*128 + ((chunk ^ (r % 8)) * 16).  Read back
    through the MMA's 128-byte-swizzle K-major rule, every code must sit at its (row, k), and
    each warp instruction must read 512 contiguous raw bytes."""
    BM, CK = 128, 128
    ids = [[r * CK + k for k in range(CK)] for r in range(BM)]
    conv = [None] * (2 * BM * 64)  # f16 elements of the two 64-column sub-tiles
    for w in range(4):
        for it in range(8):
            addrs = []
            for l in range(32):
                r, j = 32 * w + 4 * it + (l >> 3), l & 7
                addrs.append(r * CK + j * 16)
                base = (j >> 2) * BM * 64 + r * 64
                for half in range(2):
                    c = 2 * (j & 3) + half
                    for e in range(8):
                        conv[base + ((c ^ (r & 7)) * 8) + e] = ids[r][16 * j + 8 * half + e]
            addrs.sort()
            assert addrs == list(range(addrs[0], addrs[0] + 512, 16))
    for r in range(BM):
        for k in range(CK):
            c = (k % 64) // 8
            assert conv[(k // 64) * BM * 64 + r * 64 + ((c ^ (r % 8)) * 8) + k % 8] == ids[r][k]


def test_nvfp4_converter_addressing_builds_the_swizzled_k_major_tile():
    """NVFP4 tiles: a raw row is 128 bytes = 256 codes.  Lane l of converter warp w, pass it, holds
    raw bytes 16j..16j+15 (j = l % 8) of row r = 32w + 4it + l/8, i.e. codes 32j..32j+31.  Its raw
    word i (codes 32j+8i .. +7) becomes f16 chunk 4(j%2)+i of 64-column sub-tile j/2 at
    r*128 + ((chunk ^ (r % 8)) * 16); read back through the swizzle rule every code is at (r, k)."""
    BM, CK = 128, 256
    ids = [[r * CK + k for k in range(CK)] for r in range(BM)]
    conv = [None] * (4 * BM * 64)
    for w in range(4):
        for it in range(8):
            for l in range(32):
                r, j = 32 * w + 4 * it + (l >> 3), l & 7
                base = (j >> 1) * BM * 64 + r * 64
                for i in range(4):
                    ch = 4 * (j & 1) + i
                    for e in range(8):
                        conv[base + ((ch ^ (r & 7)) * 8) + e] = ids[r][32 * j + 8 * i + e]
    for r in range(BM):
        for k in range(CK):
            c = (k % 64) // 8
            assert conv[(k // 64) * BM * 64 + r * 64 + ((c ^ (r % 8)) * 8) + k % 8] == ids[r][k]
    # the MMA's block b (16 columns) is sub-tile b // 4, 16-column step b % 4
    for b in range(16):
        assert (b * 16) // 64 == b // 4 and ((b * 16) % 64) // 16 == b % 4
