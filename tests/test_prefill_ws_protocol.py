"""The barrier protocol of the warp-specialised prefill attention
(csrc/attn_prefill_ws.cu), model-checked on the CPU.

The kernel's roles, each restated as a state machine:
- the loader warp (Q once, then K and V tiles into a ring of NS stages, by TMA
  or row by row, then a drain of its copies in flight);
- the MMA lane (S_q = Q_q K^T and O_q += P_q V per slot, commits);
- four softmax warps per query slot (read S_q, rescale O_q, write P_q over
  S_q, arrive; then the epilogue reads O_q).

The asynchronous units are modelled too: the tensor core runs the MMA lane's
products and commits in issue order at times of its own choosing, and each
TMA copy lands (and completes its bytes on the stage's barrier) whenever it
likes (the barrier model is in protocol_model.py).

Random schedules over random slot geometries must finish without deadlock,
every read (of shared-memory stages, of S, P and O in tensor memory) must see
what its reader expects with no product in flight that writes it, and a
timeout of any wait at any moment must end every role with no copy landing
and no product running after the CTA frees its tensor memory.  Planted
protocol mistakes must be caught.
"""
import random

import pytest

from protocol_model import Bar, Hazard, check, run_schedule

TK = 128
WARPS = 4  # softmax warps per slot; each arrives with its 32 lanes at once


def simulate(n_tiles, ranges, paths, NS=2, seed=0, timeout_at=None, bug=None):
    """One CTA.  ranges[q] = (a, b): key tiles slot q reads (relative to the
    first tile).  paths[j]: 'tma' or 'rows' for key tile j.  timeout_at: the
    number of scheduler steps after which the first wait still blocked gives
    up (None: no timeout).  Returns (aborted, outputs)."""
    nslot = len(ranges)
    rng = random.Random(seed)
    q_full = Bar(1, "q_full")
    k_full = [Bar(1, f"k_full{i}") for i in range(NS)]
    v_full = [Bar(1, f"v_full{i}") for i in range(NS)]
    k_empty = [Bar(1, f"k_empty{i}") for i in range(NS)]
    v_empty = [Bar(1, f"v_empty{i}") for i in range(NS)]
    s_full = [Bar(1, f"s_full{q}") for q in range(2)]
    p_full = [Bar(WARPS - 1 if bug == "p_count" else WARPS, f"p_full{q}") for q in range(2)]
    o_full = Bar(1, "o_full")
    st = {"abort": False}

    # shared memory: stage -> [tile, halves landed]; Q slot -> halves landed
    smem_k = [[None, 0] for _ in range(NS)]
    smem_v = [[None, 0] for _ in range(NS)]
    smem_q = [0, 0]
    # tensor memory: S_q holds the scores of one tile; P_q[w] the tile whose
    # probabilities warp w wrote over its lanes of S_q; O_q the tiles summed
    S = [None, None]
    P = [[None] * WARPS for _ in range(2)]
    O = [[] for _ in range(2)]
    queue, inflight, outputs = [], [], {}

    def pending(kind, q=None, stage=None):
        return any(op[0] == kind and (q is None or op[1] == q) and (stage is None or op[2] == stage)
                   for op in queue)

    def write_stage(kind, stage, tile, halves):
        reader = "S" if kind == "k" else "PV"
        check(not pending(reader, stage=stage), f"{kind} stage {stage} overwritten while a product reads it")
        buf = smem_k if kind == "k" else smem_v
        if buf[stage][0] != tile:
            buf[stage][:] = [tile, 0]
        buf[stage][1] += halves

    # -------------------------------------------------------------- roles
    def loader():
        q_full.arrive_expect_tx(2 * nslot)
        for q in range(nslot):
            for h in range(2):
                inflight.append(("q", q, h, q_full))
        issued, ok = 0, True
        for j in range(n_tiles):
            s, use = j % NS, j // NS
            if j >= NS and bug != "loader_no_k_wait":
                ok = yield ("wait", k_empty[s], (use + 1) & 1)
                if not ok:
                    break
            if j >= NS and bug != "loader_no_v_wait":
                ok = yield ("wait", v_empty[s], (use + 1) & 1)
                if not ok:
                    break
            if paths[j] == "tma":
                k_full[s].arrive_expect_tx(2)
                inflight.extend([("k", s, j, k_full[s])] * 2)
                v_full[s].arrive_expect_tx(2)
                inflight.extend([("v", s, j, v_full[s])] * 2)
            else:  # row copies, waited for before the arrivals
                write_stage("k", s, j, 2)
                yield ("step",)
                write_stage("v", s, j, 2)
                yield ("step",)
                k_full[s].arrive()
                v_full[s].arrive()
            issued = j + 1
            yield ("step",)
        # copies still in flight land before the CTA can exit
        yield ("drain", q_full, 0)
        keep = 1 if bug == "drain_one" else NS
        for j in range(max(0, issued - keep), issued):
            yield ("drain", k_full[j % NS], (j // NS) & 1)
            yield ("drain", v_full[j % NS], (j // NS) & 1)

    def mma():
        def s_mma(q, s, j):
            queue.append(("S", q, s, j))
            queue.append(("commit", q, None, s_full[q]))

        ok = yield ("wait", q_full, 0)
        if ok:
            ok = yield ("wait", k_full[0], 0)
        if ok:
            for q in range(nslot):
                if ranges[q][0] == 0:
                    s_mma(q, 0, 0)
            queue.append(("commit", None, None, k_empty[0]))
        j = 0
        while ok and j < n_tiles:
            s = j % NS
            ok = yield ("wait", v_full[s], (j // NS) & 1)
            if not ok:
                break
            j1 = j + 1
            s1 = j1 % NS
            if bug == "early_v_empty":
                queue.append(("commit", None, None, v_empty[s]))
            k_next = False
            for q in range(nslot):
                a, b = ranges[q]
                if bug == "s_before_pv" and a <= j1 <= b:
                    if not k_next:
                        ok = yield ("wait", k_full[s1], (j1 // NS) & 1)
                        if not ok:
                            break
                        k_next = True
                    s_mma(q, s1, j1)
                if a <= j <= b:
                    if bug != "no_p_wait":
                        ok = yield ("wait", p_full[q], (j - a) & 1)
                        if not ok:
                            break
                    queue.append(("PV", q, s, j))
                if bug != "s_before_pv" and a <= j1 <= b:
                    if not k_next:
                        ok = yield ("wait", k_full[s1], (j1 // NS) & 1)
                        if not ok:
                            break
                        k_next = True
                    s_mma(q, s1, j1)
            if not ok:
                break
            if bug != "early_v_empty":
                queue.append(("commit", None, None, v_empty[s]))
            if j1 < n_tiles:
                queue.append(("commit", None, None, k_empty[s1]))
            j += 1
        queue.append(("commit", None, None, o_full))
        if bug != "no_o_drain":
            yield ("drain", o_full, 0)  # no product may still write TMEM when it is freed

    def softmax(q, w):
        a, b = ranges[q]
        ok = True
        for j in range(a, b + 1):
            par = (j - a + 1) & 1 if bug == "softmax_parity" else (j - a) & 1
            ok = yield ("wait", s_full[q], par)
            if not ok:
                break
            check(S[q] == j and P[q][w] is None, f"slot {q} warp {w} reads S of tile {S[q]} (P {P[q][w]}) at {j}")
            check(not pending("S", q), f"slot {q}: S read while a product writes it")
            yield ("step",)
            if j > a:  # rescale O (read, scale, write back)
                check(O[q] == list(range(a, j)), f"slot {q}: O holds {O[q]} when rescaled at {j}")
                check(not pending("PV", q), f"slot {q}: O rescaled while a product adds to it")
                yield ("step",)
            check(not pending("PV", q), f"slot {q}: P written while a product reads the old P")
            P[q][w] = j
            yield ("step",)
            p_full[q].arrive()
        if ok:
            ok = yield ("wait", o_full, 0)
            if ok:
                check(not pending("PV", q), f"slot {q}: O read while a product adds to it")
                if not st["abort"]:
                    check(O[q] == list(range(a, b + 1)), f"slot {q}: epilogue reads O of {O[q]}")
                outputs[(q, w)] = list(O[q])

    # ------------------------------------------------------- async units
    def tensor_core_step():
        op = queue.pop(0)
        kind, q, s, j = op
        if kind == "S":
            check(smem_q[q] == 2, f"S of slot {q} before Q landed")
            check(smem_k[s] == [j, 2], f"S of slot {q} tile {j} reads K stage {s} = {smem_k[s]}")
            a = ranges[q][0]
            if j > a:  # the products of the previous tile have used its P
                check(O[q] and O[q][-1] == j - 1, f"slot {q}: S of tile {j} overwrites P before P V of {j - 1}")
            S[q] = j
            P[q] = [None] * WARPS
        elif kind == "PV":
            check(all(p == j for p in P[q]), f"slot {q}: P V of tile {j} reads P {P[q]}")
            check(smem_v[s] == [j, 2], f"P V of slot {q} tile {j} reads V stage {s} = {smem_v[s]}")
            check(O[q] == list(range(ranges[q][0], j)), f"slot {q}: O {O[q]} before adding tile {j}")
            O[q].append(j)
        else:
            j.arrive()  # the commit's barrier

    def land(i):
        kind, s, j, bar = inflight.pop(i)
        if kind == "q":
            smem_q[s] += 1
        else:
            write_stage(kind, s, j, 1)
        bar.complete_tx(1)

    # -------------------------------------------------------- scheduler
    def async_actions():
        acts = [tensor_core_step] if queue else []
        return acts + [lambda i=i: land(i) for i in range(len(inflight))]

    roles = [loader(), mma()] + [softmax(q, w) for q in range(nslot) for w in range(WARPS)]
    run_schedule(roles, async_actions, rng, st, timeout_at)
    # the CTA frees TMEM and exits: nothing may still run
    check(not queue, f"products still queued at exit: {queue}")
    check(not inflight, f"copies still in flight at exit: {inflight}")
    return st["abort"], outputs


def slot_range(pf, pl, window):
    """Key tiles a query rows pf..pl read (the kernel's per-slot geometry)."""
    lo = max(0, pf - window + 1) if window > 0 else 0
    return lo // TK, pl // TK


def item(slots, window):
    """Relative ranges and tile count of a work item from its slots' first and
    last positions, as the kernel derives them."""
    r = [slot_range(pf, pl, window) for pf, pl in slots]
    lo, hi = min(a for a, _ in r), max(b for _, b in r)
    return hi - lo + 1, [(a - lo, b - lo) for a, b in r]


ITEMS = [
    item([(0, 127)], 0),                        # one slot, one tile
    item([(0, 127), (0, 127)], 0),              # two heads on the same rows
    item([(512, 639), (512, 639)], 0),          # full attention: 5 tiles each
    item([(384, 511), (512, 639)], 0),          # odd head on consecutive row tiles
    item([(384, 511), (512, 639)], 160),        # sliding window: ranges overlap in part
    item([(1000, 1127), (1128, 1255)], 160),
    item([(4096, 4223), (4224, 4351)], 4096),   # 4B window
    item([(300, 427)], 160),
    item([(0, 4)], 0),                          # a 5-row tile
]


def random_item(rng):
    n = rng.randint(1, 7)
    r = []
    for _ in range(rng.choice([1, 2])):
        a = rng.randrange(n)
        r.append((a, rng.randrange(a, n)))
    lo, hi = min(a for a, _ in r), max(b for _, b in r)
    return hi - lo + 1, [(a - lo, b - lo) for a, b in r]


def paths_for(rng, n):
    return [rng.choice(["tma", "rows"]) for _ in range(n)]


@pytest.mark.parametrize("k", range(len(ITEMS)))
def test_items_complete_and_every_read_sees_its_tile(k):
    n, ranges = ITEMS[k]
    for seed in range(40):
        rng = random.Random(seed)
        aborted, out = simulate(n, ranges, paths_for(rng, n), seed=seed)
        assert not aborted
        assert len(out) == WARPS * len(ranges)


def test_random_geometries_and_ring_depths():
    rng = random.Random(7)
    for t in range(300):
        n, ranges = random_item(rng)
        aborted, out = simulate(n, ranges, paths_for(rng, n), NS=rng.choice([2, 3]), seed=t)
        assert not aborted and len(out) == WARPS * len(ranges)


def test_one_stage_ring_deadlocks():
    """The MMA lane waits for K of tile j+1 while V of tile j is still in use,
    so the ring needs two stages: with one, the loader waits for V's stage to
    empty and the MMA lane for the next K, for good."""
    with pytest.raises(RuntimeError, match="deadlock"):
        simulate(2, [(0, 1)], ["tma", "tma"], NS=1)


def test_a_timeout_anywhere_ends_every_role_cleanly():
    """A wait that gives up at any moment sets the abort flag; every role then
    stops, the loader waits for its copies and the MMA lane for its products,
    so nothing lands or runs after the CTA frees tensor memory."""
    rng = random.Random(11)
    n_abort = 0
    for t in range(400):
        n, ranges = random_item(rng) if t % 2 else ITEMS[t // 2 % len(ITEMS)]
        aborted, _ = simulate(n, ranges, paths_for(rng, n), seed=t, timeout_at=rng.randint(1, 120))
        n_abort += aborted
    assert n_abort > 200  # most runs had a wait blocked at the chosen moment


BUGS = ["p_count", "loader_no_v_wait", "drain_one", "early_v_empty", "s_before_pv", "no_p_wait",
        "softmax_parity", "no_o_drain"]


@pytest.mark.parametrize("bug", BUGS)
def test_planted_protocol_mistakes_are_caught(bug):
    rng = random.Random(3)
    for t in range(400):
        n, ranges = random_item(rng) if t % 2 else ITEMS[t // 2 % len(ITEMS)]
        if n < 2:
            continue
        timeout_at = rng.randint(1, 120) if t % 3 == 0 else None
        try:
            simulate(n, ranges, paths_for(rng, n), seed=t, timeout_at=timeout_at, bug=bug)
        except (Hazard, RuntimeError, AssertionError):
            return
    pytest.fail(f"planted mistake {bug} not caught")


def test_p_columns_and_v_rows_meet_at_the_same_keys():
    """The softmax writes the probability of key 32h + c (c < 32) as the low
    (c even) or high half of TMEM column 16h + c/2 of S_q; the P V product's
    step kk reads columns 8kk .. 8kk+7 as the A operand (16 keys) and V rows
    (keys) at byte offset 2048 kk of the stage, 128 bytes a key.  Every key's
    probability must meet that key's V row in the same step and position."""
    col_of = {}
    for h in range(4):
        for c in range(32):
            col_of[32 * h + c] = (16 * h + c // 2, c & 1)
    for kk in range(TK // 16):
        for e in range(16):  # the e-th key of the step's K = 16 slice
            key_a = None
            for key, (col, half) in col_of.items():
                if col == 8 * kk + e // 2 and half == e % 2:
                    key_a = key
            v_row = (2048 * kk + 128 * e) // 128
            assert key_a == v_row == 16 * kk + e


def test_k_empty_wait_is_implied_by_v_empty_wait():
    """The V release of tile j is committed after the S product of every slot
    that reads K of tile j, so a loader waiting only for V's stage to empty
    would still never overwrite K in use."""
    rng = random.Random(5)
    for t in range(300):
        n, ranges = random_item(rng)
        simulate(n, ranges, paths_for(rng, n), NS=rng.choice([2, 3]), seed=t,
                 timeout_at=rng.randint(1, 120) if t % 3 == 0 else None, bug="loader_no_k_wait")
