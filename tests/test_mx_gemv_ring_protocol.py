"""The barrier protocol of the bulk-fed MXFP8 GEMV (csrc/mxfp8.cu,
k_mx_gemv_ring), model-checked on the CPU.

One CTA: a producer lane streams its units (8 weight rows each) into a ring
of 2 or 3 shared-memory stages by bulk copies (one copy of the whole unit
when a row is one run of K, else one copy a row), each completing its bytes
on the stage's full barrier; eight consumer warps stage the activations,
meet at a named barrier, then each takes one row of every unit and releases
the stage on its empty barrier (eight arrivals).  The producer waits for a
stage to empty before refilling it and, at the end, for its last copies.

Random schedules (copies landing in any order, at times of their own) must
finish, every consumer must read its row of the unit it expects with no copy
landing in the stage while any consumer reads it, every output row must be
written once, and a timeout of any wait must end every role with no copy in
flight at exit.  Planted mistakes must be caught.
"""
import random

import pytest

from protocol_model import Bar, Hazard, check, run_schedule

RPU = 8  # rows per unit = consumer warps


def simulate(n_units, stages, per_row, seed=0, timeout_at=None, bug=None):
    rng = random.Random(seed)
    full = [Bar(1, f"full{i}") for i in range(stages)]
    empty = [Bar(RPU - 1 if bug == "empty_count" else RPU, f"empty{i}") for i in range(stages)]
    staged = Bar(RPU, "x_staged")  # the consumers' named barrier after staging the activations
    st = {"abort": False}
    stage = [[None, set()] for _ in range(stages)]  # unit held, rows landed
    reading = [set() for _ in range(stages)]
    inflight, written = [], []

    def land(i):
        s, u, rows, bar = inflight.pop(i)
        check(not reading[s], f"stage {s} overwritten while warps {reading[s]} read unit {stage[s][0]}")
        if stage[s][0] != u:
            stage[s][:] = [u, set()]
        stage[s][1] |= rows
        bar.complete_tx(len(rows))

    def producer():
        i = 0
        for u in range(n_units):
            s = i % stages
            if i >= stages and bug != "no_empty_wait":
                par = (i // stages) & 1 if bug == "empty_parity" else ((i // stages) + 1) & 1
                ok = yield ("wait", empty[s], par)
                if not ok:
                    break
            full[s].arrive_expect_tx(RPU)
            if per_row:
                inflight.extend((s, u, {r}, full[s]) for r in range(RPU))
            else:
                inflight.append((s, u, set(range(RPU)), full[s]))
            i += 1
            yield ("step",)
        keep = 1 if bug == "drain_one" else stages
        for j in range(max(0, i - keep), i):
            yield ("drain", full[j % stages], (j // stages) & 1)

    def consumer(w):
        yield ("step",)  # activations into shared memory
        staged.arrive()
        yield ("drain", staged, 0)  # bar.sync: all consumer warps, not bounded
        for i in range(n_units):
            s = i % stages
            par = ((i // stages) + 1) & 1 if bug == "full_parity" else (i // stages) & 1
            ok = yield ("wait", full[s], par)
            if not ok:
                break
            check(stage[s][0] == i and w in stage[s][1], f"warp {w} reads stage {s} = {stage[s]} for unit {i}")
            reading[s].add(w)
            yield ("step",)
            written.append((i, w))
            reading[s].discard(w)
            empty[s].arrive()

    roles = [producer()] + [consumer(w) for w in range(RPU)]
    run_schedule(roles, lambda: [lambda i=i: land(i) for i in range(len(inflight))], rng, st, timeout_at)
    check(not inflight, f"copies still in flight at exit: {inflight}")
    if not st["abort"]:
        assert sorted(written) == [(u, w) for u in range(n_units) for w in range(RPU)]
    return st["abort"]


@pytest.mark.parametrize("stages", [2, 3])
@pytest.mark.parametrize("per_row", [False, True])
def test_ring_completes_and_every_read_sees_its_unit(stages, per_row):
    for n in (1, 2, 3, 4, 7, 12):
        for seed in range(15):
            assert not simulate(n, stages, per_row, seed=seed)


def test_a_timeout_anywhere_ends_every_role_cleanly():
    rng = random.Random(2)
    aborted = 0
    for t in range(300):
        aborted += simulate(rng.randint(1, 10), rng.choice([2, 3]), rng.random() < 0.5, seed=t,
                            timeout_at=rng.randint(1, 80))
    assert aborted > 150


@pytest.mark.parametrize("bug", ["empty_count", "no_empty_wait", "empty_parity", "full_parity", "drain_one"])
def test_planted_protocol_mistakes_are_caught(bug):
    rng = random.Random(4)
    for t in range(400):
        try:
            simulate(rng.randint(3, 10), rng.choice([2, 3]), rng.random() < 0.5, seed=t,
                     timeout_at=rng.randint(1, 80) if t % 3 == 0 else None, bug=bug)
        except (Hazard, RuntimeError, AssertionError):
            return
    pytest.fail(f"planted mistake {bug} not caught")
