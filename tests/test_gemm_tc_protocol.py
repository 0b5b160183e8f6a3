"""The barrier protocol of the tcgen05 GEMM (csrc/gemm_tc.cu, k_gemm_tc),
model-checked on the CPU.

One CTA runs a list of work units (weight tile, token tile, K split), each a
run of k-blocks.  Roles, each restated as a state machine:
- the TMA producer lane: fills the first STAGES stages with weight (A) tiles
  before the predecessor grid is waited for and adds the token (B) tiles
  after (all on the stage's one expect-tx arrival), then refills a stage once
  the MMA lane has released it, and at the end waits for the last
  min(issued, STAGES) fills, walking back over the ring;
- the MMA lane: per unit waits for a free accumulator (two, double-buffered
  in tensor memory), per k-block waits for the stage, issues the products,
  commits the stage's release; commits the accumulator when the unit ends,
  and before exit commits and waits for a final barrier;
- four epilogue warps: (with an operand stage, first build the resident B
  operand and signal it) per unit wait for the accumulator, read it, release
  it with one arrival a warp.

The tensor core runs the lane's products and commits in issue order at times
of its own choosing; each copy lands whenever it likes.  Random schedules
must finish, every product must read a stage holding both tiles of its
k-block, no copy may land in a stage a queued product reads, every
accumulator the epilogue reads must hold exactly its unit's k-blocks with no
product adding to it, and a timeout of any wait at any moment must leave no
copy in flight and no product queued at exit.  Planted mistakes must be
caught.
"""
import random

import pytest

from protocol_model import Bar, Hazard, check, run_schedule


def simulate(units, STAGES, prep=False, seed=0, timeout_at=None, bug=None):
    """units: k-blocks of each unit this CTA runs, in order."""
    rng = random.Random(seed)
    items = [(u, kb) for u, n in enumerate(units) for kb in range(n)]
    full = [Bar(1, f"full{i}") for i in range(STAGES)]
    empty = [Bar(1, f"empty{i}") for i in range(STAGES)]
    tfull = [Bar(1, f"tfull{i}") for i in range(2)]
    tempty = [Bar(3 if bug == "tempty_count" else 4, f"tempty{i}") for i in range(2)]
    mma_done = Bar(1, "mma_done")
    b_ready = Bar(1, "b_ready")
    epi_bar = Bar(4, "epilogue named barrier")
    st = {"abort": False}
    stage = [[None, set()] for _ in range(STAGES)]  # item held, tiles landed ('A', 'B')
    acc = [[None, []] for _ in range(2)]              # unit, k-blocks summed
    queue, inflight, read = [], [], []
    breg = {"ready": False}

    def pending_stage(s):
        return any(op[0] == "mma" and op[1] == s for op in queue)

    def pending_acc(a):
        return any(op[0] == "mma" and op[2] == a for op in queue)

    def land(i):
        s, it, tile, bar = inflight.pop(i)
        check(not pending_stage(s), f"stage {s} overwritten while a product reads it")
        if stage[s][0] != it:
            stage[s][:] = [it, set()]
        stage[s][1].add(tile)
        bar.complete_tx(1)

    def tensor_core_step():
        op = queue.pop(0)
        if op[0] == "mma":
            _, s, a, (u, kb) = op
            check(stage[s][0] == (u, kb), f"product of {(u, kb)} reads stage {s} = {stage[s]}")
            check(stage[s][1] == ({"A"} if prep else {"A", "B"}), f"stage {s} incomplete: {stage[s]}")
            if prep:
                check(breg["ready"], "product reads the resident operand before it is built")
            if kb == 0:
                acc[a] = [u, []]
            check(acc[a][0] == u and acc[a][1] == list(range(kb)), f"accumulator {a} = {acc[a]} at {(u, kb)}")
            acc[a][1].append(kb)
        else:
            op[1].arrive()

    def producer():
        npre, pre = 0, []
        while npre < STAGES and npre < len(items):
            full[npre].arrive_expect_tx(1 if prep else 2)
            inflight.append((npre, items[npre], "A", full[npre]))
            pre.append(npre)
            npre += 1
        yield ("step",)  # the predecessor grid
        if not prep:
            for i in pre:
                inflight.append((i, items[i], "B", full[i]))
        s, phase, issued = npre % STAGES, 1 if npre == STAGES else 0, npre
        for it in items[npre:]:
            ok = yield ("wait", empty[s], phase if bug == "empty_parity" else phase ^ 1)
            if not ok:
                break
            issued += 1
            full[s].arrive_expect_tx(1 if prep else 2)
            inflight.append((s, it, "A", full[s]))
            if not prep:
                inflight.append((s, it, "B", full[s]))
            s += 1
            if s == STAGES:
                s, phase = 0, phase ^ 1
            yield ("step",)
        # walk back over the last min(issued, STAGES) fills
        for _ in range(min(issued, 1 if bug == "drain_one" else STAGES)):
            if s == 0:
                s, phase = STAGES, phase ^ 1
            s -= 1
            yield ("drain", full[s], phase)

    def mma():
        s = a = 0
        phase = aph = 0
        ok = True
        if prep:
            ok = yield ("wait", b_ready, 0)
            ok = ok and not st["abort"]
        k = 0
        for u, n in enumerate(units):
            if not ok:
                break
            if bug != "no_tempty_wait":
                ok = yield ("wait", tempty[a], aph ^ 1)
                if not ok:
                    break
            for kb in range(n):
                ok = yield ("wait", full[s], phase)
                if not ok:
                    break
                queue.append(("mma", s, a, items[k]))
                k += 1
                if bug != "no_release":
                    queue.append(("commit", empty[s]))
                s += 1
                if s == STAGES:
                    s, phase = 0, phase ^ 1
            if not ok:
                break
            queue.append(("commit", tfull[a]))
            a += 1
            if a == 2:
                a, aph = 0, aph ^ 1
        queue.append(("commit", mma_done))
        if bug != "no_mma_drain":
            yield ("drain", mma_done, 0)

    def epilogue(w):
        if prep:
            yield ("step",)  # this warp's part of the operand
            epi_bar.arrive()
            yield ("drain", epi_bar, 0)  # bar.sync of the 128 epilogue threads
            if w == 0:
                breg["ready"] = True
                b_ready.arrive()
        a = aph = 0
        for u, n in enumerate(units):
            ok = yield ("wait", tfull[a], aph)
            if not ok:
                break
            check(not pending_acc(a), f"accumulator {a} read while a product adds to it")
            check(acc[a] == [u, list(range(n))], f"warp {w} reads accumulator {a} = {acc[a]} for unit {u}")
            yield ("step",)
            read.append((u, w))
            tempty[a].arrive()
            a += 1
            if a == 2:
                a, aph = 0, aph ^ 1

    def async_actions():
        acts = [tensor_core_step] if queue else []
        return acts + [lambda i=i: land(i) for i in range(len(inflight))]

    roles = [producer(), mma()] + [epilogue(w) for w in range(4)]
    run_schedule(roles, async_actions, rng, st, timeout_at)
    check(not queue, f"products still queued at exit: {queue}")
    check(not inflight, f"copies still in flight at exit: {inflight}")
    if not st["abort"]:
        assert sorted(read) == [(u, w) for u in range(len(units)) for w in range(4)]
    return st["abort"]


CASES = [[1], [4], [1, 1, 1], [3, 2], [2, 2, 2, 2, 2], [5, 1, 4], [8], [1] * 7]


@pytest.mark.parametrize("STAGES", [2, 3, 4, 6])
@pytest.mark.parametrize("prep", [False, True])
def test_gemm_completes_and_every_read_sees_its_tiles(STAGES, prep):
    for units in CASES:
        for seed in range(8):
            assert not simulate(units, STAGES, prep, seed=seed)


def test_a_timeout_anywhere_ends_every_role_cleanly():
    rng = random.Random(9)
    aborted = 0
    for t in range(400):
        units = [rng.randint(1, 5) for _ in range(rng.randint(1, 5))]
        aborted += simulate(units, rng.choice([2, 3, 4, 6]), rng.random() < 0.3, seed=t,
                            timeout_at=rng.randint(1, 100))
    assert aborted > 200


@pytest.mark.parametrize("bug", ["tempty_count", "empty_parity", "drain_one", "no_tempty_wait", "no_release",
                                 "no_mma_drain"])
def test_planted_protocol_mistakes_are_caught(bug):
    rng = random.Random(6)
    for t in range(600):
        units = [rng.randint(1, 5) for _ in range(rng.randint(2, 6))]
        try:
            simulate(units, rng.choice([2, 3, 4]), rng.random() < 0.3, seed=t,
                     timeout_at=rng.randint(1, 100) if t % 3 == 0 else None, bug=bug)
        except (Hazard, RuntimeError, AssertionError):
            return
    pytest.fail(f"planted mistake {bug} not caught")
