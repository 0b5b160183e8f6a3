"""A small model of mbarrier protocols for CPU model checks of the kernels'
wait/arrive schemes.

Roles are generators that yield ("step",), ("wait", bar, parity) (a bounded
wait: it returns True once the phase has completed, False when the CTA's abort
flag is up or when the scheduler makes it time out) or ("drain", bar, parity)
(a teardown wait that ignores the abort flag).  Asynchronous units (a tensor
core running products in issue order, copies landing) are offered to the
scheduler as actions; in some runs they lag far behind the roles, which is
where a missing wait before exit shows.

The mbarrier model: a phase completes once all its arrivals are in and its
transaction bytes are all complete; try_wait.parity(p) succeeds when the
completed-phase count's parity differs from p.
"""


class Bar:
    def __init__(self, count, name):
        self.count, self.name = count, name
        self.arrived, self.tx, self.phase = 0, 0, 0

    def _complete(self):
        if self.arrived == self.count and self.tx == 0:
            self.arrived, self.phase = 0, self.phase + 1

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count, f"{self.name}: arrivals past the count"
        self._complete()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0, f"{self.name}: bytes completed that were never expected"
        self._complete()

    def try_wait(self, parity):
        return (self.phase & 1) != parity


class Hazard(AssertionError):
    pass


def check(cond, msg):
    if not cond:
        raise Hazard(msg)


def run_schedule(roles, async_actions, rng, st, timeout_at=None):
    """Run the roles to completion under a random schedule.

    async_actions(): the asynchronous units' actions enabled now (callables).
    st: a dict holding the CTA's abort flag under "abort".
    timeout_at: after this many scheduler steps the first wait still blocked
    gives up and raises the abort flag (None: no timeout).
    Raises RuntimeError on deadlock."""
    req = [("step",)] * len(roles)
    started = [False] * len(roles)
    done = [False] * len(roles)
    steps = 0
    lazy = rng.random() < 0.5
    while not all(done):
        steps += 1
        choices, blocked = [], []
        for i, r in enumerate(req):
            if done[i]:
                continue
            if r[0] == "step" or r[1].try_wait(r[2]):
                choices.append((i, True))
            elif r[0] == "wait" and st["abort"]:
                choices.append((i, False))
            elif r[0] == "wait":
                blocked.append(i)
        if timeout_at is not None and steps >= timeout_at and blocked and not st["abort"]:
            st["abort"] = True
            choices = [(rng.choice(blocked), False)]
        acts = []
        if not choices or not lazy or rng.random() < 0.05:
            acts = async_actions()
        if not choices and not acts:
            raise RuntimeError(f"deadlock: {[r[:1] + (r[1].name,) if len(r) > 1 else r for r in req]}")
        c = rng.randrange(len(choices) + len(acts))
        if c >= len(choices):
            acts[c - len(choices)]()
            continue
        i, res = choices[c]
        try:
            req[i] = roles[i].send(res if req[i][0] == "wait" else None) if started[i] else next(roles[i])
            started[i] = True
        except StopIteration:
            done[i] = True
