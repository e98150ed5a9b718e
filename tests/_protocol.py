"""Pieces for randomized models of the kernels' barrier protocols (CPU tests).

A model restates a kernel's coordination from its code: each role (a loader, the MMA thread, a
warp of the softmax or the epilogue) is a Python generator that yields after each step, False
when it is blocked on a wait and True when it did something; `run` interleaves them at random.
"""


class Bar:
    """An mbarrier: `need` arrivals complete a phase; `count` phases have completed."""

    def __init__(self, name, need):
        self.name, self.need, self.arr, self.count = name, need, 0, 0

    def arrive(self):
        self.arr += 1
        assert self.arr <= self.need, f"{self.name}: more arrivals than the phase needs"
        if self.arr == self.need:
            self.arr, self.count = 0, self.count + 1

    def done(self, k):
        # a parity wait for phase k sees the phase bit only: it is right only while the barrier
        # is at phase k (not yet complete) or k + 1 (complete)
        assert self.count in (k, k + 1), f"{self.name}: waiter for phase {k} found {self.count} completed"
        return self.count == k + 1


def wait(bar, k):
    """A bounded-in-the-kernel parity wait for phase k of `bar`."""
    while not bar.done(k):
        yield False


class NamedBarrier:
    """A `bar.sync`-style barrier of `n` participants, reusable round after round."""

    def __init__(self, name, n):
        self.name, self.n, self.arrived, self.gen = name, n, 0, 0

    def sync(self):
        g = self.gen
        self.arrived += 1
        if self.arrived == self.n:
            self.arrived, self.gen = 0, self.gen + 1
        while self.gen == g:
            yield False


def run(roles, daemons, rnd, max_steps=400000):
    """Interleave `roles` (name -> generator, each must finish) and `daemons` (generators that
    serve forever) at random until every role has finished.  Fails on a deadlock: two polls of
    every role and daemon in a row with no progress."""
    live = dict(roles)
    idle = 0
    for _ in range(max_steps):
        if not live:
            return
        actors = list(live.items()) + [(None, d) for d in daemons]
        rnd.shuffle(actors)
        chosen = actors if idle else actors[: rnd.randint(1, len(actors))]
        progressed = False
        for name, gen in chosen:
            try:
                progressed |= bool(next(gen))
            except StopIteration:
                live.pop(name, None)
                progressed = True
        idle = 0 if progressed else idle + 1
        assert idle < 3, f"deadlock: {sorted(live)} wait"
    raise AssertionError(f"did not finish in {max_steps} steps: {sorted(live)}")
