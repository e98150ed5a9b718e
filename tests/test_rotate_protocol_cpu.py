"""A randomized model of the barrier protocol of the persistent rotate + block-quantize kernel.

`rotate_block_quant_kernel` (csrc/rotate.cu) walks its work items (operand, batch, head,
256-token chunk) in operand order.  A producer warp loads each item's input tiles into one of two
shared-memory stages (and, when the operand changes, that operand's rotation R into its single
buffer, by TMA or generated from signs); one MMA thread rotates the stage into one of two TMEM
buffers; sixteen epilogue warps read TMEM (or, for an operand without rotation, the stage
itself), reduce block maxima behind a named barrier, stage the codes and store them with TMA.

This file restates that protocol from the kernel's code (barriers, arrival counts, phases,
buffer indices, the rotation reload and the staging reuse) and interleaves the roles at random.
It does not run the kernel.  It checks progress, parity (every wait finds its barrier at the
phase waited for or one past it) and data hazards: a stage, the rotation buffer, a TMEM buffer
or a staging tile is not rewritten while a queued MMA, an epilogue warp or a store still reads
it, and each reader finds the item it expects.
"""
import random

import pytest
from _protocol import Bar, NamedBarrier, run, wait

NEPI = 16  # epilogue warps: 2 tiles x 4 TMEM lane quarters x 2 column parts


class Item:
    def __init__(self, oi, rotate, ntile):
        self.oi, self.rotate, self.ntile = oi, rotate, ntile


class Model:
    def __init__(self, items, generated_r, rnd):
        self.items, self.generated_r, self.rnd = items, generated_r, rnd
        self.XF = [Bar(f"XF{i}", 1) for i in range(2)]
        self.XE = [Bar(f"XE{i}", NEPI) for i in range(2)]
        self.TF = [Bar(f"TF{i}", 1) for i in range(2)]
        self.TE = [Bar(f"TE{i}", NEPI) for i in range(2)]
        self.RF = Bar("RF", 1)
        self.RE = Bar("RE", 1)
        self.FIN = Bar("FIN", 1)
        self.nb_max = NamedBarrier("NB_MAX", NEPI)
        self.nb_code = [NamedBarrier(f"NB_CODE{u}", NEPI // 2) for u in range(2)]
        self.X = [None, None]          # item held by each input stage
        self.x_readers = [set(), set()]
        self.R = None                  # operand whose rotation the buffer holds
        self.T = [None, None]          # item held by each TMEM buffer
        self.t_reads = [NEPI, NEPI]    # epilogue warps that have read it
        self.staging = [None, None]    # item whose codes each staging tile holds
        self.stores = []               # stores in flight: (tile, item)
        self.pipe, self.inflight = [], []

    def queued(self, pred):
        return any(op[0] == "mma" and pred(op) for op in self.pipe)

    # ------------------------------------------------------------------ roles
    def producer(self):
        rload, rop = 0, -1
        for k, it in enumerate(self.items):
            st = k & 1
            if k >= 2:
                yield from wait(self.XE[st], (k >> 1) - 1)
            if it.rotate and it.oi != rop:
                if rload > 0:
                    yield from wait(self.RE, rload - 1)
                assert not self.queued(lambda op: True), "rotation rewritten under a queued MMA"
                if self.generated_r:
                    self.R = it.oi
                    self.RF.arrive()
                else:
                    self.R = ("loading", it.oi)
                    self.inflight.append((self.RF, "R", it.oi))
                rload, rop = rload + 1, it.oi
            assert not self.queued(lambda op: op[2] == st), "input stage rewritten under a queued MMA"
            assert not self.x_readers[st], "input stage rewritten under an epilogue read"
            self.X[st] = ("loading", k)
            self.inflight.append((self.XF[st], "X", (st, k)))
            yield True

    def engine(self):
        """TMA loads and stores complete in any order."""
        while True:
            if not self.inflight and not self.stores:
                yield False
                continue
            if self.stores and (not self.inflight or self.rnd.random() < 0.5):
                self.stores.pop(self.rnd.randrange(len(self.stores)))
                yield True
                continue
            bar, what, val = self.inflight.pop(self.rnd.randrange(len(self.inflight)))
            if what == "R":
                self.R = val
            else:
                self.X[val[0]] = val[1]
            bar.arrive()
            yield True

    def tensor_pipe(self):
        while True:
            if not self.pipe:
                yield False
                continue
            op = self.pipe.pop(0)
            if op[0] == "commit":
                op[1].arrive()
            else:
                _, k, st, tb, oi = op
                assert self.X[st] == k, f"MMA of item {k} found stage {st} holding {self.X[st]}"
                assert self.R == oi, f"MMA of item {k} found rotation {self.R}"
                assert self.t_reads[tb] == NEPI, f"TMEM buffer {tb} rewritten before every warp read it"
                self.T[tb], self.t_reads[tb] = k, 0
            yield True

    def mma(self):
        tuse, rwait, rop = [0, 0], 0, -1
        for k, it in enumerate(self.items):
            if not it.rotate:
                continue
            if it.oi != rop:
                if rop >= 0:
                    self.pipe.append(("commit", self.RE))
                yield from wait(self.RF, rwait)
                rwait, rop = rwait + 1, it.oi
            st = tb = k & 1
            yield from wait(self.XF[st], k >> 1)
            if tuse[tb] > 0:
                yield from wait(self.TE[tb], tuse[tb] - 1)
            self.pipe.append(("mma", k, st, tb, it.oi))
            self.pipe.append(("commit", self.TF[tb]))
            tuse[tb] += 1
            yield True
        self.pipe.append(("commit", self.FIN))
        yield from wait(self.FIN, 0)

    def epilogue(self, e):
        u = e // 8
        issuer = e % 8 == 0  # lane 0 of each tile's first warp stores the tile's codes
        tuse = [0, 0]
        for k, it in enumerate(self.items):
            st = k & 1
            if it.rotate:
                tb = k & 1
                yield from wait(self.TF[tb], tuse[tb])
                tuse[tb] += 1
                assert self.T[tb] == k, f"epilogue {e} read TMEM buffer {tb} holding {self.T[tb]} for item {k}"
                self.t_reads[tb] += 1
                self.TE[tb].arrive()
                self.XE[st].arrive()
            else:
                yield from wait(self.XF[st], k >> 1)
                self.x_readers[st].add(e)
                assert self.X[st] == k, f"epilogue {e} read stage {st} holding {self.X[st]} for item {k}"
                yield True
                self.x_readers[st].discard(e)
                self.XE[st].arrive()
            if issuer:  # the previous store must have read the staging tile
                while any(t == u for t, _ in self.stores):
                    yield False
            yield from self.nb_max.sync()
            if u >= it.ntile:
                continue
            assert not any(t == u for t, _ in self.stores), "staging tile rewritten under a store"
            self.staging[u] = k
            yield True
            yield from self.nb_code[u].sync()
            if issuer:
                assert self.staging[u] == k
                self.stores.append((u, k))
            yield True
        if issuer:
            while any(t == u for t, _ in self.stores):
                yield False

    def run(self):
        roles = {"producer": self.producer(), "mma": self.mma()}
        for e in range(NEPI):
            roles[f"e{e}"] = self.epilogue(e)
        run(roles, [self.engine(), self.tensor_pipe()], self.rnd)
        assert not self.pipe and not self.inflight and not self.stores


def random_items(rnd, rotate):
    """A CTA's items: operands in order (Q, K, V), each with 0-5 chunks, ragged last chunks."""
    items = []
    for oi in range(3):
        for _ in range(rnd.randint(0, 5)):
            items.append(Item(oi, rotate[oi], rnd.choice((1, 2, 2))))
    return items


@pytest.mark.parametrize("rotate", [(True, True, False), (True, True, True), (False, False, False),
                                    (True, False, True)])
@pytest.mark.parametrize("generated_r", [False, True])
def test_rotate_kernel_protocol(rotate, generated_r):
    for seed in range(150):
        rnd = random.Random(seed * 7 + sum(rotate) + 10 * generated_r)
        items = random_items(rnd, rotate)
        if items:
            Model(items, generated_r, rnd).run()


def test_model_catches_a_rotation_reloaded_without_its_wait():
    """A rotation loaded for the next operand without waiting for the MMAs that read the previous
    one (the wait on the release barrier left out) is caught."""

    class NoRelease(Model):
        def producer(self):
            rop = -1
            for k, it in enumerate(self.items):
                st = k & 1
                if k >= 2:
                    yield from wait(self.XE[st], (k >> 1) - 1)
                if it.rotate and it.oi != rop:
                    self.R = ("loading", it.oi)
                    self.inflight.append((self.RF, "R", it.oi))
                    rop = it.oi
                self.X[st] = ("loading", k)
                self.inflight.append((self.XF[st], "X", (st, k)))
                yield True

    caught = 0
    for seed in range(400):
        rnd = random.Random(seed)
        items = [Item(0, True, 2)] * 3 + [Item(1, True, 2)] * 3
        try:
            NoRelease(items, False, rnd).run()
        except AssertionError as e:
            assert "rotation" in str(e), str(e)
            caught += 1
    assert caught > 0


def test_model_catches_an_input_stage_released_early():
    """An epilogue warp that releases the input stage of a rotated item before the MMA that read it
    has completed (its release moved above the wait for the TMEM buffer) is caught."""

    class Early(Model):
        def epilogue(self, e):
            u = e // 8
            tuse = [0, 0]
            for k, it in enumerate(self.items):
                st = k & 1
                if it.rotate:
                    self.XE[st].arrive()  # released before the MMA is known to be done
                    tb = k & 1
                    yield from wait(self.TF[tb], tuse[tb])
                    tuse[tb] += 1
                    self.t_reads[tb] += 1
                    self.TE[tb].arrive()
                else:
                    yield from wait(self.XF[st], k >> 1)
                    self.XE[st].arrive()
                yield from self.nb_max.sync()

    caught = 0
    for seed in range(60):
        rnd = random.Random(seed)
        try:
            Early([Item(0, True, 2)] * 6, False, rnd).run()
        except AssertionError:
            caught += 1
    assert caught > 0
