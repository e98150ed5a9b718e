"""A randomized model of the barrier protocol of the two-query-tile prefill kernel.

The kernel (`attn_pair_kernel`, csrc/attn2.cu) coordinates its roles through mbarriers only:
a K loader, a V' loader and a scale-ring loader (TMA / bulk copies), one MMA thread that issues
Q·Kᵀ, P·V and (for the MX kinds) the copies of the K tiles' scale-factor atoms into TMEM, the
tensor pipe that runs them in issue order and signals completions through commits, and two
softmax warpgroups of four warps.  Every wait is a parity wait, so a waiter must never find its
barrier two phases ahead (or a phase behind) of the phase it waits for.

This file restates that protocol from the kernel's code: the same barriers, arrival counts,
phases, ring depths and issue order, with each role as a coroutine and a scheduler that
interleaves them at random.  It does not run the kernel.  It checks, over many interleavings and
key-tile counts per query tile:
- progress: every role finishes (no wait is left without the arrival it needs);
- parity: each check of a barrier finds it at the phase waited for or one past it;
- data: a K / V' / scale-ring stage or a scale-factor slot holds the tile an operation reads
  when it runs, and is not refilled while a queued operation or a softmax warp still reads it;
  S, P' and O are read and written in the order the online softmax needs.
"""
import random

import pytest
from _protocol import Bar, run, wait


class Model:
    def __init__(self, nt, mx, ring, nks, nvs, nsc, rnd):
        self.nt, self.mx, self.ring = nt, mx, ring
        self.nks, self.nvs, self.nsc = nks, nvs, nsc
        self.n = max(nt)
        self.rnd = rnd
        B = Bar
        self.Q = B("Q", 2 if mx else 1)
        self.KF = [B(f"KF{i}", 1) for i in range(nks)]
        self.KE = [B(f"KE{i}", 1) for i in range(nks)]
        self.VF = [B(f"VF{i}", 1) for i in range(nvs)]
        self.VE = [B(f"VE{i}", 1) for i in range(nvs)]
        self.SF = [B(f"SF{x}", 1) for x in range(2)]
        self.PF = [B(f"PF{x}", 4) for x in range(2)]
        self.PVD = [B(f"PVD{x}", 1) for x in range(2)]
        self.SCF = [B(f"SCF{i}", 1) for i in range(nsc)]
        self.SCE = [B(f"SCE{i}", 8) for i in range(nsc)]
        self.FIN = B("FIN", 1)
        # data held
        self.kstage = [None] * nks
        self.vstage = [None] * nvs
        self.scstage = [None] * nsc
        self.sfslot = [None, None]
        self.q_loaded = False
        self.q_factors = False
        self.S = [[None] * 4 for _ in range(2)]  # per tile and warp: ('S', j) or ('P', j)
        self.pv_done = [0, 0]
        self.ring_readers = {}  # (x, w) -> tile whose ring stage that softmax warp still reads
        self.pipe = []          # issued tcgen05 operations, run in order
        self.inflight = []      # loads in flight: (barrier, stage list, index, tile)

    # --------------------------------------------------------------- helpers
    def wait(self, bar, k):
        return wait(bar, k)

    def pending(self, kind, pred):
        return any(op[0] == kind and pred(op) for op in self.pipe)

    # ------------------------------------------------------------------ roles
    def k_loader(self):
        self.inflight.append((self.Q, None, None, "Q"))
        for j in range(self.n):
            s = j % self.nks
            if j >= self.nks:
                yield from self.wait(self.KE[s], j // self.nks - 1)
            assert not self.pending("qk", lambda op: op[2] % self.nks == s), "K stage refilled under a queued Q·Kᵀ"
            self.kstage[s] = ("loading", j)
            self.inflight.append((self.KF[s], self.kstage, s, j))
            yield True

    def v_loader(self):
        for j in range(self.n):
            s = j % self.nvs
            if j >= self.nvs:
                yield from self.wait(self.VE[s], j // self.nvs - 1)
            assert not self.pending("pv", lambda op: op[2] % self.nvs == s), "V' stage refilled under a queued P·V"
            self.vstage[s] = ("loading", j)
            self.inflight.append((self.VF[s], self.vstage, s, j))
            yield True

    def ring_loader(self):
        if self.mx:
            self.q_factors = True  # the Q tiles' atoms, written by this warp
            self.Q.arrive()
            yield True
        if not self.ring:
            return
        for j in range(self.n):
            st = j % self.nsc
            if j >= self.nsc:
                yield from self.wait(self.SCE[st], j // self.nsc - 1)
            assert not self.pending("cp", lambda op: op[2] % self.nsc == st), "ring stage refilled under a queued copy"
            assert all(t % self.nsc != st for t in self.ring_readers.values()), "ring stage refilled under a reader"
            self.scstage[st] = ("loading", j)
            self.inflight.append((self.SCF[st], self.scstage, st, j))
            yield True

    def engine(self):
        """Loads land in any order."""
        while True:
            if not self.inflight:
                yield False
                continue
            bar, stages, i, tile = self.inflight.pop(self.rnd.randrange(len(self.inflight)))
            if stages is None:
                self.q_loaded = True
            else:
                stages[i] = tile
            bar.arrive()
            yield True

    def tensor_pipe(self):
        while True:
            if not self.pipe:
                yield False
                continue
            op = self.pipe.pop(0)
            kind = op[0]
            if kind == "commit":
                op[1].arrive()
            elif kind == "cpq":
                assert self.q_factors
            elif kind == "cp":
                _, slot, t = op
                assert self.scstage[t % self.nsc] == t, f"copy of K tile {t}'s factors found {self.scstage[t % self.nsc]}"
                self.sfslot[slot] = t
            elif kind == "qk":
                _, x, j = op
                assert self.q_loaded and self.kstage[j % self.nks] == j, f"Q·Kᵀ({x},{j}) on K stage {self.kstage}"
                if self.mx:
                    assert self.sfslot[j & 1] == j, f"Q·Kᵀ({x},{j}) read factors of tile {self.sfslot[j & 1]}"
                for w in range(4):
                    assert j == 0 or self.S[x][w] == ("P", j - 1) and self.pv_done[x] == j, \
                        f"S_{x}({j}) overwrote {self.S[x][w]} before its P·V"
                    self.S[x][w] = ("S", j)
            elif kind == "pv":
                _, x, j = op
                assert self.vstage[j % self.nvs] == j, f"P·V({x},{j}) on V' stage {self.vstage}"
                assert all(self.S[x][w] == ("P", j) for w in range(4)), f"P·V({x},{j}) before every P'"
                assert self.pv_done[x] == j
                self.pv_done[x] = j + 1
            yield True

    def factors_landed(self, j):
        """The MMA thread's wait for the ring stage that holds K tile j's factor atom."""
        yield from self.wait(self.SCF[j % self.nsc], j // self.nsc)

    def mma(self):
        nt, n, P = self.nt, self.n, self.pipe

        def k_factors(j):
            if self.mx:
                yield from self.factors_landed(j)
                P.append(("cp", j & 1, j))

        def qk(x, j):
            P.append(("qk", x, j))
            P.append(("commit", self.SF[x]))

        yield from self.wait(self.Q, 0)
        if self.mx:
            P.append(("cpq",))
        yield from self.wait(self.KF[0], 0)
        yield from k_factors(0)
        for x in (0, 1):
            if nt[x] > 0:
                qk(x, 0)
        P.append(("commit", self.KE[0]))
        yield True
        for j in range(n):
            v_ready = k_ready = False
            for x in (0, 1):
                if j >= nt[x]:
                    continue
                yield from self.wait(self.PF[x], j)
                if not v_ready:
                    yield from self.wait(self.VF[j % self.nvs], j // self.nvs)
                    v_ready = True
                P.append(("pv", x, j))
                P.append(("commit", self.PVD[x]))
                if j + 1 < nt[x]:
                    if not k_ready:
                        yield from self.wait(self.KF[(j + 1) % self.nks], (j + 1) // self.nks)
                        yield from k_factors(j + 1)
                        k_ready = True
                    qk(x, j + 1)
                yield True
            P.append(("commit", self.VE[j % self.nvs]))
            if j + 1 < n:
                P.append(("commit", self.KE[(j + 1) % self.nks]))
        P.append(("commit", self.FIN))
        yield from self.wait(self.FIN, 0)

    def softmax(self, x, w):
        nx = self.nt[x]
        for j in range(self.n):
            st = j % self.nsc
            if self.ring:
                yield from self.wait(self.SCF[st], j // self.nsc)
                assert self.scstage[st] == j
                self.ring_readers[(x, w)] = j
            if j >= nx:
                if self.ring:
                    del self.ring_readers[(x, w)]
                    self.SCE[st].arrive()
                yield True
                continue
            yield from self.wait(self.SF[x], j)
            assert self.S[x][w] == ("S", j), f"softmax {x}.{w} tile {j} read {self.S[x][w]}"
            yield True
            # the rare exact pass: O rescaled once P·V of the previous tile is done; S read again
            if j > 0 and self.rnd.random() < 0.3:
                yield from self.wait(self.PVD[x], j - 1)
                assert self.pv_done[x] == j, f"O rescaled at tile {j} with {self.pv_done[x]} P·V done"
                assert self.S[x][w] == ("S", j)
                yield True
            self.S[x][w] = ("P", j)
            self.PF[x].arrive()
            if self.ring:
                del self.ring_readers[(x, w)]
                self.SCE[st].arrive()
            yield True
        if nx > 0:
            yield from self.wait(self.PVD[x], nx - 1)
            assert self.pv_done[x] == nx, "epilogue read O before the last P·V"

    # ------------------------------------------------------------------ run
    def run(self):
        roles = {"k": self.k_loader(), "v": self.v_loader(), "ring": self.ring_loader(), "mma": self.mma()}
        for x in (0, 1):
            for w in range(4):
                roles[f"s{x}{w}"] = self.softmax(x, w)
        run(roles, [self.engine(), self.tensor_pipe()], self.rnd)
        assert not self.pipe and not self.inflight


NT = [(1, 1), (1, 0), (2, 2), (3, 0), (1, 5), (5, 1), (4, 9), (9, 4), (12, 12), (7, 13), (13, 7), (6, 6)]


@pytest.mark.parametrize("mx,ring,nks,nvs", [
    (False, True, 3, 3),    # E4M3 / INT8 with per-key or per-tile K scales
    (False, False, 3, 3),   # one scale per head: no scale ring
    (False, True, 2, 2),    # bf16 operands (mixed branches): two K and two V' stages
    (True, True, 3, 3),     # MX: the K tiles' scale-factor atoms through the ring into TMEM
])
def test_pair_kernel_protocol(mx, ring, nks, nvs):
    for nt in NT:
        for seed in range(40):
            Model(nt, mx, ring, nks, nvs, 4, random.Random(hash((nt, seed, mx, ring, nks)))).run()


def test_model_catches_a_ring_released_early():
    """The model is not vacuous: a softmax warp that releases its scale-ring stage before it is
    done with the tile (as if the release were moved above the P' store) is caught."""

    class Early(Model):
        def softmax(self, x, w):
            nx = self.nt[x]
            for j in range(self.n):
                st = j % self.nsc
                yield from self.wait(self.SCF[st], j // self.nsc)
                self.SCE[st].arrive()  # released at once
                if j >= nx:
                    yield True
                    continue
                yield from self.wait(self.SF[x], j)
                self.ring_readers[(x, w)] = j
                yield True
                assert self.scstage[st] == j, f"ring stage {st} refilled while tile {j} is read"
                del self.ring_readers[(x, w)]
                self.S[x][w] = ("P", j)
                self.PF[x].arrive()
                yield True
            if nx > 0:
                yield from self.wait(self.PVD[x], nx - 1)

    caught = 0
    for seed in range(60):
        try:
            Early((9, 9), True, True, 3, 3, 4, random.Random(seed)).run()
        except AssertionError:
            caught += 1
    assert caught > 0


def test_model_catches_a_factor_copy_without_its_wait():
    """A copy of K tile j's scale-factor atom issued without waiting for its ring stage to land
    (the wait on the stage's barrier left out) is caught."""

    class NoWait(Model):
        def factors_landed(self, j):
            return iter(())  # the copy's wait, left out

    caught = 0
    for seed in range(30):
        try:
            NoWait((6, 6), True, True, 3, 3, 4, random.Random(seed)).run()
        except AssertionError as e:
            assert "factors" in str(e), str(e)
            caught += 1
    assert caught > 0


def test_model_catches_a_ring_released_by_one_warpgroup():
    """A scale-ring stage whose release barrier counts the warps of one softmax warpgroup instead
    of both is refilled while the other warpgroup still reads it."""

    class Half(Model):
        def __init__(self, *a):
            super().__init__(*a)
            self.SCE = [Bar(f"SCE{i}", 4) for i in range(self.nsc)]

    caught = 0
    for seed in range(40):
        try:
            Half((9, 9), False, True, 3, 3, 4, random.Random(seed)).run()
        except AssertionError:
            caught += 1
    assert caught > 0
