"""A randomized model of the split-KV decode kernel's fused combine (csrc/decode.cu).

Each of a (batch, kv head)'s `splits` CTAs writes its partial (O, m, L), fences it, and takes a
ticket from a 64-bit word in the workspace with a compare-and-swap loop: the word holds this
call's epoch in its high half and a count in its low half; a word with another epoch (an older
call's, or whatever the workspace held) counts as empty.  The CTA whose ticket makes the count
equal `splits` merges every split's partial and resets the word to 0.  No CTA waits for another.

The model restates that protocol (the CAS loop step by step, interleaved at random between the
CTAs) over several calls in a row on one workspace, with the host's fresh nonzero epoch per call.
It checks that exactly one CTA per call merges, and only after every split's partial is written.
"""
import random

import pytest

MASK32 = (1 << 32) - 1


class Word:
    def __init__(self, v):
        self.v = v

    def cas(self, old, new):
        prev = self.v
        if prev == old:
            self.v = new
        return prev


def cta(word, epoch, splits, c, written, merged):
    written.add(c)          # partial written, then fenced
    yield
    old = word.v            # atomicAdd(tk, 0): a read
    yield
    while True:
        nw = old + 1 if (old >> 32) == epoch else (epoch << 32) | 1
        prev = word.cas(old, nw)
        yield
        if prev == old:
            if (nw & MASK32) == splits:
                assert written == set(range(splits)), f"merge before partials {set(range(splits)) - written}"
                merged.append(c)
                word.v = 0  # the merging CTA resets the word
            return
        old = prev


def one_call(word, epoch, splits, rnd):
    written, merged = set(), []
    gens = [cta(word, epoch, splits, c, written, merged) for c in range(splits)]
    live = list(gens)
    while live:
        g = rnd.choice(live)
        try:
            next(g)
        except StopIteration:
            live.remove(g)
    assert len(merged) == 1, f"{len(merged)} CTAs merged"
    assert word.v == 0


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 16, 63])
def test_exactly_one_cta_merges_each_call(splits):
    for seed in range(60):
        rnd = random.Random(seed * 131 + splits)
        # whatever the workspace held: zero, or a word from an earlier call (another epoch)
        word = Word(rnd.choice([0, (5 << 32) | rnd.randrange(1 << 32), rnd.randrange(1 << 32)]))
        epoch = 7
        for _ in range(4):
            one_call(word, epoch, splits, rnd)
            epoch += 1


def test_a_call_after_an_abandoned_one():
    """A call that stopped before every split took its ticket (its word keeps a partial count of
    its own epoch) does not disturb the next call, which has a new epoch."""
    rnd = random.Random(3)
    word = Word(0)
    gens = [cta(word, 1, 5, c, set(range(5)), []) for c in range(3)]  # 3 of 5 splits ran
    for g in gens:
        for _ in g:
            pass
    assert word.v == (1 << 32) | 3
    one_call(word, 2, 5, rnd)


def test_model_catches_an_epoch_left_out():
    """Without the epoch (a plain counter), the count an abandoned call left makes a CTA merge
    before every split's partial is written: the model's check fires."""

    def plain_cta(word, splits, c, written, merged):
        written.add(c)
        yield
        old = word.v
        while True:
            prev = word.cas(old, old + 1)
            yield
            if prev == old:
                if old + 1 == splits:
                    assert written == set(range(splits)), "merge before partials"
                    merged.append(c)
                    word.v = 0
                return
            old = prev

    word = Word(3)  # an abandoned call's count
    written, merged = set(), []
    with pytest.raises(AssertionError, match="merge before partials"):
        for g in [plain_cta(word, 5, c, written, merged) for c in range(5)]:
            for _ in g:
                pass
