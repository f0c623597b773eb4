"""The one-kernel short-conv mixer's grid-wide barrier protocol, checked as a
model on the host under randomized interleavings (no GPU).

The device code (tc::grid_barrier_install / _wait in csrc/gdn_tc.cuh) keeps
one 64-bit word, (48-bit tag << 16) | 16-bit count. Per launch every CTA,
from one thread:
  install: read the word; while it does not hold (this tag, count < n),
           compare-and-swap it to (tag, 0), re-reading on failure;
  arrive:  atomic add 1;
  wait:    read until it holds (this tag, count >= n).
Launches on a stream do not overlap (each waits for the previous kernel
before touching the word), a tag names one call and so one grid size, and
a CUDA graph replay repeats a call with its tag.

Each step below is one atomic access of the word, and a random scheduler
interleaves the CTAs of a launch step by step. The checks: no CTA passes
before every CTA of its own launch has arrived (safety, whatever the word
held before: garbage, another call's completed word, or this call's own
completed count from the previous replay), and every launch completes once
all its CTAs run (liveness)."""
import random

import pytest

MASK16 = 0xFFFF
MASK64 = (1 << 64) - 1


class Word:
    def __init__(self, value):
        self.v = value & MASK64


def cta_program(word, tag, n, arrived, passed, me):
    """A generator: each `yield` ends one atomic step of the word."""
    mine = (tag << 16) & MASK64
    # install
    v = word.v
    yield
    while not ((v >> 16) == tag and (v & MASK16) < n):
        prev = word.v                      # atomicCAS(word, v, mine)
        if prev == v:
            word.v = mine
        yield
        if prev == v:
            break
        v = prev
    # (other work of the CTA happens here in the kernel)
    # arrive
    word.v = (word.v + 1) & MASK64
    arrived.add(me)
    yield
    # wait
    while True:
        w = word.v
        if (w >> 16) == tag and (w & MASK16) >= n:
            break
        yield
    # safety: every CTA of this launch has arrived
    assert len(arrived) == n, f"CTA {me} passed with {len(arrived)} of {n} arrived"
    passed.add(me)


def run_launch(word, tag, n, rng, max_steps=100000):
    arrived, passed = set(), set()
    progs = {i: cta_program(word, tag, n, arrived, passed, i) for i in range(n)}
    # CTAs become resident in a random order, some late
    start_order = list(range(n))
    rng.shuffle(start_order)
    live = []
    steps = 0
    while progs:
        if start_order and (not live or rng.random() < 0.3):
            live.append(start_order.pop())
        i = rng.choice(live)
        try:
            next(progs[i])
        except StopIteration:
            del progs[i]
            live.remove(i)
        steps += 1
        assert steps < max_steps, "launch did not complete (liveness)"
    assert passed == set(range(n))
    return word.v


@pytest.mark.parametrize("seed", range(40))
def test_barrier_safe_and_live_under_random_interleavings(seed):
    rng = random.Random(seed)
    n_calls = rng.randint(2, 4)
    calls = []                        # (tag, grid size) of each captured call
    for _ in range(n_calls):
        calls.append((rng.randrange(1, 1 << 48), rng.randint(1, 12)))
    # the word starts as garbage (never holding one of the tags), or zero
    tags = {t for t, _ in calls}
    init = rng.choice([0, rng.randrange(0, 1 << 64)])
    while (init >> 16) in tags:
        init = rng.randrange(0, 1 << 64)
    word = Word(init)
    # launches: replays of the captured calls in any order, each several times
    schedule = [rng.choice(calls) for _ in range(rng.randint(3, 10))]
    for tag, n in schedule:
        end = run_launch(word, tag, n, rng)
        assert end == ((tag << 16) | n), "the word is left as (tag, n)"


def test_replay_of_a_completed_call_does_not_pass_early():
    """The case the install rule exists for: the word holds this tag with a
    complete count from the previous replay; the first CTA of the replay
    must reset it, and no CTA may pass on the stale count."""
    rng = random.Random(7)
    tag, n = 0x123456789AB, 8
    word = Word((tag << 16) | n)
    for _ in range(20):
        assert run_launch(word, tag, n, rng) == ((tag << 16) | n)
