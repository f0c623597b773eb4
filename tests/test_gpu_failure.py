"""Failure detection on the GPU without a fault: the library's bounded
mbarrier wait (used by every tensor-core kernel) must give up after its
limit on a barrier that nothing arrives at, report the timeout through a
status word the host reads, and leave the context usable."""
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports():
    timed_out, waited_us = gdn.selftest_bounded_wait(50_000_000)       # 50 ms limit
    assert timed_out
    assert 50_000 <= waited_us < 1_000_000, waited_us


def test_wait_returns_when_the_phase_completes():
    timed_out, waited_us = gdn.selftest_bounded_wait(50_000_000, arrive=True)
    assert not timed_out
    assert waited_us < 10_000, waited_us


def test_context_is_usable_after_a_timeout():
    gdn.selftest_bounded_wait(20_000_000)
    d = inputs.decode_inputs(1, 2, seed=1700)
    t = {k: torch.from_numpy(v).cuda() for k, v in d.items()}
    out = gdn.step(t["state"], t["q"], t["k"], t["v"], t["beta"], t["gate"])
    torch.cuda.synchronize()
    st_ref, out_ref = oracle.load().step(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    assert_parity(out.cpu().numpy(), out_ref, "step after timeout: out")
    assert_parity(t["state"].cpu().numpy(), st_ref, "step after timeout: state")
    x = torch.zeros((3, 16), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((8, 16), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = gdn.linear_bf16(x, w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and not bool(y.any())


def _word_value(word):
    return int(word.item()) & 0xFFFFFFFFFFFFFFFF


def test_grid_barrier_passes_runs_out_and_resets():
    """The one-kernel short-conv mixer's grid-wide barrier, run on its own.
    A tag always comes with one grid size (one tag per enqueued call, which a
    graph replay repeats). 8 CTAs meet on a word that holds stale bytes and,
    on the second run, this tag's own completed count (as a replay finds it),
    and pass. With a new tag and one CTA fewer than expected, every wait runs
    out after its limit, reports bit 16 and leaves the word cleared; that
    call then completes when replayed with its full grid, and another tag
    replaces its completed word."""
    tag = 0x5EED_0000_1234
    word = torch.full((1,), 0x0123_4567_89AB_CDEF, dtype=torch.int64, device="cuda")
    for _ in range(2):
        bits, waited = gdn.selftest_grid_barrier(word, tag, 8, 8, 50_000_000)
        assert bits == [0] * 8, bits
        assert max(waited) < 50_000, waited
        assert _word_value(word) == (tag << 16) | 8
    bits, waited = gdn.selftest_grid_barrier(word, tag + 1, 8, 9, 30_000_000)   # 30 ms limit
    assert bits == [16] * 8, bits
    assert all(30_000 <= w < 1_000_000 for w in waited), waited
    assert _word_value(word) == 0
    bits, _ = gdn.selftest_grid_barrier(word, tag + 1, 9, 9, 50_000_000)
    assert bits == [0] * 9 and _word_value(word) == ((tag + 1) << 16) | 9
    bits, _ = gdn.selftest_grid_barrier(word, tag, 3, 3, 50_000_000)
    assert bits == [0] * 3 and _word_value(word) == (tag << 16) | 3
