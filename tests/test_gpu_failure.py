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
