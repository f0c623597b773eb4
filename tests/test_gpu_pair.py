"""gdn_pair (two-position speculative verify of the recurrence) on the GPU,
through the C ABI: against the fp64 oracle with the library tolerance
(|gpu - ref| <= 1e-5 everywhere, relative 1e-4 where |ref| > 1e-3), and
against two gdn_step calls bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def to_dev(d):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in d.items()}


def run_pair(d):
    t = to_dev(d)
    scratch = torch.full_like(t["state"], float("nan"))
    out = gdn.pair(t["state"], scratch, t["q"], t["k"], t["v"], t["beta"], t["gate"])
    torch.cuda.synchronize()
    return t["state"].cpu().numpy(), scratch.cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("L,B,Hk,Hv", [(1, 3, 16, 32), (2, 2, 4, 4), (1, 5, 2, 6), (3, 1, 1, 3)])
def test_pair_matches_oracle(o, L, B, Hk, Hv):
    d = inputs.pair_inputs(L, B, Hk=Hk, Hv=Hv, seed=1700 + 10 * L + B)
    live_ref, tent_ref, out_ref = o.pair(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    live, tent, out = run_pair(d)
    assert_parity(out, out_ref, "pair out")
    assert_parity(live, live_ref, "pair committed state")
    assert_parity(tent, tent_ref, "pair scratch state")


def test_pair_l1_b64_full_size(o):
    """The benchmark's verify launch (64 sequences x 32 value heads), every
    unit against the oracle."""
    d = inputs.PAIR_WORKLOAD.draw()
    live_ref, tent_ref, out_ref = o.pair(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    live, tent, out = run_pair(d)
    assert_parity(out, out_ref, "pair_l1_b64 out")
    assert_parity(live, live_ref, "pair_l1_b64 committed state")
    assert_parity(tent, tent_ref, "pair_l1_b64 scratch state")


def test_pair_equals_two_steps_bitwise():
    """Position 0 of the pair is gdn_step from the input state; position 1 is
    gdn_step from the committed state: outputs and both states agree bit for
    bit."""
    d = inputs.pair_inputs(2, 6, seed=1720)
    t = to_dev(d)
    live = t["state"].clone()
    scratch = torch.empty_like(live)
    out = gdn.pair(live, scratch, t["q"], t["k"], t["v"], t["beta"], t["gate"])
    s = t["state"].clone()
    pos = lambda x, p: x[:, :, p].contiguous()
    o0 = gdn.step(s, pos(t["q"], 0), pos(t["k"], 0), pos(t["v"], 0), pos(t["beta"], 0),
                  pos(t["gate"], 0))
    committed = s.clone()
    o1 = gdn.step(s, pos(t["q"], 1), pos(t["k"], 1), pos(t["v"], 1), pos(t["beta"], 1),
                  pos(t["gate"], 1))
    torch.cuda.synchronize()
    assert torch.equal(out[:, :, 0], o0), "position 0 output"
    assert torch.equal(out[:, :, 1], o1), "position 1 output"
    assert torch.equal(live, committed), "committed state"
    assert torch.equal(scratch, s), "scratch state"


def test_pair_accept_then_continue(o):
    """Accepting the draft (taking the scratch state) and decoding one more
    token equals the oracle over three positions."""
    d = inputs.pair_inputs(1, 4, Hk=4, Hv=8, seed=1730)
    t = to_dev(d)
    scratch = torch.empty_like(t["state"])
    gdn.pair(t["state"], scratch, t["q"], t["k"], t["v"], t["beta"], t["gate"])
    nxt = inputs.decode_inputs(1, 4, Hk=4, Hv=8, seed=1731)
    tn = to_dev(nxt)
    out2 = gdn.step(scratch, tn["q"], tn["k"], tn["v"], tn["beta"], tn["gate"])
    torch.cuda.synchronize()
    _, tent_ref, _ = o.pair(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    st_ref, out_ref = o.step(tent_ref, nxt["q"], nxt["k"], nxt["v"], nxt["beta"], nxt["gate"])
    assert_parity(out2.cpu().numpy(), out_ref, "after accept out")
    assert_parity(scratch.cpu().numpy(), st_ref, "after accept state")


def test_pair_empty_batch_is_a_no_op():
    d = inputs.pair_inputs(1, 0, seed=1740)
    t = to_dev(d)
    scratch = torch.empty_like(t["state"])
    out = gdn.pair(t["state"], scratch, t["q"], t["k"], t["v"], t["beta"], t["gate"])
    torch.cuda.synchronize()
    assert out.shape == (1, 0, 2, 32, 128)
