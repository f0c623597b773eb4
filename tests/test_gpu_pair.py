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


def test_pair_indices_past_32_bits(o):
    """A state of 9 x 512 x 32 x 128 x 128 floats (> 2^31 elements, 9.7 GB)
    and its scratch: units in the last layer sit past the 32-bit index range.
    Every layer is a copy of one drawn layer, so a unit's oracle is that
    layer's unit."""
    base = inputs.pair_inputs(1, 512, seed=1750)
    L, B, Hv = 9, 512, 32
    dev = {k: torch.from_numpy(v).cuda().expand(L, *v.shape[1:]).contiguous()
           for k, v in base.items()}
    assert dev["state"].numel() > 2 ** 31
    scratch = torch.empty_like(dev["state"])
    out = gdn.pair(dev["state"], scratch, dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"])
    torch.cuda.synchronize()
    units = [0, 1, 777, 16383 - 5, B * Hv - 1]
    live_ref, tent_ref, out_ref = o.pair(base["state"], base["q"], base["k"], base["v"],
                                         base["beta"], base["gate"], units=units)
    for u in units:
        b, h = divmod(u, Hv)
        assert_parity(out[L - 1, b, :, h].cpu().numpy(), out_ref[0, b, :, h], f"unit {u} out")
        assert_parity(dev["state"][L - 1, b, h].cpu().numpy(), live_ref[0, b, h],
                      f"unit {u} committed state")
        assert_parity(scratch[L - 1, b, h].cpu().numpy(), tent_ref[0, b, h],
                      f"unit {u} scratch state")
    del dev, scratch, out
    torch.cuda.empty_cache()
