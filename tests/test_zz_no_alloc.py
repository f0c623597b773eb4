"""gdn_forward_batch_noalloc: the batched layer forward for callers that
cannot allocate device memory (a plugin inside a host program that owns all
device allocations, a fixed memory budget, a path where allocating is not
allowed). It takes its workspace from a fixed array inside the library
instead of from the caller.

It runs the same kernels as gdn_forward_batch on the same inputs; only the
workspace address differs. So, through the C ABI and on two calls in a row,
its output, state and ring must equal those of gdn_forward_batch (given an
ordinary workspace) bit for bit: a partial overwrite or a stale read of the
shared array would show. It is also compared with the oracle at the
forward-batch tolerances, and run at the largest batch its array holds. A
batch larger than the array must be refused with a clear error. This file is
collected last so that a run stopping at the first failure has run every
other test."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu

BF16 = ("hidden", "w_qkv", "w_z", "w_ba", "w_out")
OUT_ABS = 2e-3          # the forward-batch output tolerance (bf16 tail rounding)
SCRATCH_BYTES = 16 << 20


def to_dev(d):
    t = {}
    for k, v in d.items():
        x = torch.from_numpy(np.ascontiguousarray(v)).cuda()
        t[k] = x.to(torch.bfloat16) if k in BF16 else x
    return t


def args(t):
    return (t["hidden"], t["w_qkv"], t["w_z"], t["w_ba"], t["w_out"], t["conv_ring"],
            t["conv_w"], t["A_log"], t["dt_bias"], t["norm_w"], t["state"])


def run_both(d, calls):
    """`calls` calls in a row of both entry points, each side carrying its own
    ring and state; a new batch of positions (hidden) for every call. Asserts
    bitwise equality after each call and returns the no-allocation side's
    output and state after the first call (on the host)."""
    B, T, D = d["hidden"].shape
    ref, new = to_dev(d), to_dev(d)
    ws = torch.empty(gdn.forward_batch_workspace_size(B, T), dtype=torch.uint8, device="cuda")
    out_new = torch.empty((B, T, D), dtype=torch.float32, device="cuda")
    for call in range(calls):
        if call > 0:
            h = inputs.forward_inputs(B, T, D=D, seed=1400 + call)["hidden"]
            ref["hidden"] = torch.from_numpy(h).cuda().to(torch.bfloat16)
            new["hidden"] = ref["hidden"].clone()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out_ref = gdn.forward_batch(*args(ref), workspace=ws, Hk=16)
        gdn.forward_batch_noalloc(*args(new), out_new, Hk=16, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out_new, out_ref), f"call {call}: out differs"
        assert torch.equal(new["state"], ref["state"]), f"call {call}: state differs"
        assert torch.equal(new["conv_ring"], ref["conv_ring"]), f"call {call}: ring differs"
        if call == 0:
            first = (out_new.cpu().numpy(), new["state"].cpu().numpy())
    return first


def test_noalloc_matches_workspace_entry_on_two_calls():
    B, T, D = 2, 37, 256
    assert gdn.forward_batch_workspace_size(B, T) <= SCRATCH_BYTES
    d = inputs.forward_inputs(B, T, D=D, seed=1300, state_std=0.05)
    out1, state1 = run_both(d, 2)
    # the first call against the oracle, at the forward-batch tolerances
    out_ref, _ring_ref, st_ref = oracle.load().forward_batch(
        d["hidden"], d["w_qkv"], d["w_z"], d["w_ba"], d["w_out"], d["conv_ring"], d["conv_w"],
        d["A_log"], d["dt_bias"], d["norm_w"], d["state"], Hk=16)
    err = float(np.max(np.abs(out1.astype(np.float64) - out_ref)))
    assert np.all(np.isfinite(out1)) and err <= OUT_ABS, f"out vs oracle {err:.3e}"
    assert_parity(state1, st_ref, "state vs oracle")


@pytest.mark.parametrize("B,T", [(1, 216), (97, 1)])
def test_noalloc_at_the_largest_batch_it_holds(B, T):
    """The largest calls that fit: the intermediates reach the array's end."""
    assert gdn.forward_batch_workspace_size(B, T) <= SCRATCH_BYTES
    assert (gdn.forward_batch_workspace_size(B, T + 1) > SCRATCH_BYTES
            or gdn.forward_batch_workspace_size(B + 1, T) > SCRATCH_BYTES)
    d = inputs.forward_inputs(B, T, D=128, seed=1310 + B, state_std=0.05)
    run_both(d, 2)


def test_noalloc_refuses_batches_beyond_its_scratch():
    D = 64
    B, T = 1, 4096                                    # far more than 16 MiB of intermediates
    assert gdn.forward_batch_workspace_size(B, T) > SCRATCH_BYTES
    d = inputs.forward_inputs(1, 1, D=D, seed=1302)
    t = to_dev(d)
    hidden = torch.zeros((B, T, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, T, D), dtype=torch.float32, device="cuda")
    with pytest.raises(gdn.GdnError) as exc:
        gdn.forward_batch_noalloc(hidden, t["w_qkv"], t["w_z"], t["w_ba"], t["w_out"],
                                  t["conv_ring"], t["conv_w"], t["A_log"], t["dt_bias"],
                                  t["norm_w"], t["state"], out, Hk=16)
    assert exc.value.code == "GDN_ERR_UNSUPPORTED"
    assert "built-in scratch" in str(exc.value)
