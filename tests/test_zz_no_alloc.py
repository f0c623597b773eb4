"""gdn_forward_batch_noalloc: the batched layer forward for callers that
cannot allocate device memory (a plugin inside a host program that owns all
device allocations, a fixed memory budget, a path where allocating is not
allowed). It takes its workspace from a fixed array inside the library
instead of from the caller.

Through the C ABI, on two calls in a row, its outputs, ring and state must
match those of gdn_forward_batch (given an ordinary workspace) within the
tolerances the forward-batch tests use; a batch larger than the built-in
scratch must be refused with a clear error. This file is collected last so
that a run stopping at the first failure has run every other test."""
import numpy as np
import pytest
import torch

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


def test_noalloc_matches_workspace_entry_on_two_calls():
    B, T, D = 2, 37, 256
    assert gdn.forward_batch_workspace_size(B, T) <= SCRATCH_BYTES
    d = inputs.forward_inputs(B, T, D=D, seed=1300, state_std=0.05)
    ref = to_dev(d)                                  # gdn_forward_batch, own workspace
    new = to_dev(d)                                  # gdn_forward_batch_noalloc
    ws = torch.empty(gdn.forward_batch_workspace_size(B, T), dtype=torch.uint8, device="cuda")
    out_new = torch.empty((B, T, D), dtype=torch.float32, device="cuda")
    for call in range(2):
        if call == 1:                                # a second, different batch of positions
            h = inputs.forward_inputs(B, T, D=D, seed=1301)["hidden"]
            ref["hidden"] = torch.from_numpy(h).cuda().to(torch.bfloat16)
            new["hidden"] = ref["hidden"].clone()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out_ref = gdn.forward_batch(*args(ref), workspace=ws, Hk=16)
        gdn.forward_batch_noalloc(*args(new), out_new, Hk=16, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        err = float((out_new - out_ref).abs().max())
        assert torch.isfinite(out_new).all() and err <= OUT_ABS, f"call {call}: out {err:.3e}"
        assert_parity(new["state"].cpu().numpy(), ref["state"].cpu().numpy().astype(np.float64),
                      f"call {call} state")
        assert_parity(new["conv_ring"].cpu().numpy(),
                      ref["conv_ring"].cpu().numpy().astype(np.float64), f"call {call} ring")


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
