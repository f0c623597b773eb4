"""gdn_step on the GPU against the fp64 oracle (through the C ABI)."""
import os

import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs
from parity import assert_parity, gather_step_units

pytestmark = pytest.mark.gpu

HOST_THREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def to_dev(d):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in d.items()}


def run_gpu(d):
    t = to_dev(d)
    out = gdn.step(t["state"], t["q"], t["k"], t["v"], t["beta"], t["gate"])
    torch.cuda.synchronize()
    return t["state"].cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("L,B,Hk,Hv", [(2, 3, 16, 32), (1, 5, 4, 4), (3, 2, 2, 8), (1, 7, 1, 3),
                                       (1, 1, 16, 32)])
def test_step_small_full_parity(o, L, B, Hk, Hv):
    d = inputs.decode_inputs(L, B, Hk=Hk, Hv=Hv, seed=100 + L * 10 + B)
    st_ref, out_ref = o.step(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    st, out = run_gpu(d)
    assert_parity(out, out_ref, "out")
    assert_parity(st, st_ref, "state")


@pytest.mark.parametrize("name", ["decode_l1_b1", "decode_l1_b64"])
def test_step_workload_full_parity(o, name):
    d = inputs.WORKLOADS[name].draw()
    st_ref, out_ref = o.step(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    st, out = run_gpu(d)
    assert_parity(out, out_ref, f"{name} out")
    assert_parity(st, st_ref, f"{name} state")


def test_step_36_layers_full_parity(o):
    """L = 36 layers x B = 16 in one launch (1.125 GiB of state): every output
    and state element of all 18,432 (layer, sequence, head) units against the
    oracle, one layer at a time to bound host memory, the oracle's units
    split over the host cores."""
    d = inputs.WORKLOADS["decode_l36_b16"].draw()
    L = d["state"].shape[0]
    st, out = run_gpu(d)
    for l in range(L):
        st_ref, out_ref = o.step(*(d[n][l:l + 1] for n in ("state", "q", "k", "v", "beta",
                                                           "gate")), threads=HOST_THREADS)
        assert_parity(out[l:l + 1], out_ref, f"L36 out, layer {l}")
        assert_parity(st[l:l + 1], st_ref, f"L36 state, layer {l}")


def test_step_chained_tokens(o):
    """Three tokens in a row, each side feeding its own state forward."""
    d0 = inputs.decode_inputs(1, 4, seed=321)
    t = to_dev(d0)
    st_ref = d0["state"].astype(np.float64)
    for tok in range(3):
        d = inputs.decode_inputs(1, 4, seed=400 + tok)
        dt = to_dev(d)
        out = gdn.step(t["state"], dt["q"], dt["k"], dt["v"], dt["beta"], dt["gate"])
        st_ref, out_ref = o.step(st_ref, d["q"], d["k"], d["v"], d["beta"], d["gate"])
        assert_parity(out.cpu().numpy(), out_ref, f"token {tok} out")
    assert_parity(t["state"].cpu().numpy(), st_ref, "chained state")


def test_step_edge_values(o):
    """gate = 0 (no decay), very negative gate (decay to exactly zero),
    beta = 0 and beta = 1, zero key."""
    d = inputs.decode_inputs(1, 2, seed=77)
    d["gate"][0, 0, :8] = 0.0
    d["gate"][0, 0, 8:16] = -200.0
    d["beta"][0, 1, :8] = 0.0
    d["beta"][0, 1, 8:16] = 1.0
    d["k"][0, 1, 3] = 0.0
    st_ref, out_ref = o.step(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    st, out = run_gpu(d)
    assert_parity(out, out_ref, "edge out")
    assert_parity(st, st_ref, "edge state")


def test_step_empty():
    st = torch.zeros(0, 2, 32, 128, 128, device="cuda")
    q = torch.zeros(0, 2, 16, 128, device="cuda")
    out = gdn.step(st, q, q, torch.zeros(0, 2, 32, 128, device="cuda"),
                   torch.zeros(0, 2, 32, device="cuda"), torch.zeros(0, 2, 32, device="cuda"))
    assert out.shape == (0, 2, 32, 128)


def test_step_beyond_int32_indices(o):
    """A state of 9 x 512 x 32 x 128 x 128 floats (> 2^31 elements, 9.7 GB):
    units in the last layer sit past the 32-bit index range."""
    base = inputs.decode_inputs(1, 512, seed=909)
    L = 9
    dev = {k: torch.from_numpy(v).cuda().expand(L, *v.shape[1:]).contiguous()
           for k, v in base.items()}
    assert dev["state"].numel() > 2 ** 31
    out = gdn.step(dev["state"], dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"])
    torch.cuda.synchronize()
    B, Hv, Hk = 512, 32, 16
    units = np.array([(L - 1) * B * Hv + u for u in (0, 1, 777, 16383 - 5, B * Hv - 1)])
    # every layer is a copy of `base`, so unit (l, b, h) has base's (0, b, h) data
    g = gather_step_units(base, units % (B * Hv), Hk, Hv)
    st_ref, out_ref = o.step(g["state"], g["q"], g["k"], g["v"], g["beta"], g["gate"])
    lb, h = np.divmod(units, Hv)
    l, b = np.divmod(lb, B)
    got_out = out[l, b, h].cpu().numpy()
    got_st = dev["state"][l, b, h].cpu().numpy()
    assert_parity(got_out, out_ref[0, :, 0], "int64 out")
    assert_parity(got_st, st_ref[0, :, 0], "int64 state")
    del dev, out
    torch.cuda.empty_cache()
