"""gdn_prefill on the GPU against the fp64 oracle (through the C ABI)."""
import os

import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu

HOST_THREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def to_dev(d):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in d.items()}


def run_gpu(d):
    """Runs through the C ABI with a status word, which must stay zero: no
    bounded wait of the stage pipeline gave up."""
    t = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gdn.prefill(t["state"], t["q"], t["k"], t["v"], t["beta"], t["gate"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "prefill pipeline timeout bit set"
    return t["state"].cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("B,T,Hk,Hv,std", [(2, 37, 16, 32, 0.05), (1, 5, 4, 4, 0.05),
                                           (3, 9, 2, 6, 0.0), (1, 16, 2, 8, 0.05),
                                           (1, 1, 16, 32, 0.05),
                                           (10, 70, 16, 32, 0.05)])   # two waves of CTAs
def test_prefill_small_full_parity(o, B, T, Hk, Hv, std):
    d = inputs.prefill_inputs(B, T, Hk=Hk, Hv=Hv, seed=500 + B * 100 + T, state_std=std)
    st_ref, out_ref = o.prefill(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    st, out = run_gpu(d)
    assert_parity(out, out_ref, "prefill out")
    assert_parity(st, st_ref, "prefill state")


def test_prefill_one_position_equals_step():
    d = inputs.prefill_inputs(3, 1, seed=61, state_std=0.05)
    st_p, out_p = run_gpu(d)
    # prefill's [B, T=1, ...] is step's [L=1, B, ...]
    s = {"state": d["state"][None]}
    for n in ("q", "k", "v", "beta", "gate"):
        s[n] = d[n][:, 0][None]
    t = to_dev(s)
    out_s = gdn.step(t["state"], t["q"], t["k"], t["v"], t["beta"], t["gate"])
    torch.cuda.synchronize()
    assert_parity(out_p[:, 0], out_s[0].cpu().numpy().astype(np.float64), "T=1 out vs step")
    assert_parity(st_p, t["state"][0].cpu().numpy().astype(np.float64), "T=1 state vs step")


def test_prefill_resume_matches_one_pass(o):
    """prefill(T1) then prefill(T2) from the returned state == oracle prefill(T1 + T2)."""
    d = inputs.prefill_inputs(2, 50, seed=62, state_std=0.05)
    t = to_dev(d)
    cut = 23
    sl = lambda x, a, b: x[:, a:b].contiguous()
    o1 = gdn.prefill(t["state"], sl(t["q"], 0, cut), sl(t["k"], 0, cut), sl(t["v"], 0, cut),
                     sl(t["beta"], 0, cut), sl(t["gate"], 0, cut))
    o2 = gdn.prefill(t["state"], sl(t["q"], cut, 50), sl(t["k"], cut, 50), sl(t["v"], cut, 50),
                     sl(t["beta"], cut, 50), sl(t["gate"], cut, 50))
    torch.cuda.synchronize()
    st_ref, out_ref = o.prefill(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    assert_parity(torch.cat([o1, o2], 1).cpu().numpy(), out_ref, "resumed out")
    assert_parity(t["state"].cpu().numpy(), st_ref, "resumed state")


def test_prefill_decay_extremes(o):
    """Runs of no decay, of decay to exactly zero (gate = -200), of strong
    decay, and of growth (gate > 0), which push the kernel's running scale
    through both of its fold-back bounds (2^-40 and 2^40), at the library
    tolerance with no rescaling. The growth run starts from a state cleared
    by gate = -200 and writes values scaled by e^-30, so the state grows by
    about e^30 from about 1e-13 and ends near 0.1: bounded in absolute terms
    while the scale crosses 2^40."""
    d = inputs.prefill_inputs(1, 300, seed=63, state_std=0.05)
    d["gate"][0, :100, :] = 0.0
    d["gate"][0, 100, :] = -200.0
    d["gate"][0, 101:200, :] = -0.45     # the scale shrinks past 2^-40 and folds
    d["gate"][0, 200, :] = -200.0        # clear again
    d["gate"][0, 201:300, :] = 0.3       # and grows past 2^40 and folds
    d["v"][0, 200:300] *= np.float32(np.exp(-30.0))
    st_ref, out_ref = o.prefill(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    assert np.max(np.abs(st_ref)) < 1.0 and np.max(np.abs(out_ref)) < 1.0
    st, out = run_gpu(d)
    assert_parity(out, out_ref, "extreme out")
    assert_parity(st, st_ref, "extreme state")


def test_prefill_empty():
    st = torch.zeros(2, 32, 128, 128, device="cuda")
    q = torch.zeros(2, 0, 16, 128, device="cuda")
    out = gdn.prefill(st, q, q, torch.zeros(2, 0, 32, 128, device="cuda"),
                      torch.zeros(2, 0, 32, device="cuda"), torch.zeros(2, 0, 32, device="cuda"))
    assert out.shape == (2, 0, 32, 128) and not st.any()


def test_prefill_full_workload_full_parity(o):
    """B = 4 x T = 4096 in the benchmark's launch shape: every output of all
    128 (sequence, head) units at all 4096 positions, and the final state,
    against the oracle (its units split over the host cores)."""
    d = inputs.WORKLOADS["prefill_b4_t4096"].draw()
    st, out = run_gpu(d)
    st_ref, out_ref = o.prefill(d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"],
                                threads=HOST_THREADS)
    B = out.shape[0]
    for b in range(B):
        assert_parity(out[b], out_ref[b], f"full prefill out, sequence {b}")
    assert_parity(st, st_ref, "full prefill state")
