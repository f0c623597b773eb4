"""gdn_layer_decode on the GPU against the fp64 oracle (through the C ABI)."""
import os

import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu

HOST_THREADS = max(1, len(os.sched_getaffinity(0)))

ORDER = ("mixed_qkv", "z", "a", "b", "conv_ring", "conv_w", "A_log", "dt_bias", "norm_w",
         "state")


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def to_dev(d):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in d.items()}


def run_gpu(t, Hk):
    out = gdn.layer_decode(*(t[n] for n in ORDER), Hk=Hk)
    torch.cuda.synchronize()
    return out


def run_oracle(o, d, Hk, seqs=None, threads=1):
    return o.layer_decode(d["mixed_qkv"], d["z"], d["a"], d["b"], d["conv_ring"], d["conv_w"],
                          d["A_log"], d["dt_bias"], d["norm_w"], d["state"], Hk=Hk, seqs=seqs,
                          threads=threads)


@pytest.mark.parametrize("B,Hk,Hv", [(3, 16, 32), (2, 4, 4), (2, 2, 8), (1, 16, 32)])
def test_layer_small_full_parity(o, B, Hk, Hv):
    d = inputs.layer_inputs(B, Hk=Hk, Hv=Hv, seed=700 + B * 10 + Hv)
    out_ref, ring_ref, st_ref = run_oracle(o, d, Hk)
    t = to_dev(d)
    out = run_gpu(t, Hk)
    assert_parity(out.cpu().numpy(), out_ref, "layer out")
    assert_parity(t["state"].cpu().numpy(), st_ref, "layer state")
    assert np.array_equal(t["conv_ring"].cpu().numpy().astype(np.float64), ring_ref), "ring"


def test_layer_chained_two_tokens(o):
    """Two tokens in a row; each side carries its own state and ring (the
    pages' chained, non-reset comparison)."""
    d = inputs.layer_inputs(4, seed=71)
    t = to_dev(d)
    ref = {k: v.astype(np.float64) for k, v in d.items()}
    for tok in range(2):
        fresh = inputs.layer_inputs(4, seed=80 + tok)
        for n in ("mixed_qkv", "z", "a", "b"):
            t[n] = torch.from_numpy(fresh[n]).cuda()
            ref[n] = fresh[n]
        out = run_gpu(t, 16)
        out_ref, ref["conv_ring"], ref["state"] = run_oracle(o, ref, 16)
        assert_parity(out.cpu().numpy(), out_ref, f"token {tok} out")
    assert_parity(t["state"].cpu().numpy(), ref["state"], "chained state")
    assert_parity(t["conv_ring"].cpu().numpy(), ref["conv_ring"], "chained ring")


def test_layer_full_workload_full_parity(o):
    """B = 256 in the benchmark's launch shape: out, state and ring of every
    sequence against the oracle (its sequences split over the host cores);
    the ring update (pure data movement) also checked exactly."""
    d = inputs.WORKLOADS["layer_decode_b256"].draw()
    t = to_dev(d)
    out = run_gpu(t, 16).cpu().numpy()
    ring = t["conv_ring"].cpu().numpy()
    assert np.array_equal(ring[:, :2], d["conv_ring"][:, 1:])
    assert np.array_equal(ring[:, 2], d["mixed_qkv"])
    out_ref, ring_ref, st_ref = run_oracle(o, d, 16, threads=HOST_THREADS)
    assert np.array_equal(ring.astype(np.float64), ring_ref), "B256 ring"
    assert_parity(out, out_ref, "B256 out")
    st = t["state"].cpu().numpy()
    for b0 in range(0, st.shape[0], 64):
        assert_parity(st[b0:b0 + 64], st_ref[b0:b0 + 64], f"B256 state, sequences {b0}..")


def test_layer_empty():
    d = inputs.layer_inputs(1, seed=3)
    t = to_dev(d)
    for n in ("mixed_qkv", "z", "a", "b", "conv_ring", "state"):
        t[n] = t[n][:0]
    out = run_gpu(t, 16)
    assert out.shape == (0, 4096)
