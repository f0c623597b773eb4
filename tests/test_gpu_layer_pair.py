"""gdn_layer_pair (two-position speculative verify) on the GPU against the
fp64 oracle, through the C ABI."""
import os

import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_04_b200 import gdn, inputs
from parity import assert_parity

pytestmark = pytest.mark.gpu

ORDER = ("mixed_qkv", "z", "a", "b", "conv_ring", "conv_w", "A_log", "dt_bias", "norm_w",
         "state")


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def pair_inputs(B, Hk=16, Hv=32, seed=0):
    """Layer inputs with the per-token activations drawn for two positions."""
    d = inputs.layer_inputs(B, Hk=Hk, Hv=Hv, seed=seed)
    d2 = inputs.layer_inputs(B, Hk=Hk, Hv=Hv, seed=seed + 1)
    for n in ("mixed_qkv", "z", "a", "b"):
        d[n] = np.ascontiguousarray(np.stack([d[n], d2[n]], axis=1))
    return d


def to_dev(d):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in d.items()}


def run_pair(t, Hk):
    out, sring, sstate = gdn.layer_pair(*(t[n] for n in ORDER), Hk=Hk)
    torch.cuda.synchronize()
    return out, sring, sstate


def oracle_pair(o, d, Hk):
    return o.layer_pair(*(d[n] for n in ORDER), Hk=Hk)


@pytest.mark.parametrize("B,Hk,Hv", [(3, 16, 32), (2, 4, 4), (2, 2, 8), (1, 16, 32)])
def test_pair_small_full_parity(o, B, Hk, Hv):
    d = pair_inputs(B, Hk, Hv, seed=900 + B * 10 + Hv)
    out_r, ring_r, st_r, sring_r, sst_r = oracle_pair(o, d, Hk)
    t = to_dev(d)
    out, sring, sstate = run_pair(t, Hk)
    assert_parity(out.cpu().numpy(), out_r, "pair out")
    assert_parity(t["state"].cpu().numpy(), st_r, "pair committed state")
    assert_parity(sstate.cpu().numpy(), sst_r, "pair scratch state")
    assert np.array_equal(t["conv_ring"].cpu().numpy().astype(np.float64), ring_r)
    assert np.array_equal(sring.cpu().numpy().astype(np.float64), sring_r)


def test_pair_equals_two_layer_decodes():
    """The committed half equals gdn_layer_decode of position 0; the scratch
    half equals gdn_layer_decode of position 1 on the committed buffers."""
    d = pair_inputs(4, seed=911)
    t = to_dev(d)
    out, sring, sstate = run_pair(t, 16)
    s = to_dev({k: (v[:, 0] if k in ("mixed_qkv", "z", "a", "b") else v) for k, v in d.items()})
    s = {k: v.contiguous() for k, v in s.items()}
    o0 = gdn.layer_decode(*(s[n] for n in ORDER), Hk=16)
    torch.cuda.synchronize()
    assert torch.equal(s["conv_ring"], t["conv_ring"])
    assert_parity(t["state"].cpu().numpy(), s["state"].cpu().numpy().astype(np.float64),
                  "committed vs one decode")
    assert_parity(out[:, 0].cpu().numpy(), o0.cpu().numpy().astype(np.float64), "out 0")
    for n in ("mixed_qkv", "z", "a", "b"):
        s[n] = torch.from_numpy(np.ascontiguousarray(d[n][:, 1])).cuda()
    o1 = gdn.layer_decode(*(s[n] for n in ORDER), Hk=16)
    torch.cuda.synchronize()
    assert torch.equal(s["conv_ring"], sring)
    assert_parity(sstate.cpu().numpy(), s["state"].cpu().numpy().astype(np.float64),
                  "scratch vs second decode")
    assert_parity(out[:, 1].cpu().numpy(), o1.cpu().numpy().astype(np.float64), "out 1")


def test_pair_accept_then_reject(o):
    """Accept the first draft (the scratch buffers become live), then reject
    the second (the live buffers keep the committed position)."""
    d = pair_inputs(3, seed=921)
    t = to_dev(d)
    ref = {k: v.astype(np.float64) for k, v in d.items()}
    out, sring, sstate = run_pair(t, 16)
    out_r, ring_r, st_r, sring_r, sst_r = oracle_pair(o, ref, 16)
    assert_parity(out.cpu().numpy(), out_r, "first verify out")
    t["conv_ring"], t["state"] = sring, sstate            # accept
    ref["conv_ring"], ref["state"] = sring_r, sst_r
    d2 = pair_inputs(3, seed=931)
    for n in ("mixed_qkv", "z", "a", "b"):
        t[n] = torch.from_numpy(d2[n]).cuda()
        ref[n] = d2[n]
    out, sring, sstate = run_pair(t, 16)
    out_r, ring_r, st_r, sring_r, sst_r = oracle_pair(o, ref, 16)
    assert_parity(out.cpu().numpy(), out_r, "second verify out")
    assert_parity(t["state"].cpu().numpy(), st_r, "second verify committed (draft rejected)")
    assert_parity(t["conv_ring"].cpu().numpy(), ring_r, "second verify ring")


def test_pair_full_workload_full_parity(o):
    """B = 256 sequences, two positions each: both outputs, the committed and
    scratch states and both rings of every sequence against the oracle (its
    sequences split over the host cores); the rings also checked exactly
    against the inputs they must hold."""
    d = pair_inputs(256, seed=941)
    t = to_dev(d)
    out, sring, sstate = run_pair(t, 16)
    ring = t["conv_ring"].cpu().numpy()
    assert np.array_equal(ring[:, :2], d["conv_ring"][:, 1:])
    assert np.array_equal(ring[:, 2], d["mixed_qkv"][:, 0])
    sr = sring.cpu().numpy()
    assert np.array_equal(sr[:, 0], d["conv_ring"][:, 2])
    assert np.array_equal(sr[:, 1], d["mixed_qkv"][:, 0])
    assert np.array_equal(sr[:, 2], d["mixed_qkv"][:, 1])
    out_r, ring_r, st_r, sring_r, sst_r = o.layer_pair(
        *(d[n] for n in ORDER), Hk=16, threads=max(1, len(os.sched_getaffinity(0))))
    assert np.array_equal(ring.astype(np.float64), ring_r), "B256 committed ring"
    assert np.array_equal(sr.astype(np.float64), sring_r), "B256 scratch ring"
    assert_parity(out.cpu().numpy(), out_r, "B256 pair out")
    st, sst = t["state"].cpu().numpy(), sstate.cpu().numpy()
    for b0 in range(0, 256, 64):
        assert_parity(st[b0:b0 + 64], st_r[b0:b0 + 64], f"B256 committed, sequences {b0}..")
        assert_parity(sst[b0:b0 + 64], sst_r[b0:b0 + 64], f"B256 scratch, sequences {b0}..")
