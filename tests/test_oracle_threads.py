"""The oracle wrapper's `threads` option splits the listed units (or
sequences) over host threads; each C call writes only its own units, so the
results must equal one single-threaded call bit for bit. The full-size GPU
parity tests rely on it."""
import numpy as np
import pytest

import oracle
from linear_attention_recurrence_04_b200 import inputs

LAYER = ("mixed_qkv", "z", "a", "b", "conv_ring", "conv_w", "A_log", "dt_bias", "norm_w",
         "state")


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def same(a, b):
    return all(np.array_equal(x, y) for x, y in zip(a, b))


def test_step_threads(o):
    d = inputs.decode_inputs(2, 3, seed=11)
    args = (d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    assert same(o.step(*args), o.step(*args, threads=5))
    units = [3, 70, 71, 190]
    assert same(o.step(*args, units=units), o.step(*args, units=units, threads=3))


def test_prefill_threads(o):
    d = inputs.prefill_inputs(2, 9, Hk=4, Hv=8, seed=12, state_std=0.05)
    args = (d["state"], d["q"], d["k"], d["v"], d["beta"], d["gate"])
    assert same(o.prefill(*args), o.prefill(*args, threads=4))


def test_layer_threads(o):
    d = inputs.layer_inputs(5, seed=13)
    a = tuple(d[n] for n in LAYER)
    assert same(o.layer_decode(*a, Hk=16), o.layer_decode(*a, Hk=16, threads=3))
    d2 = inputs.layer_inputs(5, seed=14)
    p = dict(d)
    for n in ("mixed_qkv", "z", "a", "b"):
        p[n] = np.ascontiguousarray(np.stack([d[n], d2[n]], axis=1))
    a = tuple(p[n] for n in LAYER)
    assert same(o.layer_pair(*a, Hk=16), o.layer_pair(*a, Hk=16, threads=2))


def test_kda_prefill_threads(o):
    d = inputs.kda_prefill_inputs(2, 7, Hk=2, Hv=4, seed=15, state_std=0.05)
    args = (d["state"], d["q"], d["k"], d["v"], d["beta"], d["g"])
    assert same(o.kda_prefill(*args), o.kda_prefill(*args, threads=3))
