"""The seeded generators: shapes, recipe properties, determinism."""
import numpy as np

from linear_attention_recurrence_04_b200 import inputs


def test_decode_shapes_and_recipe():
    d = inputs.decode_inputs(2, 3, seed=5)
    assert d["state"].shape == (2, 3, 32, 128, 128) and d["state"].dtype == np.float32
    assert d["q"].shape == (2, 3, 16, 128) and d["k"].shape == (2, 3, 16, 128)
    assert d["v"].shape == (2, 3, 32, 128)
    assert d["beta"].shape == (2, 3, 32) and d["gate"].shape == (2, 3, 32)
    np.testing.assert_allclose(np.linalg.norm(d["q"].astype(np.float64), axis=-1), 1, atol=1e-6)
    np.testing.assert_allclose(np.linalg.norm(d["k"].astype(np.float64), axis=-1), 1, atol=1e-6)
    assert np.all((d["beta"] > 0) & (d["beta"] < 1))
    assert np.all((d["gate"] >= -1) & (d["gate"] <= 0))
    assert abs(float(d["state"].std()) - 0.05) < 0.001


def test_deterministic_and_layer_streams_differ():
    a = inputs.decode_inputs(2, 1, seed=7)
    b = inputs.decode_inputs(2, 1, seed=7)
    for key in a:
        assert np.array_equal(a[key], b[key])
    assert not np.array_equal(a["v"][0], a["v"][1])


def test_empty_decode():
    d = inputs.decode_inputs(0, 4, seed=1)
    assert d["state"].shape == (0, 4, 32, 128, 128)


def test_prefill_and_layer_shapes():
    p = inputs.prefill_inputs(2, 5, seed=3)
    assert p["state"].shape == (2, 32, 128, 128) and not p["state"].any()
    assert p["q"].shape == (2, 5, 16, 128) and p["v"].shape == (2, 5, 32, 128)
    assert np.all((p["gate"] >= -0.5) & (p["gate"] <= 0))
    lay = inputs.layer_inputs(3, seed=4)
    assert lay["mixed_qkv"].shape == (3, 8192) and lay["z"].shape == (3, 4096)
    assert lay["conv_ring"].shape == (3, 3, 8192) and lay["conv_w"].shape == (8192, 4)
    assert lay["A_log"].shape == (32,) and lay["norm_w"].shape == (128,)
    assert lay["state"].shape == (3, 32, 128, 128)


def test_workload_table():
    assert set(inputs.WORKLOADS) == {"decode_l1_b1", "decode_l1_b64", "decode_l36_b16",
                                     "prefill_b4_t4096", "layer_decode_b256"}
