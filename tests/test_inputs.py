"""The seeded input generator: determinism, bf16 rounding, per-head regeneration."""
import numpy as np

import kda_inputs as ki


def test_round_bf16_ties_to_even_and_exactness():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e-39], np.float32)
    r = ki.round_bf16(x)
    assert r[0] == 1.0
    assert r[1] == 1.0                      # tie -> even (mantissa ...0)
    assert r[2] == np.float32(1.0 + 2 ** -6)  # tie -> even (round up)
    assert r[3] == -2.5
    assert np.all(ki.round_bf16(r) == r)     # idempotent
    assert np.all((r.view(np.uint32) & 0xFFFF) == 0)


def test_deterministic_and_head_regeneration():
    w = ki.custom("t", 2, 33, 3, 8, 8, 16, "bf16", seed=5, s0_std=0.02)
    a = ki.make_inputs(w)
    b = ki.make_inputs(w)
    for n in ("q", "k", "v", "z", "beta", "gate", "W_o", "S0"):
        np.testing.assert_array_equal(a[n], b[n])
    h1 = ki.head_inputs(w, 1)
    np.testing.assert_array_equal(a["q"][:, :, 1], h1["q"])
    np.testing.assert_array_equal(a["beta"][:, :, 1], h1["beta"])
    np.testing.assert_array_equal(a["S0"][:, 1], h1["S0"])


def test_distributions():
    w = ki.custom("t", 1, 512, 2, 64, 64, 32, "bf16", seed=9)
    a = ki.make_inputs(w)
    n = np.linalg.norm(a["q"].astype(np.float64), axis=-1)
    assert np.all(np.abs(n - 1) < 1e-2)
    assert a["beta"].min() >= 0 and a["beta"].max() <= 1
    assert a["W_o"].shape == (32, 128)
    assert abs(a["W_o"].std() - 1 / np.sqrt(128)) < 0.01
    assert a["S0"] is None
    assert ki.WORKLOADS["batch_8x8k"].z_std == 2.0
