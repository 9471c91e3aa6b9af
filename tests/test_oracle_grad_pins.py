"""Pins of the oracle's gradient of the recurrence (oracle.recurrence_bwd)
against central finite differences of the forward oracle, which is pinned on
its own: every input (q, k, v, beta, z or log-decay, initial state) on tiny
problems, with a random linear loss L = <dO, o~> + <dS_T, S_T>."""
import numpy as np
import pytest

import oracle


def _problem(seed, B=1, S=6, H=2, Dk=3, Dv=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, S, H, Dk)).astype(np.float32)
    k = rng.standard_normal((B, S, H, Dk))
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((B, S, H, Dv)).astype(np.float32)
    z = rng.standard_normal((B, S, H, Dk)).astype(np.float32)
    beta = rng.random((B, S, H)).astype(np.float32)
    S0 = (0.5 * rng.standard_normal((B, H, Dk, Dv))).astype(np.float32)
    dO = rng.standard_normal((B, S, H, Dv)).astype(np.float32)
    dST = rng.standard_normal((B, H, Dk, Dv)).astype(np.float32)
    return dict(q=q, k=k, v=v, z=z, beta=beta, S0=S0), dO, dST


def _loss(x, dO, dST, g_min, use_log):
    kw = dict(log_decay=x["ld"]) if use_log else dict(z=x["z"])
    o, sf = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], g_min=g_min, initial_state=x["S0"], threads=1, **kw)
    return float(np.sum(o * dO) + np.sum(sf * dST))


def _fd(x, name, dO, dST, g_min, use_log, h=2e-3):
    """Central difference of the loss for every element of input `name`, using the exact
    float32 perturbation actually applied."""
    g = np.zeros(x[name].shape)
    flat = x[name].reshape(-1)
    for i in range(flat.size):
        orig = flat[i]
        flat[i] = np.float32(orig + h)
        up, hu = _loss(x, dO, dST, g_min, use_log), float(flat[i]) - float(orig)
        flat[i] = np.float32(orig - h)
        dn, hd = _loss(x, dO, dST, g_min, use_log), float(orig) - float(flat[i])
        flat[i] = orig
        g.reshape(-1)[i] = (up - dn) / (hu + hd)
    return g


@pytest.mark.parametrize("use_log", [False, True])
def test_gradient_matches_central_differences(use_log):
    x, dO, dST = _problem(3)
    g_min = -2.0
    if use_log:
        x["ld"] = (g_min / (1.0 + np.exp(-x.pop("z").astype(np.float64)))).astype(np.float32)
    kw = dict(log_decay=x["ld"]) if use_log else dict(z=x["z"])
    got = oracle.recurrence_bwd(x["q"], x["k"], x["v"], x["beta"], dO, g_min=g_min, initial_state=x["S0"],
                                d_final_state=dST, threads=1, **kw)
    names = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "S0": "d_initial_state",
             ("ld" if use_log else "z"): ("dlog_decay" if use_log else "dz")}
    for inp, key in names.items():
        want = _fd(x, inp, dO, dST, g_min, use_log)
        # O(h^2) truncation (h = 2e-3) on O(1) curvature: agreement to ~1e-5 of the gradient's scale
        scale = max(1.0, float(np.max(np.abs(want))))
        err = float(np.max(np.abs(got[key] - want)))
        assert err <= 2e-5 * scale, f"{key}: max-abs error {err:.3e} against finite differences"


def test_gradient_without_final_state_term_and_zero_initial_state():
    # dS_T = None and S_0 = None: only the outputs drive the loss; the sequence starts from zero
    x, dO, _ = _problem(4, S=5, H=1, Dk=4, Dv=3)
    x["S0"] = np.zeros_like(x["S0"])
    got = oracle.recurrence_bwd(x["q"], x["k"], x["v"], x["beta"], dO, z=x["z"], g_min=-5.0, threads=1)
    for inp, key in (("q", "dq"), ("k", "dk"), ("z", "dz"), ("S0", "d_initial_state")):
        want = _fd(x, inp, dO, np.zeros((1, 1, 4, 3), np.float32), -5.0, False)
        assert float(np.max(np.abs(got[key] - want))) <= 2e-5 * max(1.0, float(np.max(np.abs(want)))), key


def test_gradient_of_the_first_token_alone():
    # one token from S_0 = 0: o = beta (q.k) v, so do/dv = beta (q.k) and dL/dbeta = (q.k) <v, dO>
    x, dO, _ = _problem(5, S=1, H=1, Dk=3, Dv=2)
    got = oracle.recurrence_bwd(x["q"], x["k"], x["v"], x["beta"], dO, z=x["z"], g_min=-5.0, threads=1)
    q, k, v, b, d = (x["q"][0, 0, 0].astype(np.float64), x["k"][0, 0, 0].astype(np.float64),
                     x["v"][0, 0, 0].astype(np.float64), float(x["beta"][0, 0, 0]), dO[0, 0, 0].astype(np.float64))
    np.testing.assert_allclose(got["dv"][0, 0, 0], b * (q @ k) * d, rtol=1e-12)
    np.testing.assert_allclose(got["dbeta"][0, 0, 0], (q @ k) * (v @ d), rtol=1e-12)
    np.testing.assert_allclose(got["dq"][0, 0, 0], b * (v @ d) * k, rtol=1e-12)
    np.testing.assert_allclose(got["dz"][0, 0, 0], 0.0, atol=1e-300)   # no state to decay
