"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: the values
the "KDA Recurrence" page prints, closed forms of special cases, the other
pages' statements of the same update (DPLR form with bound variables, the
bra-ket form, the fused recurrent pseudo-code, Gated DeltaNet), brute-force
products of explicitly formed transition matrices, and invariants.  Together
they fail on a dropped term, a wrong sign, a read before the update, a decay
applied on the wrong side or dimension, a transposed operand, eps outside the
root, or a transposed projection.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import chunk_mirror

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "kda_recurrence_examples.json")))


def _rand(shape, rng, scale=1.0):
    return (scale * rng.standard_normal(shape)).astype(np.float32)


def _unit(x):
    x = np.asarray(x, np.float64)
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)


def _problem(B, S, H, Dk, Dv, seed, unit_keys=True):
    rng = np.random.default_rng(seed)
    q = _rand((B, S, H, Dk), rng)
    k = _rand((B, S, H, Dk), rng)
    if unit_keys:
        k = _unit(k)
    v = _rand((B, S, H, Dv), rng)
    z = _rand((B, S, H, Dk), rng)
    beta = rng.random((B, S, H)).astype(np.float32)
    S0 = _rand((B, H, Dk, Dv), rng, 0.3)
    return q, k, v, z, beta, S0


def _alpha(z, g_min):
    return np.exp(g_min / (1.0 + np.exp(-np.asarray(z, np.float64))))


# ---------------------------------------------------------------- the page's values

def test_worked_example_exact():
    ex = GOLD["worked_example"]
    i = ex["inputs"]
    out = oracle.forward(np.array(i["query"]), np.array(i["key"]), np.array(i["value"]),
                         np.array(i["decay_logits"]), np.array(i["write_strength"]),
                         np.array(i["output_gate_logits"]), np.array(i["output_projection"]),
                         np.array(i["initial_state"]), g_min=i["g_min"], eps=i["eps"])
    want_y = np.array(ex["outputs"])
    want_s = np.array(ex["final_state"])
    assert out["outputs"].shape == want_y.shape
    assert out["final_state"].shape == want_s.shape
    # fp64 result must equal the printed value to within one unit in the last place
    assert abs(out["outputs"].item() - want_y.item()) <= np.spacing(want_y.item())
    assert out["final_state"].item() == want_s.item()


def test_worked_example_rejects_eps_outside_root():
    # The printed value separates eps inside the root from eps added to the RMS.
    inside = 0.5 / np.sqrt(1.0 + 1e-6)
    outside = 0.5 / (1.0 + 1e-6)
    want = GOLD["worked_example"]["outputs"][0][0][0]
    assert abs(inside - want) <= np.spacing(want)
    assert abs(outside - want) > 1e-7


@pytest.mark.parametrize("case", GOLD["shape_examples"], ids=lambda c: c["cite"])
def test_shape_examples(case):
    rng = np.random.default_rng(3)
    B, S, H, Dk = case["query_key_decay_shape"]
    Dv = case["value_shape"][-1]
    Dm = case["output_projection_shape"][0]
    q, k, v, z, beta, S0 = _problem(B, S, H, Dk, Dv, 11)
    W = _rand(case["output_projection_shape"], rng)
    gl = _rand((B, S, H, Dv), rng)
    out = oracle.forward(q, k, v, z, beta, gl, W, S0.reshape(case["initial_state_shape"]))
    assert list(out["outputs"].shape) == case["outputs_shape"]
    assert list(out["final_state"].shape) == case["final_state_shape"]
    assert Dm == case["outputs_shape"][-1]   # W_o is (D_model, H*Dv)
    assert set(out) >= {"outputs", "final_state"}


# ---------------------------------------------------------------- closed forms

def test_gate_limits():
    # alpha = exp(g_min * sigmoid(z)): z=0 -> exp(g_min/2); z>>0 -> exp(g_min); z<<0 -> 1.
    g_min = -5.0
    Dk, Dv = 3, 1
    z = np.array([0.0, 60.0, -60.0], np.float32).reshape(1, 1, 1, Dk)
    zeros = np.zeros((1, 1, 1, Dk), np.float32)
    S0 = np.ones((1, 1, Dk, Dv), np.float32)
    _, sf = oracle.recurrence(zeros, zeros, np.zeros((1, 1, 1, Dv), np.float32),
                              np.zeros((1, 1, 1), np.float32), z=z, g_min=g_min, initial_state=S0)
    np.testing.assert_allclose(sf[0, 0, :, 0], [np.exp(-2.5), np.exp(-5.0), 1.0], rtol=1e-14, atol=1e-25)


def test_beta_zero_is_pure_channel_decay():
    # beta = 0: S_t = Diag(prod_{i<=t} alpha_i) S_0 and o_t = S_t^T q_t.
    q, k, v, z, beta, S0 = _problem(2, 9, 3, 5, 4, 1)
    beta[:] = 0
    o, sf = oracle.recurrence(q, k, v, beta, z=z, g_min=-3.0, initial_state=S0)
    cum = np.cumprod(_alpha(z, -3.0), axis=1)               # (B,S,H,Dk)
    St = cum[..., :, None] * S0[:, None, :, :, :].astype(np.float64)  # (B,S,H,Dk,Dv)
    np.testing.assert_allclose(o, np.einsum("bshc,bshcj->bshj", q.astype(np.float64), St), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sf, St[:, -1], rtol=1e-12, atol=1e-14)


def test_unit_key_full_write_reads_back_value():
    # beta = 1, ||k|| = 1, q = k: (I - k k^T) k = 0 so S_t^T k_t = v_t exactly,
    # whatever the decay and the earlier state (read-after-update + delta rule).
    q, k, v, z, beta, S0 = _problem(2, 17, 2, 8, 6, 2)
    beta[:] = 1
    kd = k.astype(np.float64)
    k = (kd / np.linalg.norm(kd, axis=-1, keepdims=True)).astype(np.float32)
    o, _ = oracle.recurrence(k, k, v, beta, z=z, g_min=-5.0, initial_state=S0)
    # k is only unit-norm to fp32 precision, hence the tolerance
    np.testing.assert_allclose(o, v.astype(np.float64), atol=5e-6)


def test_orthonormal_keys_give_linear_attention():
    # alpha = 1, beta = 1, one-hot keys on distinct channels, S_0 = 0:
    # S_t = sum_{i<=t} k_i v_i^T (plain linear attention, the derivation's first step).
    S, Dk, Dv = 6, 8, 5
    rng = np.random.default_rng(4)
    k = np.zeros((1, S, 1, Dk), np.float32)
    perm = rng.permutation(Dk)[:S]
    k[0, np.arange(S), 0, perm] = 1.0
    q = _rand((1, S, 1, Dk), rng)
    v = _rand((1, S, 1, Dv), rng)
    beta = np.ones((1, S, 1), np.float32)
    o, sf = oracle.recurrence(q, k, v, beta, log_decay=np.zeros_like(k))
    Sacc = np.zeros((Dk, Dv))
    for t in range(S):
        Sacc = Sacc + np.outer(k[0, t, 0], v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], Sacc.T @ q[0, t, 0], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(sf[0, 0], Sacc, rtol=0, atol=0)


# ---------------------------------------------------------------- other statements of the update

def test_brute_force_transition_matrices():
    # Explicit D_k x D_k transition (I - beta k k^T) Diag(alpha) times S (Dk != Dv,
    # non-unit keys, channel-varying decay).
    B, S, H, Dk, Dv = 1, 7, 2, 3, 2
    q, k, v, z, beta, S0 = _problem(B, S, H, Dk, Dv, 5, unit_keys=False)
    o, sf = oracle.recurrence(q, k, v, beta, z=z, g_min=-4.0, initial_state=S0)
    a = _alpha(z, -4.0)
    for h in range(H):
        St = S0[0, h].astype(np.float64)
        for t in range(S):
            kt = k[0, t, h].astype(np.float64)
            T = (np.eye(Dk) - beta[0, t, h] * np.outer(kt, kt)) @ np.diag(a[0, t, h])
            St = T @ St + beta[0, t, h] * np.outer(kt, v[0, t, h])
            np.testing.assert_allclose(o[0, t, h], St.T @ q[0, t, h], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(sf[0, h], St, rtol=1e-12, atol=1e-13)


def test_dplr_form_with_bound_variables():
    # DPLR post, section 3: S_t = (Diag(alpha) - a b^T) S + beta k v^T with
    # a = beta k and b = k * alpha.
    q, k, v, z, beta, S0 = _problem(1, 8, 1, 4, 3, 6)
    o, sf = oracle.recurrence(q, k, v, beta, z=z, g_min=-2.0, initial_state=S0)
    a_ = _alpha(z, -2.0)
    St = S0[0, 0].astype(np.float64)
    for t in range(8):
        kt = k[0, t, 0].astype(np.float64)
        av = beta[0, t, 0] * kt
        bv = kt * a_[0, t, 0]
        St = (np.diag(a_[0, t, 0]) - np.outer(av, bv)) @ St + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
    np.testing.assert_allclose(sf[0, 0], St, rtol=1e-12, atol=1e-13)


def test_braket_transposed_form():
    # Bra-ket form (state D_v x D_k): S~_t = S~ D + beta (v - S~ D k) k^T.
    q, k, v, z, beta, S0 = _problem(1, 10, 1, 5, 3, 7)
    _, sf = oracle.recurrence(q, k, v, beta, z=z, g_min=-5.0, initial_state=S0)
    a_ = _alpha(z, -5.0)
    St = S0[0, 0].astype(np.float64).T
    for t in range(10):
        D = np.diag(a_[0, t, 0])
        kt = k[0, t, 0].astype(np.float64)
        SD = St @ D
        St = SD + beta[0, t, 0] * np.outer(v[0, t, 0] - SD @ kt, kt)
    np.testing.assert_allclose(sf[0, 0], St.T, rtol=1e-12, atol=1e-13)


def test_fused_recurrent_pseudocode_order():
    # The blog's fused recurrent step with SCALE = 1:
    # state *= exp(g); pred = sum(state*k); res = beta (v - pred);
    # state += k res; out = sum(state * q).
    q, k, v, z, beta, S0 = _problem(1, 12, 1, 6, 4, 8)
    o, sf = oracle.recurrence(q, k, v, beta, z=z, g_min=-5.0, initial_state=S0)
    g = np.log(_alpha(z, -5.0))
    st = S0[0, 0].astype(np.float64)
    for t in range(12):
        st = st * np.exp(g[0, t, 0])[:, None]
        pred = np.sum(st * k[0, t, 0][:, None], axis=0)
        res = beta[0, t, 0] * (v[0, t, 0] - pred)
        st = st + k[0, t, 0][:, None] * res[None, :]
        out = np.sum(st * q[0, t, 0][:, None], axis=0)
        np.testing.assert_allclose(o[0, t, 0], out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sf[0, 0], st, rtol=1e-12, atol=1e-13)


def test_gated_deltanet_when_decay_is_channel_constant():
    # Same alpha on every channel: S_t = alpha (I - beta k k^T) S + beta k v^T (GDN).
    q, k, v, z, beta, S0 = _problem(1, 9, 2, 4, 3, 9)
    z[:] = z[..., :1]
    _, sf = oracle.recurrence(q, k, v, beta, z=z, g_min=-5.0, initial_state=S0)
    a_ = _alpha(z[..., 0], -5.0)
    for h in range(2):
        St = S0[0, h].astype(np.float64)
        for t in range(9):
            kt = k[0, t, h].astype(np.float64)
            St = a_[0, t, h] * (np.eye(4) - beta[0, t, h] * np.outer(kt, kt)) @ St + \
                beta[0, t, h] * np.outer(kt, v[0, t, h])
        np.testing.assert_allclose(sf[0, h], St, rtol=1e-12, atol=1e-13)


def test_gdn_recurrence_matches_the_scalar_decay_form():
    # the GDN oracle (per-head decay inputs) against the DPLR post's scalar form evaluated directly,
    # for z and for a log-decay input, readouts included (o_t = S_t^T q_t after the update)
    q, k, v, z, beta, S0 = _problem(2, 11, 3, 5, 4, 21)
    zh = z[..., 0]
    o, sf = oracle.gdn_recurrence(q, k, v, beta, z=zh, g_min=-3.0, initial_state=S0)
    ld = -3.0 / (1.0 + np.exp(-zh.astype(np.float64)))
    o2, sf2 = oracle.gdn_recurrence(q, k, v, beta, log_decay=ld.astype(np.float32), g_min=-3.0, initial_state=S0)
    for b in range(2):
        for h in range(3):
            St = S0[b, h].astype(np.float64)
            for t in range(11):
                kt = k[b, t, h].astype(np.float64)
                St = np.exp(ld[b, t, h]) * (np.eye(5) - beta[b, t, h] * np.outer(kt, kt)) @ St + \
                    beta[b, t, h] * np.outer(kt, v[b, t, h])
                np.testing.assert_allclose(o[b, t, h], St.T @ q[b, t, h], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(sf[b, h], St, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(sf2, sf, rtol=1e-6, atol=1e-7)   # log alpha rounded to fp32 on that path


def test_gdn_recurrence_pure_decay_closed_form():
    # beta = 0: S_t = (prod alpha) S_0 exactly, for a scalar decay as large as g_min = -20 allows
    q, k, v, z, beta, S0 = _problem(1, 40, 2, 4, 3, 22)
    beta[:] = 0
    zh = z[..., 0]
    _, sf = oracle.gdn_recurrence(q, k, v, beta, z=zh, g_min=-20.0, initial_state=S0)
    tot = np.sum(-20.0 / (1.0 + np.exp(-zh.astype(np.float64))), axis=1)   # (1, H)
    np.testing.assert_allclose(sf, np.exp(tot)[..., None, None] * S0, rtol=1e-12, atol=1e-300)


# ---------------------------------------------------------------- output head

def test_rms_norm_and_gate():
    # constant vector c*1 normalises to c/sqrt(c^2+eps); gate 0 halves, gate +40 keeps.
    o = np.full((1, 1, 2, 4), 3.0)
    gl = np.zeros((1, 1, 2, 4)); gl[..., 1, :] = 40.0
    x = oracle.norm_gate(o, gl, 1e-6)
    np.testing.assert_allclose(x[..., 0, :], 0.5 * 3.0 / np.sqrt(9.0 + 1e-6), rtol=1e-15)
    np.testing.assert_allclose(x[..., 1, :], 3.0 / np.sqrt(9.0 + 1e-6), rtol=1e-15)
    # normalisation is per head: scaling one head does not change the other
    o2 = o.copy(); o2[..., 0, :] *= 10
    x2 = oracle.norm_gate(o2, gl, 1e-6)
    np.testing.assert_allclose(x2[..., 1, :], x[..., 1, :], rtol=1e-15)


def test_projection_concat_order_and_layout():
    x = np.arange(1 * 2 * 3 * 2, dtype=np.float64).reshape(1, 2, 3, 2)  # (B,S,H,Dv)
    eye = np.eye(6)
    np.testing.assert_array_equal(oracle.project(x, eye), x.reshape(1, 2, 6))
    # a W_o with D_model=1 that picks head 2, channel 1 -> flat index 2*Dv+1 = 5
    pick = np.zeros((1, 6)); pick[0, 5] = 1
    np.testing.assert_array_equal(oracle.project(x, pick)[..., 0], x[:, :, 2, 1])


# ---------------------------------------------------------------- invariants

def test_state_handoff():
    q, k, v, z, beta, S0 = _problem(2, 21, 2, 6, 5, 10)
    o, sf = oracle.recurrence(q, k, v, beta, z=z, initial_state=S0)
    o1, s1 = oracle.recurrence(q[:, :8], k[:, :8], v[:, :8], beta[:, :8], z=z[:, :8], initial_state=S0)
    o2, s2 = oracle.recurrence(q[:, 8:], k[:, 8:], v[:, 8:], beta[:, 8:], z=z[:, 8:],
                               initial_state=s1.astype(np.float32))
    # the handoff state is rounded to fp32, so agreement is to fp32 precision
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(s2, sf, rtol=1e-5, atol=1e-6)


def test_frobenius_bound_with_unit_keys():
    # ||(I - beta k k^T) Diag(alpha)||_2 <= 1 for unit k, beta in [0,1], alpha in (0,1]:
    # ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t||.
    q, k, v, z, beta, S0 = _problem(1, 30, 1, 7, 4, 12)
    st = S0
    prev = np.linalg.norm(S0[0, 0].astype(np.float64))
    for t in range(30):
        _, s = oracle.recurrence(q[:, t:t+1], k[:, t:t+1], v[:, t:t+1], beta[:, t:t+1],
                                 z=z[:, t:t+1], initial_state=st)
        now = np.linalg.norm(s[0, 0])
        assert now <= prev + beta[0, t, 0] * np.linalg.norm(v[0, t, 0].astype(np.float64)) + 1e-6
        st = s.astype(np.float32)
        prev = np.linalg.norm(st[0, 0].astype(np.float64))


def test_sampled_rows_match_full_readout():
    q, k, v, z, beta, S0 = _problem(2, 20, 2, 4, 3, 13)
    o, _ = oracle.recurrence(q, k, v, beta, z=z, initial_state=S0)
    rec = [0, 3, 4, 19]
    os_, _ = oracle.recurrence(q, k, v, beta, z=z, initial_state=S0, t_rec=rec)
    np.testing.assert_array_equal(os_, o[:, rec])


def test_threads_do_not_change_result():
    q, k, v, z, beta, S0 = _problem(3, 15, 4, 5, 5, 14)
    a = oracle.recurrence(q, k, v, beta, z=z, initial_state=S0, threads=1)
    b = oracle.recurrence(q, k, v, beta, z=z, initial_state=S0, threads=5)
    np.testing.assert_array_equal(a[0], b[0]); np.testing.assert_array_equal(a[1], b[1])


# ---------------------------------------------------------------- chunk algebra (appendix B)

def test_props_1_2_against_explicit_products():
    rng = np.random.default_rng(15)
    C, Dk, Dv = 6, 4, 3
    k = rng.standard_normal((C, Dk)); v = rng.standard_normal((C, Dv))
    beta = rng.random(C); alpha = np.exp(-3 * rng.random((C, Dk)))
    w, u, P, H = chunk_mirror.wy_chunk(k, v, beta, alpha)
    Pbf = np.eye(Dk); Hbf = np.zeros((Dk, Dv))
    for r in range(C):
        T = (np.eye(Dk) - beta[r] * np.outer(k[r], k[r])) @ np.diag(alpha[r])
        Pbf = T @ Pbf
        Hbf = T @ Hbf + beta[r] * np.outer(k[r], v[r])
        np.testing.assert_allclose(P[r], Pbf, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(H[r], Hbf, rtol=1e-12, atol=1e-13)


def test_beta_outside_bracket_reading_is_wrong():
    # The rendered Eq. 17 could be read with beta on the first term only; the
    # explicit product rejects that reading.
    rng = np.random.default_rng(16)
    C, Dk = 5, 3
    k = rng.standard_normal((C, Dk)); beta = 0.3 + 0.6 * rng.random(C)
    alpha = np.exp(-rng.random((C, Dk)))
    w, _, P, _ = chunk_mirror.wy_chunk(k, np.zeros((C, 1)), beta, alpha)
    gam = np.cumprod(alpha, axis=0)
    w_alt = np.zeros_like(w)
    for r in range(C):
        acc = beta[r] * gam[r] * k[r]
        for i in range(r):
            g = np.prod(alpha[i + 1:r + 1], axis=0)
            acc = acc - w_alt[i] * float(k[i] @ (g * k[r]))
        w_alt[r] = acc
    P_alt = np.diag(gam[-1]) - sum(np.outer(np.prod(alpha[i + 1:], axis=0) * k[i], w_alt[i]) for i in range(C))
    assert np.max(np.abs(P_alt - P[-1])) > 1e-3


@pytest.mark.parametrize("C", [1, 4, 5, 16])
def test_chunk_forms_match_recurrence(C):
    q, k, v, z, beta, S0 = _problem(1, 19, 1, 5, 4, 17)
    o, sf = oracle.recurrence(q, k, v, beta, z=z, initial_state=S0)
    la = np.log(_alpha(z, -5.0))[0, :, 0]
    args = (q[0, :, 0], k[0, :, 0], v[0, :, 0], beta[0, :, 0], la, S0[0, 0])
    for fn in (chunk_mirror.wy_forward, chunk_mirror.matrix_forward):
        oc, sc = fn(*args, C)
        np.testing.assert_allclose(oc, o[0, :, 0], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(sc, sf[0, 0], rtol=1e-10, atol=1e-12)


def test_log_decay_gate_limits():
    z = np.array([0.0, 60.0, -60.0, 1.0])
    g = oracle.log_decay(z, -5.0)
    np.testing.assert_allclose(g[:3], [-2.5, -5.0, 0.0], atol=1e-20)
    # sigmoid(1) = e/(1+e)
    np.testing.assert_allclose(g[3], -5.0 * np.e / (1 + np.e), rtol=1e-15)


# ---------------------------------------------------------------- general DPLR (comparator)

def test_dplr_with_kda_binding_is_kda():
    # a = beta k, b = k * alpha and the write key beta k turn the general DPLR transition into Eq. 1
    from oracle.dplr import dplr_recurrence
    q, k, v, z, beta, S0 = _problem(2, 9, 2, 5, 3, 31)
    alpha = _alpha(z, -4.0)
    a = beta[..., None].astype(np.float64) * k.astype(np.float64)
    b = k.astype(np.float64) * alpha
    o, sf = dplr_recurrence(q, a, v, a, b, z=z, g_min=-4.0, initial_state=S0)
    o2, sf2 = oracle.recurrence(q, k, v, beta, z=z, g_min=-4.0, initial_state=S0)
    np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sf, sf2, rtol=1e-10, atol=1e-12)


def test_dplr_without_erase_is_decayed_linear_attention():
    # a = 0: S_T = Gamma_T S_0 + sum_i Gamma_{i->T} k_i v_i^T with Gamma the channel-wise decay products
    from oracle.dplr import dplr_recurrence
    q, k, v, z, beta, S0 = _problem(1, 7, 1, 4, 3, 32)
    rng = np.random.default_rng(1)
    b = rng.standard_normal(k.shape)
    o, sf = dplr_recurrence(q, k, v, np.zeros_like(k), b, z=z, g_min=-2.0, initial_state=S0)
    g = -2.0 / (1.0 + np.exp(-z[0, :, 0].astype(np.float64)))          # (S, Dk)
    want = np.exp(g.sum(0))[:, None] * S0[0, 0].astype(np.float64)
    for i in range(7):
        want = want + np.exp(g[i + 1:].sum(0))[:, None] * np.outer(k[0, i, 0].astype(np.float64),
                                                                   v[0, i, 0].astype(np.float64))
    np.testing.assert_allclose(sf[0, 0], want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[0, -1, 0], want.T @ q[0, -1, 0].astype(np.float64), rtol=1e-12, atol=1e-13)
