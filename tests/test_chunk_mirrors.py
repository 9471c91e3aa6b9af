"""The chunk-form algebra of the two SIMT chunk engines, in fp64 numpy beside the
oracle, pinned against the oracle's own token-by-token results: the chunkwise
backward (``chunk_mirror.matrix_backward``) against the gradient of the plain
recurrence (``oracle.recurrence_bwd``, itself pinned by finite differences),
and the chunked general DPLR (``dplr_chunk_mirror``) against the DPLR
recurrence.  A dropped term, a wrong sign or a wrong decay exponent in either
derivation fails these."""
import numpy as np
import pytest

import oracle
from oracle import chunk_mirror
from oracle.dplr import dplr_chunk_mirror, dplr_recurrence


def _inputs(rng, T, Dk, Dv):
    q = (rng.standard_normal((T, Dk)) * 0.5).astype(np.float32)
    k = rng.standard_normal((T, Dk))
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((T, Dv)).astype(np.float32)
    la = (-5.0 / (1.0 + np.exp(-2.0 * rng.standard_normal((T, Dk))))).astype(np.float32)
    return q, k, v, la


@pytest.mark.parametrize("T,Dk,Dv,C", [(150, 8, 6, 64), (150, 8, 6, 16), (1, 4, 3, 64), (64, 5, 7, 64)])
def test_chunk_backward_mirror_matches_oracle_gradient(T, Dk, Dv, C):
    rng = np.random.default_rng(T + 7 * Dk + C)
    q, k, v, la = _inputs(rng, T, Dk, Dv)
    beta = rng.uniform(0, 1, T).astype(np.float32)
    S0 = (rng.standard_normal((Dk, Dv)) * 0.3).astype(np.float32)
    dO = rng.standard_normal((T, Dv)).astype(np.float32)
    dST = rng.standard_normal((Dk, Dv)).astype(np.float32)
    got = chunk_mirror.matrix_backward(q, k, v, beta, la, S0, dO, dST, C)
    w = lambda x: x[None, :, None]  # (T, D) -> (1, T, 1, D)
    want = oracle.recurrence_bwd(w(q), w(k), w(v), beta[None, :, None], w(dO), log_decay=w(la), g_min=-5.0,
                                 initial_state=S0[None, None], d_final_state=dST[None, None])
    pairs = (("dq", want["dq"][0, :, 0]), ("dk", want["dk"][0, :, 0]), ("dv", want["dv"][0, :, 0]),
             ("dbeta", want["dbeta"][0, :, 0]), ("dlog_alpha", want["dlog_decay"][0, :, 0]),
             ("dS0", want["d_initial_state"][0, 0]))
    for name, ref in pairs:
        np.testing.assert_allclose(got[name], ref, rtol=1e-9, atol=1e-10 * max(1.0, np.abs(ref).max()), err_msg=name)


@pytest.mark.parametrize("T,Dk,Dv,C", [(150, 8, 6, 64), (150, 8, 6, 16), (1, 4, 3, 64), (130, 6, 5, 64)])
def test_dplr_chunk_mirror_matches_recurrence(T, Dk, Dv, C):
    rng = np.random.default_rng(3 * T + Dk + C)
    q, k, v, la = _inputs(rng, T, Dk, Dv)
    a = (rng.standard_normal((T, Dk)) * 0.4).astype(np.float32)
    b = (rng.standard_normal((T, Dk)) * 0.4).astype(np.float32)
    S0 = (rng.standard_normal((Dk, Dv)) * 0.3).astype(np.float32)
    o, sf = dplr_chunk_mirror(q, k, v, a, b, la, S0, C)
    w = lambda x: x[None, :, None]
    o_ref, s_ref = dplr_recurrence(w(q), w(k), w(v), w(a), w(b), log_decay=w(la), initial_state=S0[None, None])
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(sf, s_ref[0, 0], rtol=1e-9, atol=1e-11)


def test_dplr_chunk_mirror_with_kda_binding_is_kda():
    """With a = beta k, b = alpha * k and the write key beta k, the DPLR chunk form is KDA's chunk form."""
    rng = np.random.default_rng(5)
    T, Dk, Dv = 100, 6, 4
    q, k, v, la = (x.astype(np.float64) for x in _inputs(rng, T, Dk, Dv))  # the binding formed in fp64
    beta = rng.uniform(0, 1, T)
    S0 = rng.standard_normal((Dk, Dv)) * 0.3
    bk = beta[:, None] * k
    o, sf = dplr_chunk_mirror(q, bk, v, bk, np.exp(la) * k, la, S0, 64)
    o_kda, s_kda = chunk_mirror.matrix_forward(q, k, v, beta, la, S0, 64)
    np.testing.assert_allclose(o, o_kda, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(sf, s_kda, rtol=1e-9, atol=1e-11)
