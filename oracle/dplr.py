"""TEST INFRASTRUCTURE — fp64 oracle of the general diagonal-plus-low-rank (DPLR)
recurrence of the "Diagonal-Plus-Low-Rank Matrices and Kimi Delta Attention"
post (sections 1 and 3):

    S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,    o_t = S_t^T q_t

with free erase directions a_t, b_t (one per token, key-sized), the diagonal
decay alpha_t = exp(g_min * sigmoid(z_t)) per key channel (or exp(log_decay)),
and the readout from the updated state as in KDA (the post states the DPLR
update only; reading o_t after the update is KDA's Eq. 1 readout, kept so that
KDA is the special case a_t = beta_t k_t, b_t = k_t * alpha_t with the write
key beta_t k_t).  Token by token in numpy fp64, the matrix products written
out; only tests/ and bench.py's CPU baseline may use it.

``dplr_chunk_mirror`` is the chunk form (the algebra of the chunked GPU
engine) in numpy, a debugging aid pinned against ``dplr_recurrence``.
"""
from __future__ import annotations

import numpy as np


def dplr_recurrence(q, k, v, a, b, *, z=None, log_decay=None, g_min=-5.0, initial_state=None):
    """q, k, a, b, z, log_decay (B,S,H,Dk); v (B,S,H,Dv); initial_state (B,H,Dk,Dv) or None.
    Returns (o (B,S,H,Dv) fp64, final state (B,H,Dk,Dv) fp64)."""
    q, k, v, a, b = (np.asarray(x, np.float64) for x in (q, k, v, a, b))
    B, S, H, Dk = q.shape
    Dv = v.shape[-1]
    if log_decay is None:
        if z is None:
            raise ValueError("need z or log_decay")
        log_decay = float(g_min) / (1.0 + np.exp(-np.asarray(z, np.float64)))
    alpha = np.exp(np.asarray(log_decay, np.float64))
    o = np.zeros((B, S, H, Dv))
    sf = np.zeros((B, H, Dk, Dv))
    for bi in range(B):
        for h in range(H):
            St = np.zeros((Dk, Dv)) if initial_state is None else np.asarray(initial_state[bi, h], np.float64).copy()
            for t in range(S):
                transition = np.diag(alpha[bi, t, h]) - np.outer(a[bi, t, h], b[bi, t, h])
                St = transition @ St + np.outer(k[bi, t, h], v[bi, t, h])
                o[bi, t, h] = St.T @ q[bi, t, h]
            sf[bi, h] = St
    return o, sf


def dplr_chunk_mirror(q, k, v, a, b, log_alpha, S0, C):
    """One sequence of the DPLR recurrence in chunk form.  q, k, a, b, log_alpha (T,Dk), v (T,Dv), S0
    (Dk,Dv).  Inside a chunk, with G the cumulative log-decay and y_r = b_r^T S_{r-1}, the erased rows
    Y solve (I + Ba) Y = (b e^{G_{r-1}}) S + Bk V, and O = (Q e^G) S + Mk V - Ma Y, S_next =
    Diag(e^{G_last}) S + (K e^{G_last - G})^T V - (A e^{G_last - G})^T Y, where Bk, Ba (i < r) decay from
    token r - 1 and Mk, Ma (i <= r) from token r.  Returns (o (T,Dv), S_T), fp64."""
    f = lambda x: np.asarray(x, np.float64)
    q, k, v, a, b, log_alpha = f(q), f(k), f(v), f(a), f(b), f(log_alpha)
    S = f(S0).copy()
    T = q.shape[0]
    o = np.zeros((T, v.shape[1]))
    for s in range(0, T, C):
        e = min(T, s + C)
        n = e - s
        G = np.cumsum(log_alpha[s:e], axis=0)
        Gp = G - log_alpha[s:e]
        decay = lambda X, Y: np.exp(X[:, None, :] - Y[None, :, :])
        low, le = np.tril(np.ones((n, n)), -1), np.tril(np.ones((n, n)))
        Bk = np.einsum('rc,ic,ric->ri', b[s:e], k[s:e], decay(Gp, G)) * low
        Ba = np.einsum('rc,ic,ric->ri', b[s:e], a[s:e], decay(Gp, G)) * low
        Mk = np.einsum('rc,ic,ric->ri', q[s:e], k[s:e], decay(G, G)) * le
        Ma = np.einsum('rc,ic,ric->ri', q[s:e], a[s:e], decay(G, G)) * le
        Y = np.linalg.solve(np.eye(n) + Ba, (b[s:e] * np.exp(Gp)) @ S + Bk @ v[s:e])
        o[s:e] = (q[s:e] * np.exp(G)) @ S + Mk @ v[s:e] - Ma @ Y
        ed = np.exp(G[-1] - G)
        S = np.exp(G[-1])[:, None] * S + (k[s:e] * ed).T @ v[s:e] - (a[s:e] * ed).T @ Y
    return o, S
