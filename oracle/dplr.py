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
