"""TEST INFRASTRUCTURE — fp64 numpy mirror of the chunkwise algebra.

A debugging aid beside the oracle, never used by the product path.  Two forms:

* ``wy_chunk``: Propositions 1 and 2 of the Kimi Linear report (appendix B,
  Eqs. 16-19), written in the report's notation for one chunk:

    gamma_r      = prod_{i<=r} alpha_i,    gamma_{i->r} = prod_{i<j<=r} alpha_j
    w_r = beta_r ( Diag(gamma_r) k_r - sum_{i<r} w_i (k_i^T Diag(gamma_{i->r}) k_r) )   (17)
    u_r = beta_r ( v_r             - sum_{i<r} u_i (k_i^T Diag(gamma_{i->r}) k_r) )     (19)
    P_r = Diag(gamma_r) - sum_{i<=r} Diag(gamma_{i->r}) k_i w_i^T                       (16)
    H_r = sum_{i<=r} Diag(gamma_{i->r}) k_i u_i^T                                       (18)
    S_r = P_r S_0 + H_r

  The scraped equations leave the extent of beta_r open; the induction in the
  proof of Proposition 2 fixes it as multiplying the whole bracket (reading
  recorded in the design notes), and the brute-force pin confirms it.

* ``matrix_backward``: reverse-mode differentiation of the ``matrix_chunk``
  lines, chunk by chunk (the chunkwise backward's algebra), pinned against the
  oracle's gradient of the plain recurrence.

* ``matrix_chunk``: the same chunk in matrix form, as a GPU kernel evaluates
  it: A = strictly-lower decayed beta-weighted K K^T, the unit-lower solve
  (I + A)[W | U] = [Diag(beta)(K * e^G) | Diag(beta) V], V' = U - W S_0,
  O = (Q * e^G) S_0 + M V' with M the causal (diagonal included) decayed
  Q K^T, and S_C = Diag(e^{G_C}) S_0 + (K * e^{G_C - G})^T V'.  Here G is the
  in-chunk cumulative sum of log alpha.  Used to diagnose intermediate
  mismatches; pinned against ``wy_chunk`` and the recurrence.
"""
from __future__ import annotations

import numpy as np


def wy_chunk(k, v, beta, alpha):
    """One chunk (C tokens) of Props. 1-2.  k (C,Dk), v (C,Dv), beta (C,),
    alpha (C,Dk).  Returns (w (C,Dk), u (C,Dv), P list, H list) with P[r], H[r]
    the matrices of Eqs. 16 and 18 after token r (0-based)."""
    k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    beta = np.asarray(beta, np.float64); alpha = np.asarray(alpha, np.float64)
    C, Dk = k.shape
    Dv = v.shape[1]

    def gamma_to(i, r):  # prod over i < j <= r (empty product = 1)
        g = np.ones(Dk)
        for j in range(i + 1, r + 1):
            g = g * alpha[j]
        return g

    def gamma(r):  # prod over j <= r
        return gamma_to(-1, r)

    w = np.zeros((C, Dk)); u = np.zeros((C, Dv))
    for r in range(C):
        acc_w = gamma(r) * k[r]
        acc_u = v[r].copy()
        for i in range(r):
            s = float(k[i] @ (gamma_to(i, r) * k[r]))
            acc_w = acc_w - w[i] * s
            acc_u = acc_u - u[i] * s
        w[r] = beta[r] * acc_w
        u[r] = beta[r] * acc_u
    P, H = [], []
    for r in range(C):
        Pr = np.diag(gamma(r))
        Hr = np.zeros((Dk, Dv))
        for i in range(r + 1):
            dk = gamma_to(i, r) * k[i]
            Pr = Pr - np.outer(dk, w[i])
            Hr = Hr + np.outer(dk, u[i])
        P.append(Pr); H.append(Hr)
    return w, u, P, H


def wy_forward(q, k, v, beta, log_alpha, S0, C):
    """Single sequence through Props. 1-2 chunk by chunk.  q,k,log_alpha (T,Dk),
    v (T,Dv), beta (T,), S0 (Dk,Dv).  Returns (o (T,Dv), S_T)."""
    q = np.asarray(q, np.float64); S = np.array(S0, np.float64)
    T = q.shape[0]
    o = np.zeros((T, np.asarray(v).shape[1]))
    for s in range(0, T, C):
        e = min(T, s + C)
        _, _, P, H = wy_chunk(k[s:e], v[s:e], beta[s:e], np.exp(np.asarray(log_alpha[s:e], np.float64)))
        for r in range(e - s):
            Sr = P[r] @ S + H[r]
            o[s + r] = Sr.T @ q[s + r]
        S = P[e - s - 1] @ S + H[e - s - 1]
    return o, S


def matrix_chunk(q, k, v, beta, log_alpha, S0):
    """One chunk in the matrix form described in the module docstring.
    Returns dict with G, A, M, W, U, Vp, O and S_next (all fp64)."""
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64); beta = np.asarray(beta, np.float64)
    S0 = np.asarray(S0, np.float64)
    C = k.shape[0]
    G = np.cumsum(np.asarray(log_alpha, np.float64), axis=0)
    A = np.zeros((C, C)); M = np.zeros((C, C))
    for r in range(C):
        for i in range(r + 1):
            d = np.exp(G[r] - G[i])
            if i < r:
                A[r, i] = beta[r] * float(np.sum(k[r] * k[i] * d))
            M[r, i] = float(np.sum(q[r] * k[i] * d))
    rhs_w = beta[:, None] * k * np.exp(G)
    rhs_u = beta[:, None] * v
    W = np.zeros_like(rhs_w); U = np.zeros_like(rhs_u)
    for r in range(C):  # forward substitution on the unit-lower system
        W[r] = rhs_w[r] - A[r, :r] @ W[:r]
        U[r] = rhs_u[r] - A[r, :r] @ U[:r]
    Vp = U - W @ S0
    O = (q * np.exp(G)) @ S0 + M @ Vp
    Ktil = k * np.exp(G[-1][None, :] - G)
    S_next = np.exp(G[-1])[:, None] * S0 + Ktil.T @ Vp
    return {"G": G, "A": A, "M": M, "W": W, "U": U, "Vp": Vp, "O": O, "S_next": S_next}


def matrix_forward(q, k, v, beta, log_alpha, S0, C):
    """Single sequence through ``matrix_chunk`` (ragged last chunk allowed)."""
    S = np.array(S0, np.float64)
    T = np.asarray(q).shape[0]
    o = np.zeros((T, np.asarray(v).shape[1]))
    for s in range(0, T, C):
        e = min(T, s + C)
        r = matrix_chunk(q[s:e], k[s:e], v[s:e], beta[s:e], log_alpha[s:e], S)
        o[s:e] = r["O"]
        S = r["S_next"]
    return o, S


def matrix_backward(q, k, v, beta, log_alpha, S0, dO, dST, C):
    """Gradient of one sequence through ``matrix_chunk``, chunk by chunk.  q,k,log_alpha (T,Dk), v, dO
    (T,Dv), beta (T,), S0, dST (Dk,Dv) (dST = dL/dS_T).  Returns a dict of fp64 arrays dq, dk (T,Dk), dv
    (T,Dv), dbeta (T,), dlog_alpha (T,Dk) and dS0 (Dk,Dv).  Per chunk, with E[r,i,c] = e^{G_rc - G_ic}:
    the state gradient runs back through the chunks (dV' = M^T dO + Kd dS_next, dS = (Q e^G)^T dO +
    Diag(e^{G_C}) dS_next - W^T dV'), everything else is chunk-local (through T = (I + A)^{-1}:
    dA = -T^T dT T^T), and every decayed product contributes in its row role and its column role."""
    f = lambda x: np.asarray(x, np.float64)
    q, k, v, beta, log_alpha, dO = f(q), f(k), f(v), f(beta), f(log_alpha), f(dO)
    T = q.shape[0]
    starts = list(range(0, T, C))
    fwd, entering = [], []
    S = f(S0).copy()
    for s in starts:
        e = min(T, s + C)
        n = e - s
        G = np.cumsum(log_alpha[s:e], axis=0)
        E = np.exp(G[:, None, :] - G[None, :, :])
        low, le = np.tril(np.ones((n, n)), -1), np.tril(np.ones((n, n)))
        P = np.einsum('rc,ic,ric->ri', k[s:e], k[s:e], E) * low
        M = np.einsum('rc,ic,ric->ri', q[s:e], k[s:e], E) * le
        Tm = np.linalg.inv(np.eye(n) + beta[s:e, None] * P)
        Kg, Qg, Kd = k[s:e] * np.exp(G), q[s:e] * np.exp(G), k[s:e] * np.exp(G[-1] - G)
        W, U = Tm @ (beta[s:e, None] * Kg), Tm @ (beta[s:e, None] * v[s:e])
        Vp = U - W @ S
        entering.append(S)
        fwd.append(dict(G=G, E=E, P=P, M=M, T=Tm, Kg=Kg, Qg=Qg, Kd=Kd, W=W, Vp=Vp, low=low, le=le))
        S = np.exp(G[-1])[:, None] * S + Kd.T @ Vp
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dbeta", beta),
                                            ("dlog_alpha", log_alpha))}
    dS = f(dST).copy()
    leaving = [None] * len(starts)
    dvp = [None] * len(starts)
    for j in reversed(range(len(starts))):
        s, e, c = starts[j], min(T, starts[j] + C), fwd[j]
        leaving[j] = dS
        dvp[j] = c["M"].T @ dO[s:e] + c["Kd"] @ dS
        dS = c["Qg"].T @ dO[s:e] + np.exp(c["G"][-1])[:, None] * dS - c["W"].T @ dvp[j]
    out["dS0"] = dS
    for j, s in enumerate(starts):
        e, c = min(T, s + C), fwd[j]
        Sj, dSn, dVp = entering[j], leaving[j], dvp[j]
        kk, qq, vv, bb, do = k[s:e], q[s:e], v[s:e], beta[s:e], dO[s:e]
        dQg, dKd = do @ Sj.T, c["Vp"] @ dSn.T
        dgam = np.sum(dSn * Sj, axis=1)
        dM = (do @ c["Vp"].T) * c["le"]
        dW = -dVp @ Sj.T
        dT = dVp @ (bb[:, None] * vv).T + dW @ (bb[:, None] * c["Kg"]).T
        dBv, dBk = c["T"].T @ dVp, c["T"].T @ dW
        dA = -(c["T"].T @ dT @ c["T"].T) * c["low"]
        out["dbeta"][s:e] = np.sum(dBv * vv, 1) + np.sum(dBk * c["Kg"], 1) + np.sum(dA * c["P"], 1)
        dP, E = bb[:, None] * dA, c["E"]
        out["dv"][s:e] = bb[:, None] * dBv
        dKg = bb[:, None] * dBk
        x_row = np.einsum('ri,ic,ric->rc', dP, kk, E)   # P[r,i] in its row role
        x_col = np.einsum('ri,rc,ric->ic', dP, kk, E)   # ... and its column role
        y_row = np.einsum('ri,ic,ric->rc', dM, kk, E)
        y_col = np.einsum('ri,rc,ric->ic', dM, qq, E)
        eG, eD = np.exp(c["G"]), np.exp(c["G"][-1] - c["G"])
        out["dq"][s:e] = dQg * eG + y_row
        out["dk"][s:e] = dKg * eG + dKd * eD + x_row + x_col + y_col
        dG = dQg * c["Qg"] + dKg * c["Kg"] - dKd * c["Kd"] + kk * x_row - kk * x_col + qq * y_row - kk * y_col
        dG[-1] += np.sum(dKd * c["Kd"], 0) + dgam * np.exp(c["G"][-1])
        out["dlog_alpha"][s:e] = np.cumsum(dG[::-1], axis=0)[::-1]
    return out
