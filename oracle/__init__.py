"""TEST INFRASTRUCTURE — the fp64 CPU oracle for the Kimi Delta Attention layer.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline``
leg may import this package.  It shares no code with the CUDA library
(``kimi_delta_attention_21_b200``) and neither imports the other.

What it computes, in the order the "KDA Recurrence" problem page states it:

1. ``alpha_t = exp(g_min * sigmoid(z_t))`` per key channel (decay-gate formula).
2. ``S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T``
   (Kimi Linear report, section 3, Eq. 1), token by token in fp64, in C
   (``kda_oracle.c``).
3. ``o~_t = S_t^T q_t`` from the updated state.
4. Per head: RMS normalisation over the D_v values, ``o~ / sqrt(mean(o~^2) + eps)``
   (eps inside the root: the page's worked example, 0.4999997500001875, fixes it).
5. Multiply by ``sigmoid(gate logits)`` element-wise.
6. Concatenate heads (index ``h * D_v + j``) and apply the projection
   ``y = x W_o^T`` with ``W_o`` of shape ``(D_model, H * D_v)`` (the page's
   second shape example fixes this layout).

Returns ``{"outputs", "final_state"}`` as the page's Requirements list.
Every floating-point step runs in fp64.  Inputs are promoted from fp32 (values
that are exactly fp32 or bf16) before any arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_SRC_BWD = os.path.join(_HERE, "kda_oracle_bwd.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` and ``kda_oracle_bwd.c`` with gcc (IEEE fp64, no fast-math)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_BWD))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
             "-std=c11", "-o", tmp, _SRC, _SRC_BWD, "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            f = lib.kda_oracle_recurrence
            i64, p = ctypes.c_int64, ctypes.c_void_p
            f.argtypes = [i64, i64, i64, i64, i64, p, p, p, p, p, p,
                          ctypes.c_double, p, p, i64, p, p, ctypes.c_int]
            f.restype = ctypes.c_int
            g = lib.kda_oracle_recurrence_bwd
            g.argtypes = [i64, i64, i64, i64, i64, p, p, p, p, p, p, ctypes.c_double, p, p, p,
                          p, p, p, p, p, p, ctypes.c_int]
            g.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f32(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def recurrence(q, k, v, beta, *, z=None, log_decay=None, g_min=-5.0,
               initial_state=None, t_rec=None, want_outputs=True, threads=None):
    """Eq. 1 recurrence and updated-state readout, fp64.

    Shapes follow the "KDA Recurrence" page: q, k, z, log_decay (B,S,H,Dk);
    v (B,S,H,Dv); beta (B,S,H) or (B,S,H,1); initial_state (B,H,Dk,Dv) or None.
    ``log_decay`` (= log alpha) replaces ``g_min * sigmoid(z)`` when given.
    ``t_rec`` optionally lists the (sorted) token indices whose o~ to return.
    Returns (o_core (B,n_rec,H,Dv) fp64 or None, final_state (B,H,Dk,Dv) fp64).
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, S, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, S, H):
        raise ValueError("q/k/v shapes disagree")
    beta = _f32(beta).reshape(B, S, H)
    z = _f32(z)
    log_decay = _f32(log_decay)
    if z is None and log_decay is None:
        raise ValueError("need z or log_decay")
    for name, a in (("z", z), ("log_decay", log_decay)):
        if a is not None and a.shape != q.shape:
            raise ValueError(f"{name} must have the key shape")
    if not g_min < 0:
        raise ValueError("g_min must be negative")
    s0 = _f32(initial_state)
    if s0 is not None and s0.shape != (B, H, Dk, Dv):
        raise ValueError("initial_state must be (B,H,Dk,Dv)")
    rec = None
    n_rec = S
    if t_rec is not None:
        rec = np.ascontiguousarray(np.asarray(t_rec, dtype=np.int64))
        if rec.size and (np.any(np.diff(rec) <= 0) or rec[0] < 0 or rec[-1] >= S):
            raise ValueError("t_rec must be sorted, unique and in range")
        n_rec = rec.size
    o = np.zeros((B, n_rec, H, Dv), np.float64) if want_outputs else None
    sf = np.zeros((B, H, Dk, Dv), np.float64)
    lib = _load()
    rc = lib.kda_oracle_recurrence(
        B, S, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(log_decay), _ptr(beta),
        float(g_min), _ptr(s0), _ptr(rec), n_rec, _ptr(o), _ptr(sf),
        int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle recurrence failed ({rc})")
    return o, sf


def recurrence_bwd(q, k, v, beta, d_o, *, z=None, log_decay=None, g_min=-5.0, initial_state=None,
                   d_final_state=None, threads=None):
    """Gradient of the Eq. 1 recurrence (outputs o~_t read after the update, and
    the final state) by reverse-mode differentiation of the token loop, fp64
    (the steps are listed in kda_oracle_bwd.c).  Given d_o = dL/do~ (B,S,H,Dv)
    and d_final_state = dL/dS_T (B,H,Dk,Dv) or None, returns a dict of fp64
    arrays: dq, dk (B,S,H,Dk), dv (B,S,H,Dv), dbeta (B,S,H), dz (d/dz, when z is
    given) or dlog_decay (when log_decay is given) (B,S,H,Dk), and
    d_initial_state (B,H,Dk,Dv)."""
    q, k, v, d_o = _f32(q), _f32(k), _f32(v), _f32(d_o)
    B, S, H, Dk = q.shape
    Dv = v.shape[-1]
    beta = _f32(beta).reshape(B, S, H)
    z, log_decay = _f32(z), _f32(log_decay)
    if z is None and log_decay is None:
        raise ValueError("need z or log_decay")
    s0, dst = _f32(initial_state), _f32(d_final_state)
    out = {n: np.zeros(shp, np.float64) for n, shp in
           (("dq", (B, S, H, Dk)), ("dk", (B, S, H, Dk)), ("dv", (B, S, H, Dv)), ("dbeta", (B, S, H)),
            ("dg", (B, S, H, Dk)), ("d_initial_state", (B, H, Dk, Dv)))}
    rc = _load().kda_oracle_recurrence_bwd(
        B, S, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(log_decay), _ptr(beta), float(g_min),
        _ptr(s0), _ptr(d_o), _ptr(dst), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dbeta"]),
        _ptr(out["dg"]), _ptr(out["d_initial_state"]), int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle backward failed ({rc})")
    out["dz" if z is not None else "dlog_decay"] = out.pop("dg")
    return out


def gdn_recurrence(q, k, v, beta, *, z=None, log_decay=None, g_min=-5.0, initial_state=None, t_rec=None,
                   want_outputs=True, threads=None):
    """Gated DeltaNet: the DPLR post's GDN form with one scalar decay per token
    and head, S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
    which is Eq. 1 with Diag(alpha_t) = alpha_t I.  ``z`` / ``log_decay`` are
    (B,S,H); every key channel gets the token's value and the Eq. 1 recurrence
    above runs unchanged (same readout from the updated state).  Returns what
    ``recurrence`` returns."""
    Dk = np.asarray(q).shape[-1]
    widen = lambda a: None if a is None else np.repeat(np.asarray(a, np.float32)[..., None], Dk, axis=-1)
    return recurrence(q, k, v, beta, z=widen(z), log_decay=widen(log_decay), g_min=g_min,
                      initial_state=initial_state, t_rec=t_rec, want_outputs=want_outputs, threads=threads)


def log_decay(z, g_min):
    """The decay gate in log form, g_min * sigmoid(z) = log(alpha) ("KDA Recurrence"
    page, gate formula), fp64."""
    return float(g_min) / (1.0 + np.exp(-np.asarray(z, np.float64)))


def norm_gate(o_core, gate_logits, eps):
    """Per-head RMS normalisation over D_v with eps inside the root, then the
    sigmoid output gate ("KDA Recurrence" page, problem statement)."""
    o = np.asarray(o_core, np.float64)
    gl = np.asarray(gate_logits, np.float64)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + float(eps))
    return (o / rms) * (1.0 / (1.0 + np.exp(-gl)))


def project(x, W_o):
    """Head concat (index h*D_v + j) then y = x W_o^T, W_o (D_model, H*D_v)."""
    x = np.asarray(x, np.float64)
    flat = x.reshape(*x.shape[:-2], x.shape[-2] * x.shape[-1])
    return flat @ np.asarray(W_o, np.float64).T


def forward(query, key, value, decay_logits, write_strength, output_gate_logits,
            output_projection, initial_state=None, g_min=-5.0, eps=1e-6,
            log_decay=None, threads=None):
    """The whole layer forward with the "KDA Recurrence" page's argument names.

    Returns {"outputs": (B,S,D_model) fp64, "final_state": (B,H,Dk,Dv) fp64,
    "o_core": (B,S,H,Dv) fp64}.  ``o_core`` (the pre-normalisation readout)
    is extra, for diagnosing a mismatch.
    """
    o, sf = recurrence(query, key, value, write_strength, z=decay_logits,
                       log_decay=log_decay, g_min=g_min,
                       initial_state=initial_state, threads=threads)
    x = norm_gate(o, output_gate_logits, eps)
    y = project(x, output_projection)
    return {"outputs": y, "final_state": sf, "o_core": o}


__all__ = ["build", "recurrence", "recurrence_bwd", "gdn_recurrence", "log_decay", "norm_gate", "project", "forward",
           "default_threads"]
