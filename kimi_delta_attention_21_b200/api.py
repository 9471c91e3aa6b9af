"""Torch-facing binding of libkda: argument marshalling only.

Every step of the layer runs inside libkda's CUDA kernels; torch supplies the
device memory and the current stream.  Names follow the "KDA Recurrence"
problem page: query, key (B,S,H,D_k); value, output gate logits (B,S,H,D_v);
write strength beta (B,S,H); decay logits (B,S,H,D_k); state (B,H,D_k,D_v);
output projection (D_model, H*D_v).
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import ChunkArgs, DecodeArgs, DplrArgs, RecBwdArgs, check

_DT = {torch.float32: _lib.KDA_F32, torch.bfloat16: _lib.KDA_BF16}
ENGINES = {"auto": _lib.ENGINE_AUTO, "simt": _lib.ENGINE_SIMT, "tc": _lib.ENGINE_TC}


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)") from None


def _dev(t, name, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def gate(z: torch.Tensor, g_min: float) -> torch.Tensor:
    """log(alpha) = g_min * sigmoid(z), fp32, same shape as z."""
    _dev(z, "z")
    out = torch.empty(z.shape, dtype=torch.float32, device=z.device)
    check("kda_gate", _lib.load().kda_gate(_ptr(z), _dtype_code(z), z.numel(), float(g_min), _ptr(out),
                                           _stream(z.device)))
    return out


def chunk_fwd(q, k, v, beta, *, z=None, log_decay=None, g_min=-5.0, initial_state=None,
              gate_logits=None, eps=1e-6, chunk=64, engine="auto", want_final_state=True,
              out=None, final_state=None, dev_status=None, workspace=None, scalar_decay=False):
    """Chunkwise prefill.  Returns (o, final_state):
    o (B,S,H,D_v) in the input dtype holds o~ (gate_logits None) or
    RMSNorm(o~) * sigmoid(gate_logits); final_state (B,H,D_k,D_v) fp32 or None.
    ``final_state`` may be the same tensor as ``initial_state`` (in-place handoff).
    ``workspace`` is an optional uint8 CUDA tensor at least
    ``chunk_workspace_bytes(...)`` long (allocated per call when omitted).
    ``scalar_decay=True`` runs the Gated DeltaNet case (kda_gdn_chunk_fwd): z
    and log_decay are then (B,S,H), one decay per token and head."""
    _dev(q, "q")
    dt = q.dtype
    B, S, H, Dk = q.shape
    Dv = v.shape[-1]
    _dev(k, "k", dt, q.shape)
    _dev(v, "v", dt, (B, S, H, Dv))
    if beta.dim() == 4 and beta.shape[-1] == 1:
        beta = beta.view(B, S, H)
    _dev(beta, "beta", dt, (B, S, H))
    dshape = (B, S, H) if scalar_decay else q.shape
    _dev(z, "z", dt, dshape)
    _dev(log_decay, "log_decay", torch.float32, dshape)
    _dev(initial_state, "initial_state", torch.float32, (B, H, Dk, Dv))
    _dev(gate_logits, "gate_logits", dt, (B, S, H, Dv))
    _dev(dev_status, "dev_status", torch.int32)
    if out is None:
        out = torch.empty((B, S, H, Dv), dtype=dt, device=q.device)
    _dev(out, "out", dt, (B, S, H, Dv))
    if final_state is None and want_final_state:
        final_state = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    _dev(final_state, "final_state", torch.float32, (B, H, Dk, Dv))
    a = ChunkArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_dtype_code(q),
                  q=_ptr(q), k=_ptr(k), v=_ptr(v), z=_ptr(z), log_decay=_ptr(log_decay),
                  g_min=float(g_min), beta=_ptr(beta), initial_state=_ptr(initial_state),
                  gate_logits=_ptr(gate_logits), eps=float(eps), o=_ptr(out),
                  final_state=_ptr(final_state), workspace=None, workspace_bytes=0,
                  chunk=int(chunk), engine=ENGINES[engine], dev_status=_ptr(dev_status),
                  stream=_stream(q.device))
    lib = _lib.load()
    ws_fn, fwd_fn = (("kda_gdn_chunk_workspace_size", "kda_gdn_chunk_fwd") if scalar_decay
                     else ("kda_chunk_workspace_size", "kda_chunk_fwd"))
    nbytes = ctypes.c_size_t(0)
    check(ws_fn, getattr(lib, ws_fn)(ctypes.byref(a), ctypes.byref(nbytes)))
    ws = workspace
    if nbytes.value:
        if ws is None:
            ws = torch.empty(nbytes.value, dtype=torch.uint8, device=q.device)
        _dev(ws, "workspace", torch.uint8)
        a.workspace = _ptr(ws)
        a.workspace_bytes = ws.numel()
    check(fwd_fn, getattr(lib, fwd_fn)(ctypes.byref(a)))
    return out, final_state


def chunk_workspace_bytes(B, S, H, Dk, Dv, dtype=torch.bfloat16, chunk=64, engine="auto", g_min=-5.0,
                          scalar_decay=False):
    a = ChunkArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_DT[dtype], g_min=float(g_min), eps=1e-6,
                  chunk=chunk, engine=ENGINES[engine])
    n = ctypes.c_size_t(0)
    fn = "kda_gdn_chunk_workspace_size" if scalar_decay else "kda_chunk_workspace_size"
    check(fn, getattr(_lib.load(), fn)(ctypes.byref(a), ctypes.byref(n)))
    return n.value


def gdn_chunk_fwd(q, k, v, beta, **kw):
    """Gated DeltaNet prefill (one scalar decay per token and head): chunk_fwd with
    z / log_decay of shape (B,S,H).  Returns (o, final_state)."""
    return chunk_fwd(q, k, v, beta, scalar_decay=True, **kw)


def recurrent_bwd(q, k, v, beta, d_o, *, z=None, log_decay=None, g_min=-5.0, initial_state=None,
                  d_final_state=None, want_d_initial_state=True, workspace=None):
    """Gradient of the prefill recurrence (kda_recurrent_bwd): given d_o = dL/do~
    (B,S,H,D_v) and d_final_state = dL/dS_T (B,H,D_k,D_v) or None, returns a dict
    of fp32 tensors dq, dk, dv, dbeta, dz (d/dz, or d/dlog_decay when log_decay is
    given) and d_initial_state (or None)."""
    return _bwd("kda_recurrent_bwd", q, k, v, beta, d_o, z, log_decay, g_min, initial_state, d_final_state,
                want_d_initial_state, workspace)


def chunk_bwd(q, k, v, beta, d_o, *, z=None, log_decay=None, g_min=-5.0, initial_state=None,
              d_final_state=None, want_d_initial_state=True, workspace=None):
    """The same gradients as ``recurrent_bwd``, in the chunk form (kda_chunk_bwd:
    chunks in parallel, only the state and its gradient carried in order)."""
    return _bwd("kda_chunk_bwd", q, k, v, beta, d_o, z, log_decay, g_min, initial_state, d_final_state,
                want_d_initial_state, workspace)


def _bwd(entry, q, k, v, beta, d_o, z, log_decay, g_min, initial_state, d_final_state, want_d_initial_state,
         workspace):
    _dev(q, "q")
    dt = q.dtype
    B, S, H, Dk = q.shape
    Dv = v.shape[-1]
    _dev(k, "k", dt, q.shape)
    _dev(v, "v", dt, (B, S, H, Dv))
    if beta.dim() == 4 and beta.shape[-1] == 1:
        beta = beta.view(B, S, H)
    _dev(beta, "beta", dt, (B, S, H))
    _dev(d_o, "d_o", dt, (B, S, H, Dv))
    _dev(z, "z", dt, q.shape)
    _dev(log_decay, "log_decay", torch.float32, q.shape)
    _dev(initial_state, "initial_state", torch.float32, (B, H, Dk, Dv))
    _dev(d_final_state, "d_final_state", torch.float32, (B, H, Dk, Dv))
    f32 = dict(dtype=torch.float32, device=q.device)
    out = {"dq": torch.empty((B, S, H, Dk), **f32), "dk": torch.empty((B, S, H, Dk), **f32),
           "dv": torch.empty((B, S, H, Dv), **f32), "dbeta": torch.empty((B, S, H), **f32),
           "dz": torch.empty((B, S, H, Dk), **f32),
           "d_initial_state": torch.empty((B, H, Dk, Dv), **f32) if want_d_initial_state else None}
    a = RecBwdArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_dtype_code(q), q=_ptr(q), k=_ptr(k), v=_ptr(v),
                   z=_ptr(z), log_decay=_ptr(log_decay), g_min=float(g_min), beta=_ptr(beta),
                   initial_state=_ptr(initial_state), d_o=_ptr(d_o), d_final_state=_ptr(d_final_state),
                   dq=_ptr(out["dq"]), dk=_ptr(out["dk"]), dv=_ptr(out["dv"]), dbeta=_ptr(out["dbeta"]),
                   dz=_ptr(out["dz"]), d_initial_state=_ptr(out["d_initial_state"]), workspace=None,
                   workspace_bytes=0, stream=_stream(q.device))
    lib = _lib.load()
    n = ctypes.c_size_t(0)
    check(entry + "_workspace_size", getattr(lib, entry + "_workspace_size")(ctypes.byref(a), ctypes.byref(n)))
    ws = workspace
    if n.value:
        if ws is None:
            ws = torch.empty(n.value, dtype=torch.uint8, device=q.device)
        _dev(ws, "workspace", torch.uint8)
        a.workspace = _ptr(ws)
        a.workspace_bytes = ws.numel()
    check(entry, getattr(lib, entry)(ctypes.byref(a)))
    if log_decay is not None:
        out["dlog_decay"] = out.pop("dz")
    return out


def dplr_recurrent_fwd(q, k, v, a, b, *, z=None, log_decay=None, g_min=-5.0, initial_state=None, out=None,
                       final_state=None):
    """General DPLR recurrence S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T, o_t = S_t^T q_t
    (kda_dplr_recurrent_fwd, token by token).  q, k, a, b, z (B,S,H,D_k); v (B,S,H,D_v).  Returns (o,
    final_state fp32)."""
    return _dplr(False, q, k, v, a, b, z, log_decay, g_min, initial_state, out, final_state, None)


def dplr_chunk_fwd(q, k, v, a, b, *, z=None, log_decay=None, g_min=-5.0, initial_state=None, out=None,
                   final_state=None, workspace=None):
    """The same recurrence and outputs in chunk form (kda_dplr_chunk_fwd)."""
    return _dplr(True, q, k, v, a, b, z, log_decay, g_min, initial_state, out, final_state, workspace)


def dplr_chunk_workspace_bytes(B, S, H, Dk, Dv):
    """Workspace bytes kda_dplr_chunk_fwd needs for these sizes."""
    args = DplrArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_lib.KDA_BF16, g_min=-1.0)
    n = ctypes.c_size_t(0)
    check("kda_dplr_chunk_workspace_size", _lib.load().kda_dplr_chunk_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    return n.value


def _dplr(chunked, q, k, v, a, b, z, log_decay, g_min, initial_state, out, final_state, workspace):
    _dev(q, "q")
    dt = q.dtype
    B, S, H, Dk = q.shape
    Dv = v.shape[-1]
    for name, t in (("k", k), ("a", a), ("b", b)):
        _dev(t, name, dt, q.shape)
    _dev(v, "v", dt, (B, S, H, Dv))
    _dev(z, "z", dt, q.shape)
    _dev(log_decay, "log_decay", torch.float32, q.shape)
    _dev(initial_state, "initial_state", torch.float32, (B, H, Dk, Dv))
    if out is None:
        out = torch.empty((B, S, H, Dv), dtype=dt, device=q.device)
    if final_state is None:
        final_state = torch.empty((B, H, Dk, Dv), dtype=torch.float32, device=q.device)
    _dev(out, "out", dt, (B, S, H, Dv))
    _dev(final_state, "final_state", torch.float32, (B, H, Dk, Dv))
    args = DplrArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_dtype_code(q), q=_ptr(q), k=_ptr(k), v=_ptr(v),
                    a=_ptr(a), b=_ptr(b), z=_ptr(z), log_decay=_ptr(log_decay), g_min=float(g_min),
                    initial_state=_ptr(initial_state), o=_ptr(out), final_state=_ptr(final_state),
                    stream=_stream(q.device))
    lib = _lib.load()
    if not chunked:
        check("kda_dplr_recurrent_fwd", lib.kda_dplr_recurrent_fwd(ctypes.byref(args)))
        return out, final_state
    n = ctypes.c_size_t(0)
    check("kda_dplr_chunk_workspace_size", lib.kda_dplr_chunk_workspace_size(ctypes.byref(args), ctypes.byref(n)))
    ws = workspace
    if ws is None:
        ws = torch.empty(max(1, n.value), dtype=torch.uint8, device=q.device)
    _dev(ws, "workspace", torch.uint8)
    check("kda_dplr_chunk_fwd", lib.kda_dplr_chunk_fwd(ctypes.byref(args), _ptr(ws), ws.numel()))
    return out, final_state


def decode_step(q, k, v, beta, state, *, z=None, log_decay=None, g_min=-5.0, gate_logits=None, eps=1e-6,
                out=None):
    """One token for B sequences: q,k,z (B,H,D_k); v, gate_logits (B,H,D_v); beta (B,H);
    state (B,H,D_k,D_v) fp32 is advanced IN PLACE.  Returns o (B,H,D_v) in the input dtype."""
    _dev(q, "q")
    dt = q.dtype
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    _dev(k, "k", dt, q.shape)
    _dev(v, "v", dt, (B, H, Dv))
    if beta.dim() == 3 and beta.shape[-1] == 1:
        beta = beta.view(B, H)
    _dev(beta, "beta", dt, (B, H))
    _dev(z, "z", dt, q.shape)
    _dev(log_decay, "log_decay", torch.float32, q.shape)
    _dev(state, "state", torch.float32, (B, H, Dk, Dv))
    _dev(gate_logits, "gate_logits", dt, (B, H, Dv))
    if out is None:
        out = torch.empty((B, H, Dv), dtype=dt, device=q.device)
    _dev(out, "out", dt, (B, H, Dv))
    a = DecodeArgs(B=B, H=H, D_k=Dk, D_v=Dv, dtype=_dtype_code(q), q=_ptr(q), k=_ptr(k), v=_ptr(v),
                   z=_ptr(z), log_decay=_ptr(log_decay), g_min=float(g_min), beta=_ptr(beta),
                   state=_ptr(state), gate_logits=_ptr(gate_logits), eps=float(eps), o=_ptr(out),
                   stream=_stream(q.device))
    check("kda_decode_step", _lib.load().kda_decode_step(ctypes.byref(a)))
    return out


def norm_gate(o, gate_logits, eps=1e-6, out=None):
    """Per-head RMSNorm over D_v then sigmoid gate; o, gate_logits (..., H, D_v)."""
    _dev(o, "o")
    _dev(gate_logits, "gate_logits", o.dtype, o.shape)
    H, Dv = o.shape[-2], o.shape[-1]
    N = o.numel() // (H * Dv)
    if out is None:
        out = torch.empty_like(o)
    _dev(out, "out", o.dtype, o.shape)
    check("kda_norm_gate", _lib.load().kda_norm_gate(_ptr(o), _ptr(gate_logits), N, H, Dv, float(eps),
                                                     _ptr(out), _dtype_code(o), _stream(o.device)))
    return out


def out_proj(x, W_o, out=None):
    """y = x W_o^T with x (..., K) and W_o (D_model, K)."""
    _dev(x, "x")
    Dm, K = W_o.shape
    _dev(W_o, "W_o", x.dtype)
    if x.shape[-1] != K:
        raise ValueError("x's last dimension must equal W_o's second")
    N = x.numel() // K
    if out is None:
        out = torch.empty((*x.shape[:-1], Dm), dtype=x.dtype, device=x.device)
    _dev(out, "out", x.dtype, (*x.shape[:-1], Dm))
    check("kda_out_proj", _lib.load().kda_out_proj(_ptr(x), _ptr(W_o), N, K, Dm, _ptr(out), _dtype_code(x),
                                                   _stream(x.device)))
    return out


def out_norm_gate_proj(o, gate_logits, W_o, eps=1e-6, out=None):
    """y = concat_h(RMSNorm(o_h) * sigmoid(gate_h)) W_o^T; o, gate_logits (..., H, D_v)."""
    _dev(o, "o")
    _dev(gate_logits, "gate_logits", o.dtype, o.shape)
    _dev(W_o, "W_o", o.dtype)
    H, Dv = o.shape[-2], o.shape[-1]
    Dm = W_o.shape[0]
    N = o.numel() // (H * Dv)
    lib = _lib.load()
    n = ctypes.c_size_t(0)
    check("kda_out_norm_gate_proj_workspace_size",
          lib.kda_out_norm_gate_proj_workspace_size(N, H, Dv, _dtype_code(o), ctypes.byref(n)))
    ws = torch.empty(max(n.value, 16), dtype=torch.uint8, device=o.device)
    if out is None:
        out = torch.empty((*o.shape[:-2], Dm), dtype=o.dtype, device=o.device)
    check("kda_out_norm_gate_proj",
          lib.kda_out_norm_gate_proj(_ptr(o), _ptr(gate_logits), _ptr(W_o), N, H, Dv, Dm, float(eps), _ptr(out),
                                     _dtype_code(o), _ptr(ws), n.value, _stream(o.device)))
    return out


def kda_forward(query, key, value, decay_logits, write_strength, output_gate_logits, output_projection,
                initial_state=None, g_min=-5.0, eps=1e-6, *, state_dtype=None, chunk=64, engine="auto",
                outputs=None, final_state_out=None):
    """The KDA layer forward with the "KDA Recurrence" page's interface.

    Returns {"outputs": (B,S,D_model), "final_state": (B,H,D_k,D_v)}, both in the
    input dtype (``state_dtype`` overrides the state's dtype, e.g. torch.float32 to
    keep the library's fp32 state) and on the inputs' device.  CPU inputs are
    copied to the current CUDA device and the results copied back; no input is
    modified.  ``outputs`` / ``final_state_out`` optionally receive the results
    (tensors of the right shape and dtype on the inputs' device, e.g. reused
    pinned host buffers).
    """
    dt = query.dtype
    cpu = not query.is_cuda
    dev = torch.device("cuda", torch.cuda.current_device()) if cpu else query.device

    def up(t, dtype=None):
        if t is None:
            return None
        if t.device != dev:
            t = t.pin_memory().to(dev, non_blocking=True) if cpu else t.to(dev)
        if dtype is not None and t.dtype != dtype:
            t = t.to(dtype)
        return t.contiguous()

    q, k, v, z, gl, W = (up(t) for t in (query, key, value, decay_logits, output_gate_logits, output_projection))
    beta = up(write_strength)
    B, S, H, Dk = q.shape
    beta = beta.reshape(B, S, H)
    s0 = up(initial_state, torch.float32)
    if s0 is not None and s0.data_ptr() == (initial_state.data_ptr() if initial_state is not None else -1):
        s0 = s0.clone()  # never hand the caller's tensor to a kernel that could write it
    x, sf = chunk_fwd(q, k, v, beta, z=z, g_min=g_min, initial_state=s0, gate_logits=gl, eps=eps,
                      chunk=chunk, engine=engine)
    y = out_proj(x.view(B, S, H * v.shape[-1]), W)
    sf = sf.to(state_dtype or dt)

    def dest(given, like, name):
        if given is None:
            return torch.empty(like.shape, dtype=like.dtype, pin_memory=True) if cpu else None
        if tuple(given.shape) != tuple(like.shape) or given.dtype != like.dtype or given.is_cuda == cpu:
            raise ValueError(f"{name} must be a {like.dtype} tensor of shape {tuple(like.shape)} on the inputs' device")
        return given

    y_o, s_o = dest(outputs, y, "outputs"), dest(final_state_out, sf, "final_state_out")
    if cpu:
        y_o.copy_(y, non_blocking=True)
        s_o.copy_(sf, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()
        return {"outputs": y_o, "final_state": s_o}
    if y_o is not None:
        y_o.copy_(y)
        y = y_o
    if s_o is not None:
        s_o.copy_(sf)
        sf = s_o
    return {"outputs": y, "final_state": sf}


def kda_decode(query, key, value, decay_logits, write_strength, output_gate_logits, output_projection, state,
               g_min=-5.0, eps=1e-6):
    """One decode token through the whole layer: q,k,z (B,H,D_k); v, gate (B,H,D_v);
    beta (B,H); state (B,H,D_k,D_v) fp32 advanced in place.  Returns y (B, D_model)."""
    x = decode_step(query, key, value, write_strength, state, z=decay_logits, g_min=g_min,
                    gate_logits=output_gate_logits, eps=eps)
    B, H, Dv = x.shape
    return out_proj(x.view(B, H * Dv), output_projection)
