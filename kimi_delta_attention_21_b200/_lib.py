"""ctypes view of libkda.so (the C ABI declared in include/kda.h).

Loading fails loudly: there is no fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# KDA_LIBRARY picks another in-tree build of the same ABI by file name (libkda_checked.so: the
# bounds-checked build); absent, the library is libkda.so
LIB_PATH = os.path.join(_HERE, os.path.basename(os.environ.get("KDA_LIBRARY", "libkda.so")))

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(6)
KDA_F32, KDA_BF16 = 0, 1
ENGINE_AUTO, ENGINE_SIMT, ENGINE_TC = 0, 1, 2

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_f32 = ctypes.c_float


class ChunkArgs(ctypes.Structure):
    _fields_ = [
        ("B", _i64), ("S", _i64),
        ("H", _i32), ("D_k", _i32), ("D_v", _i32),
        ("dtype", ctypes.c_int),
        ("q", _p), ("k", _p), ("v", _p), ("z", _p), ("log_decay", _p),
        ("g_min", _f32),
        ("beta", _p), ("initial_state", _p), ("gate_logits", _p),
        ("eps", _f32),
        ("o", _p), ("final_state", _p),
        ("workspace", _p), ("workspace_bytes", ctypes.c_size_t),
        ("chunk", _i32), ("engine", ctypes.c_int),
        ("dev_status", _p), ("stream", _p),
    ]


class RecBwdArgs(ctypes.Structure):
    _fields_ = [
        ("B", _i64), ("S", _i64),
        ("H", _i32), ("D_k", _i32), ("D_v", _i32),
        ("dtype", ctypes.c_int),
        ("q", _p), ("k", _p), ("v", _p), ("z", _p), ("log_decay", _p),
        ("g_min", _f32),
        ("beta", _p), ("initial_state", _p), ("d_o", _p), ("d_final_state", _p),
        ("dq", _p), ("dk", _p), ("dv", _p), ("dbeta", _p), ("dz", _p), ("d_initial_state", _p),
        ("workspace", _p), ("workspace_bytes", ctypes.c_size_t),
        ("stream", _p),
    ]


class DplrArgs(ctypes.Structure):
    _fields_ = [
        ("B", _i64), ("S", _i64),
        ("H", _i32), ("D_k", _i32), ("D_v", _i32),
        ("dtype", ctypes.c_int),
        ("q", _p), ("k", _p), ("v", _p), ("a", _p), ("b", _p), ("z", _p), ("log_decay", _p),
        ("g_min", _f32),
        ("initial_state", _p), ("o", _p), ("final_state", _p), ("stream", _p),
    ]


class DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("B", _i64),
        ("H", _i32), ("D_k", _i32), ("D_v", _i32),
        ("dtype", ctypes.c_int),
        ("q", _p), ("k", _p), ("v", _p), ("z", _p), ("log_decay", _p),
        ("g_min", _f32),
        ("beta", _p), ("state", _p), ("gate_logits", _p),
        ("eps", _f32),
        ("o", _p), ("stream", _p),
    ]


# name -> (restype, argtypes); every symbol declared in include/kda.h
SIGNATURES = {
    "kda_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kda_last_error": (ctypes.c_char_p, []),
    "kda_version": (ctypes.c_int, []),
    "kda_launch_count": (ctypes.c_uint64, []),
    "kda_device_timeouts": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]),
    "kda_device_bounds_errors": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, _p]),
    "kda_selftest_wait_timeout": (ctypes.c_int, [_p, ctypes.c_uint32, _p]),
    "kda_gate": (ctypes.c_int, [_p, ctypes.c_int, _i64, _f32, _p, _p]),
    "kda_chunk_workspace_size": (ctypes.c_int, [ctypes.POINTER(ChunkArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "kda_chunk_fwd": (ctypes.c_int, [ctypes.POINTER(ChunkArgs)]),
    "kda_gdn_chunk_workspace_size": (ctypes.c_int, [ctypes.POINTER(ChunkArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "kda_gdn_chunk_fwd": (ctypes.c_int, [ctypes.POINTER(ChunkArgs)]),
    "kda_decode_step": (ctypes.c_int, [ctypes.POINTER(DecodeArgs)]),
    "kda_recurrent_bwd_workspace_size": (ctypes.c_int, [ctypes.POINTER(RecBwdArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "kda_recurrent_bwd": (ctypes.c_int, [ctypes.POINTER(RecBwdArgs)]),
    "kda_chunk_bwd_workspace_size": (ctypes.c_int, [ctypes.POINTER(RecBwdArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "kda_chunk_bwd": (ctypes.c_int, [ctypes.POINTER(RecBwdArgs)]),
    "kda_dplr_recurrent_fwd": (ctypes.c_int, [ctypes.POINTER(DplrArgs)]),
    "kda_dplr_chunk_workspace_size": (ctypes.c_int, [ctypes.POINTER(DplrArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "kda_dplr_chunk_fwd": (ctypes.c_int, [ctypes.POINTER(DplrArgs), ctypes.c_void_p, ctypes.c_size_t]),
    "kda_norm_gate": (ctypes.c_int, [_p, _p, _i64, _i32, _i32, _f32, _p, ctypes.c_int, _p]),
    "kda_out_proj": (ctypes.c_int, [_p, _p, _i64, _i32, _i32, _p, ctypes.c_int, _p]),
    "kda_out_norm_gate_proj_workspace_size": (ctypes.c_int, [_i64, _i32, _i32, ctypes.c_int,
                                                             ctypes.POINTER(ctypes.c_size_t)]),
    "kda_out_norm_gate_proj": (ctypes.c_int, [_p, _p, _p, _i64, _i32, _i32, _i32, _f32, _p, ctypes.c_int,
                                              _p, ctypes.c_size_t, _p]),
    "kda_out_norm_gate_proj_noalloc": (ctypes.c_int, [_p, _p, _p, _i64, _i32, _i32, _i32, _f32, _p, ctypes.c_int,
                                                      _p]),
}

_lib = None


def load():
    """Load libkda.so and bind every exported entry point (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m kimi_delta_attention_21_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


class KDAError(RuntimeError):
    def __init__(self, fn, status, msg):
        self.status = status
        super().__init__(f"{fn}: {_name(status)}: {msg}")


def _name(status):
    lib = load()
    return lib.kda_status_string(status).decode()


def check(fn, status):
    if status != KDA_OK:
        raise KDAError(fn, status, load().kda_last_error().decode())
