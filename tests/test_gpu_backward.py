"""The recurrent backward (kda_recurrent_bwd) and the chunkwise backward
(kda_chunk_bwd) against the oracle's gradient of the recurrence, which finite
differences pin: every input's gradient, with and without an initial state and
a final-state gradient, for z and log-decay inputs, fp32 and bf16 inputs,
across several chunks with a ragged tail; plus guard bands around every
gradient output and the workspace."""
import numpy as np
import pytest

import kda_inputs as ki
import oracle
from kda_testlib import small, to_dev, to_np, upload

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dbeta", "dz", "d_initial_state")


@pytest.fixture(scope="module")
def K():
    import kimi_delta_attention_21_b200 as K
    K.load_library()
    return K


def _close(got, want, what):
    # fp32 arithmetic on both sides' inputs (bf16 inputs are exact in fp32): sums of O(S) terms
    scale = max(1.0, float(np.max(np.abs(want))))
    err = float(np.max(np.abs(got - want))) if want.size else 0.0
    assert err <= 2e-4 * scale, f"{what}: max-abs error {err:.3e} (scale {scale:.3e})"


ENGINES = ("recurrent_bwd", "chunk_bwd")


def _run(K, w, seed, with_s0, with_dst, use_log, engine="recurrent_bwd"):
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    rng = np.random.default_rng(seed)
    dO = rng.standard_normal((w.B, w.S, w.H, w.Dv)).astype(np.float32)
    if w.dtype == "bf16":
        dO = ki.round_bf16(dO)
    dst = rng.standard_normal((w.B, w.H, w.Dk, w.Dv)).astype(np.float32) if with_dst else None
    s0 = inp["S0"] if with_s0 else None
    kw_dev, kw_ref = {}, {}
    if use_log:
        ld = oracle.log_decay(inp["z"], w.g_min).astype(np.float32)
        kw_dev["log_decay"], kw_ref["log_decay"] = to_dev(ld, torch.float32), ld
    else:
        kw_dev["z"], kw_ref["z"] = d["z"], inp["z"]
    got = getattr(K, engine)(d["q"], d["k"], d["v"], d["beta"], to_dev(dO, d["q"].dtype), g_min=w.g_min,
                          initial_state=d["S0"] if with_s0 else None,
                          d_final_state=to_dev(dst, torch.float32), **kw_dev)
    torch.cuda.synchronize()
    want = oracle.recurrence_bwd(inp["q"], inp["k"], inp["v"], inp["beta"], dO, g_min=w.g_min, initial_state=s0,
                                 d_final_state=dst, **kw_ref)
    return got, want


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("B,S,H,D,dtype", [(1, 1, 1, 16, "f32"), (2, 63, 2, 16, "f32"), (1, 130, 3, 24, "f32"),
                                           (2, 200, 2, 40, "f32"), (2, 300, 3, 128, "bf16"), (1, 129, 2, 128, "f32")])
def test_backward_matches_oracle(K, engine, B, S, H, D, dtype):
    w = small("bwd", B, S, H, D, D, 16, dtype, seed=S + D, s0_std=0.05)
    got, want = _run(K, w, seed=S, with_s0=True, with_dst=True, use_log=False, engine=engine)
    for n in NAMES:
        _close(to_np(got[n]), want[n], f"{engine} {n} (B{B} S{S} H{H} D{D} {dtype})")


@pytest.mark.parametrize("B,S,H,Dk,Dv,dtype", [(1, 200, 2, 32, 128, "bf16"), (2, 70, 1, 128, 20, "f32"),
                                               (1, 100, 2, 18, 13, "f32"), (1, 640, 2, 128, 128, "bf16")])
def test_chunk_backward_unequal_heads_and_long(K, B, S, H, Dk, Dv, dtype):
    """D_k != D_v (value slices of 16 with a ragged last one; sizes that are not multiples of 4, which
    take the element-wise copies), and ten chunks of 64 at D = 128."""
    w = small("bwdc", B, S, H, Dk, Dv, 16, dtype, seed=S + Dk, s0_std=0.05)
    got, want = _run(K, w, seed=S + 1, with_s0=True, with_dst=True, use_log=False, engine="chunk_bwd")
    for n in NAMES:
        _close(to_np(got[n]), want[n], f"chunk_bwd {n} (B{B} S{S} H{H} Dk{Dk} Dv{Dv} {dtype})")


@pytest.mark.parametrize("engine", ENGINES)
def test_backward_log_decay_no_state(K, engine):
    w = small("bwdl", 1, 150, 2, 32, 20, 16, "f32", seed=3, s0_std=0.0)
    got, want = _run(K, w, seed=4, with_s0=False, with_dst=False, use_log=True, engine=engine)
    for n in ("dq", "dk", "dv", "dbeta", "d_initial_state"):
        _close(to_np(got[n]), want[n], n)
    _close(to_np(got["dlog_decay"]), want["dlog_decay"], "dlog_decay")


@pytest.mark.parametrize("engine", ENGINES)
def test_backward_writes_stay_inside(K, engine):
    from test_gpu_guard_bands import Guarded
    w = small("bwdg", 2, 100, 3, 48, 40, 16, "bf16", seed=8, s0_std=0.05)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    dO = to_dev(ki.round_bf16(np.ones((w.B, w.S, w.H, w.Dv), np.float32)), torch.bfloat16)
    ref = getattr(K, engine)(d["q"], d["k"], d["v"], d["beta"], dO, z=d["z"], g_min=w.g_min, initial_state=d["S0"])
    import ctypes
    from kimi_delta_attention_21_b200 import _lib
    lib = _lib.load()
    shapes = {"dq": (w.B, w.S, w.H, w.Dk), "dk": (w.B, w.S, w.H, w.Dk), "dv": (w.B, w.S, w.H, w.Dv),
              "dbeta": (w.B, w.S, w.H), "dz": (w.B, w.S, w.H, w.Dk), "d_initial_state": (w.B, w.H, w.Dk, w.Dv)}
    guards = {n: Guarded(int(np.prod(s)) * 4) for n, s in shapes.items()}
    views = {n: g.view(torch.float32, shapes[n]) for n, g in guards.items()}
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    a = _lib.RecBwdArgs(B=w.B, S=w.S, H=w.H, D_k=w.Dk, D_v=w.Dv, dtype=_lib.KDA_BF16, q=p(d["q"]), k=p(d["k"]),
                        v=p(d["v"]), z=p(d["z"]), log_decay=None, g_min=w.g_min, beta=p(d["beta"]),
                        initial_state=p(d["S0"]), d_o=p(dO), d_final_state=None, dq=p(views["dq"]),
                        dk=p(views["dk"]), dv=p(views["dv"]), dbeta=p(views["dbeta"]), dz=p(views["dz"]),
                        d_initial_state=p(views["d_initial_state"]), workspace=None, workspace_bytes=0,
                        stream=ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    n = ctypes.c_size_t(0)
    entry = "kda_" + engine
    assert getattr(lib, entry + "_workspace_size")(ctypes.byref(a), ctypes.byref(n)) == 0
    gw = Guarded(n.value)
    a.workspace = p(gw.bytes_view())
    a.workspace_bytes = n.value
    assert getattr(lib, entry)(ctypes.byref(a)) == 0, lib.kda_last_error().decode()
    for name, g in guards.items():
        g.check(f"{engine} {name}")
    gw.check(f"{engine} workspace")
    for name in shapes:   # the same call through the binding (atomic sums: equal up to fp32 rounding order)
        _close(to_np(views[name]), to_np(ref[name]), f"guarded {name}")
