"""The no-allocation variant of the norm + gate + projection step.

Callers that cannot allocate device memory (an integration point that passes
only input and output buffers, or a loop that must not call cudaMalloc while it
runs) use kda_out_norm_gate_proj_noalloc, which keeps its intermediate in a
fixed scratch array inside the library.  Its results must match the
workspace-based entry point on two calls in a row (the second call finds the
first call's data still in the shared scratch array).  Collected last on
purpose.
"""
import ctypes

import numpy as np
import pytest

import kda_inputs as ki
from kda_testlib import to_dev, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(N, H, Dv, Dm, dtype, seed):
    rng = np.random.default_rng(seed)
    o = rng.standard_normal((N, H, Dv)).astype(np.float32)
    gl = rng.standard_normal((N, H, Dv)).astype(np.float32)
    W = (rng.standard_normal((Dm, H * Dv)) / np.sqrt(H * Dv)).astype(np.float32)
    if dtype == torch.bfloat16:
        o, gl, W = ki.round_bf16(o), ki.round_bf16(gl), ki.round_bf16(W)
    return to_dev(o, dtype), to_dev(gl, dtype), to_dev(W, dtype)


def _both(lib, o, gl, W, eps=1e-6):
    from kimi_delta_attention_21_b200 import _lib
    N, H, Dv = o.shape
    Dm = W.shape[0]
    code = _lib.KDA_F32 if o.dtype == torch.float32 else _lib.KDA_BF16
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    n = ctypes.c_size_t(0)
    assert lib.kda_out_norm_gate_proj_workspace_size(N, H, Dv, code, ctypes.byref(n)) == 0
    ws = torch.empty(max(n.value, 16), dtype=torch.uint8, device="cuda")
    y_ref = torch.empty((N, Dm), dtype=o.dtype, device="cuda")
    y_new = torch.full((N, Dm), float("nan"), dtype=o.dtype, device="cuda")
    assert lib.kda_out_norm_gate_proj(_ptr(o), _ptr(gl), _ptr(W), N, H, Dv, Dm, eps, _ptr(y_ref), code,
                                      _ptr(ws), n.value, stream) == 0
    st = lib.kda_out_norm_gate_proj_noalloc(_ptr(o), _ptr(gl), _ptr(W), N, H, Dv, Dm, eps, _ptr(y_new), code, stream)
    assert st == 0, lib.kda_last_error().decode()
    torch.cuda.synchronize()
    return to_np(y_ref), to_np(y_new)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    from kimi_delta_attention_21_b200 import _lib
    lib = _lib.load()
    # two calls in a row with different shapes: the second reuses the scratch
    # the first one filled
    for call, (N, H, Dv, Dm) in enumerate([(512, 16, 128, 256), (300, 8, 64, 136)]):
        o, gl, W = _inputs(N, H, Dv, Dm, dtype, seed=100 + call)
        y_ref, y_new = _both(lib, o, gl, W)
        assert np.all(np.isfinite(y_new))
        # the same kernels on the same inputs: the results are identical bit for bit
        assert np.array_equal(y_new, y_ref), float(np.max(np.abs(y_new - y_ref)))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from kimi_delta_attention_21_b200 import _lib
    lib = _lib.load()
    H, Dv, Dm = 16, 128, 64
    N = SCRATCH_BYTES // (H * Dv * 2) + 1      # one row too many in bf16
    o = torch.zeros((N, H, Dv), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((Dm, H * Dv), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((N, Dm), dtype=torch.bfloat16, device="cuda")
    n0 = lib.kda_launch_count()
    st = lib.kda_out_norm_gate_proj_noalloc(_ptr(o), _ptr(o), _ptr(W), N, H, Dv, Dm, 1e-6, _ptr(y), _lib.KDA_BF16,
                                            None)
    assert st == _lib.KDA_ERR_UNSUPPORTED
    assert "scratch" in lib.kda_last_error().decode()
    assert lib.kda_launch_count() == n0        # nothing launched


def test_noalloc_clears_the_previous_error_message():
    from kimi_delta_attention_21_b200 import _lib
    lib = _lib.load()
    assert lib.kda_gate(None, _lib.KDA_BF16, 4, -5.0, None, None) != 0      # leaves a message behind
    assert lib.kda_last_error().decode() != ""
    o, gl, W = _inputs(8, 2, 64, 16, torch.bfloat16, seed=3)
    y = torch.empty((8, 16), dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.kda_out_norm_gate_proj_noalloc(_ptr(o), _ptr(gl), _ptr(W), 8, 2, 64, 16, 1e-6, _ptr(y),
                                              _lib.KDA_BF16, stream) == 0
    assert lib.kda_last_error().decode() == ""
