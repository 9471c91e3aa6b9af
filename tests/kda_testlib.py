"""Helpers shared by the GPU parity tests: upload seeded inputs, run the CUDA
path through the C ABI, run the oracle on the same values, compare."""
from __future__ import annotations

import numpy as np

import kda_inputs as ki
import oracle

# Tolerances fixed for the layer (fp32: the "KDA Recurrence" page's Requirements;
# bf16: max-abs output error and final-state relative Frobenius error).
F32_ATOL, F32_RTOL = 1e-6, 1e-5
BF16_OUT_ATOL = 2e-2
BF16_STATE_RELFRO = 1e-2


def torch_dtype(w):
    import torch
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def to_dev(a, dtype, device="cuda"):
    import torch
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    return t.to(dtype).contiguous()


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_f32_close(got, want, what=""):
    np.testing.assert_allclose(got, want, atol=F32_ATOL, rtol=F32_RTOL, err_msg=what)


def assert_bf16_outputs(got, want, what=""):
    err = float(np.max(np.abs(np.asarray(got) - np.asarray(want)))) if np.size(want) else 0.0
    assert err <= BF16_OUT_ATOL, f"{what}: max-abs error {err:.3e} > {BF16_OUT_ATOL}"


def assert_bf16_state(got, want, what=""):
    e = rel_fro(got, want)
    assert e <= BF16_STATE_RELFRO, f"{what}: relative Frobenius error {e:.3e} > {BF16_STATE_RELFRO}"


def upload(inp, w):
    """Device copies of make_inputs() output in the workload dtype (state fp32)."""
    import torch
    dt = torch_dtype(w)
    d = {n: to_dev(inp[n], dt) for n in ("q", "k", "v", "z", "beta", "gate", "W_o")}
    d["S0"] = to_dev(inp["S0"], torch.float32)
    return d


def oracle_layer(inp, w, threads=None):
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["z"], inp["beta"], inp["gate"], inp["W_o"],
                          inp["S0"], g_min=w.g_min, eps=w.eps, threads=threads)


def small(name, B, S, H, Dk, Dv, Dm, dtype, seed, **kw):
    return ki.custom(name, B, S, H, Dk, Dv, Dm, dtype, seed=seed, **kw)
