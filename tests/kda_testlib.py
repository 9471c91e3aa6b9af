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


def upload_by_head(w, device="cuda"):
    """Device tensors in the page's layout, generated one head at a time (host
    memory stays at one head's worth even for the 1M-token workload)."""
    import torch
    dt = torch_dtype(w)
    d = {
        "q": torch.empty((w.B, w.S, w.H, w.Dk), dtype=dt, device=device),
        "k": torch.empty((w.B, w.S, w.H, w.Dk), dtype=dt, device=device),
        "z": torch.empty((w.B, w.S, w.H, w.Dk), dtype=dt, device=device),
        "v": torch.empty((w.B, w.S, w.H, w.Dv), dtype=dt, device=device),
        "gate": torch.empty((w.B, w.S, w.H, w.Dv), dtype=dt, device=device),
        "beta": torch.empty((w.B, w.S, w.H), dtype=dt, device=device),
    }
    s0 = None
    for h in range(w.H):
        hd = ki.head_inputs(w, h)
        for n in ("q", "k", "z", "v", "gate"):
            d[n][:, :, h, :] = torch.from_numpy(hd[n]).to(device).to(dt)
        d["beta"][:, :, h] = torch.from_numpy(hd["beta"]).to(device).to(dt)
        if hd["S0"] is not None:
            if s0 is None:
                s0 = torch.empty((w.B, w.H, w.Dk, w.Dv), dtype=torch.float32, device=device)
            s0[:, h] = torch.from_numpy(hd["S0"]).to(device)
    d["S0"] = s0
    d["W_o"] = to_dev(ki.weights(w), dt, device)
    return d


def oracle_head(w, b, h, t_rec=None, threads=1):
    """Oracle o~ (at t_rec tokens) and final state for one (b, h) of a workload,
    regenerating only that head's inputs."""
    hd = ki.head_inputs(w, h)
    sl = lambda a: a[b:b + 1, :, None, :]
    s0 = None if hd["S0"] is None else hd["S0"][b:b + 1, None]
    o, sf = oracle.recurrence(sl(hd["q"]), sl(hd["k"]), sl(hd["v"]), hd["beta"][b:b + 1, :, None],
                              z=sl(hd["z"]), g_min=w.g_min, initial_state=s0, t_rec=t_rec, threads=threads)
    gate = hd["gate"][b, t_rec if t_rec is not None else slice(None)]
    return o[0, :, 0], sf[0, 0], gate


def oracle_head_dev(w, d, b, h, t_rec=None, threads=1):
    """Oracle o~ (at t_rec tokens), final state and gate logits for one (b, h) of
    device-generated inputs ``d`` (kda_inputs.device_inputs): the device's own
    input bytes are copied to the host and run through the fp64 recurrence."""
    hs = ki.host_slice(d, b, h)
    o, sf = oracle.recurrence(hs["q"], hs["k"], hs["v"], hs["beta"], z=hs["z"], g_min=w.g_min,
                              initial_state=hs["S0"], t_rec=t_rec, threads=threads)
    gate = hs["gate"][0, t_rec if t_rec is not None else slice(None), 0]
    return o[0, :, 0], sf[0, 0], gate


def oracle_heads_dev(w, d, pairs, t_rec=None, workers=None):
    """oracle_head_dev over several (b, h) pairs in parallel host threads (the
    oracle's C recurrence runs without the interpreter lock)."""
    import concurrent.futures as cf
    import os
    workers = workers or max(1, min(len(pairs), len(os.sched_getaffinity(0))))
    with cf.ThreadPoolExecutor(workers) as ex:
        futs = {bh: ex.submit(oracle_head_dev, w, d, bh[0], bh[1], t_rec) for bh in pairs}
        return {bh: f.result() for bh, f in futs.items()}
