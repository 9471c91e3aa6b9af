"""Seeded synthetic inputs for the KDA layer forward.

Shared by the tests, ``bench.py`` and ``__graft_entry__.smoke()``; it holds none
of the layer's arithmetic (no gate, recurrence, normalisation or projection),
only random draws, the per-token L2 normalisation of q and k that defines the
input distribution, and round-to-nearest-even bf16 quantisation.

Every tensor has its own PCG64 sub-stream per head, keyed
``SeedSequence([seed, tensor_id, head])``, so one head of a long workload can be
regenerated on its own (the 1M-token case is generated head by head).

Workloads (shapes and distributions):

=====================  ===================================================
``tiny_fp32``          B1 S64 H2 Dk=Dv=16 D_model 32, fp32, S0 = 0
``prefill_4k``         B1 S4096 H16 D128 D_model 2048, bf16, S0 = 0
``batch_8x8k``         B8 S8192 H32 D128 D_model 4096, bf16, z std 2, S0 = 0
``long_1m``            B1 S1048576 H16 D128 D_model 2048, bf16, S0 ~ N(0, 0.02)
``decode_256``         256 sequences x 128 single-token steps, H32 D128,
                       D_model 4096, S0 ~ N(0, 0.02) fp32 (512 MiB)
=====================  ===================================================

Distributions: q, k ~ N(0,1) then L2-normalised per (token, head); v, decay
logits z and gate logits ~ N(0,1) (z ~ N(0,2) for ``batch_8x8k``);
beta ~ U(0,1); W_o ~ N(0, std 1/sqrt(H*Dv)); g_min = -5, eps = 1e-6.
Values are drawn in fp32 and rounded once to the workload dtype; the device and
the oracle consume the same rounded values.

Two generators draw these distributions:

* ``make_inputs`` / ``head_inputs`` (host, numpy PCG64): the small and
  medium cases the oracle runs in full, and the CPU tests.  For B = 1, the
  first n tokens of a head are the first n draws of its stream
  (``head_inputs(w, h, tokens=n)`` is an exact prefix of the full draw).
* ``device_inputs`` (CUDA, torch's seeded Philox generator): the full-size
  workloads (21.5 GB of bf16 for ``long_1m``), generated on the device in
  under a second.  Its values differ from the host generator's for the same
  seed; whoever compares against the oracle copies the device's own bytes
  back to the host (``host_slice``), so both sides read identical inputs.
"""
from __future__ import annotations

import dataclasses

import numpy as np

TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "z": 4, "beta": 5, "gate": 6, "W_o": 7, "S0": 8}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    H: int
    Dk: int
    Dv: int
    D_model: int
    dtype: str            # "f32" or "bf16"
    seed: int
    z_std: float = 1.0
    s0_std: float = 0.0   # 0 -> zero initial state
    g_min: float = -5.0
    eps: float = 1e-6
    decode_steps: int = 0  # > 0: a decode workload, S is the number of steps

    @property
    def tokens(self) -> int:
        return self.B * self.S


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 64, 2, 16, 16, 32, "f32", 1000),
    "prefill_4k": Workload("prefill_4k", 1, 4096, 16, 128, 128, 2048, "bf16", 1001),
    "batch_8x8k": Workload("batch_8x8k", 8, 8192, 32, 128, 128, 4096, "bf16", 1002, z_std=2.0),
    "long_1m": Workload("long_1m", 1, 1 << 20, 16, 128, 128, 2048, "bf16", 1003, s0_std=0.02),
    "decode_256": Workload("decode_256", 256, 128, 32, 128, 128, 4096, "bf16", 1004,
                           s0_std=0.02, decode_steps=128),
}


def custom(name, B, S, H, Dk, Dv, D_model, dtype="bf16", seed=7, **kw) -> Workload:
    return Workload(name, B, S, H, Dk, Dv, D_model, dtype, seed, **kw)


def _rng(seed: int, tensor: str, head: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, TENSOR_IDS[tensor], head])))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    r = ((b.astype(np.uint64) + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of fp32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _quant(w: Workload, x: np.ndarray) -> np.ndarray:
    return round_bf16(x) if w.dtype == "bf16" else np.ascontiguousarray(x, np.float32)


def _l2n(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def head_inputs(w: Workload, h: int, tokens: int | None = None) -> dict:
    """Per-head tensors (B, S, D) / (B, S) for head h, already rounded.
    ``tokens`` (B = 1 only) draws just the first ``tokens`` tokens: an exact
    prefix of the full draw, because each stream is consumed in token order."""
    S = w.S
    if tokens is not None:
        if w.B != 1:
            raise ValueError("a token prefix is defined for B = 1 only")
        S = min(int(tokens), w.S)
    shp_k = (w.B, S, w.Dk)
    shp_v = (w.B, S, w.Dv)
    out = {
        "q": _quant(w, _l2n(_rng(w.seed, "q", h).standard_normal(shp_k, dtype=np.float32))),
        "k": _quant(w, _l2n(_rng(w.seed, "k", h).standard_normal(shp_k, dtype=np.float32))),
        "v": _quant(w, _rng(w.seed, "v", h).standard_normal(shp_v, dtype=np.float32)),
        "z": _quant(w, np.float32(w.z_std) * _rng(w.seed, "z", h).standard_normal(shp_k, dtype=np.float32)),
        "beta": _quant(w, _rng(w.seed, "beta", h).random((w.B, S), dtype=np.float32)),
        "gate": _quant(w, _rng(w.seed, "gate", h).standard_normal(shp_v, dtype=np.float32)),
    }
    if w.s0_std > 0:
        out["S0"] = (np.float32(w.s0_std) *
                     _rng(w.seed, "S0", h).standard_normal((w.B, w.Dk, w.Dv), dtype=np.float32))
    else:
        out["S0"] = None
    return out


def weights(w: Workload) -> np.ndarray:
    """Output projection W_o, (D_model, H*Dv), rounded to the workload dtype."""
    std = np.float32(1.0 / np.sqrt(w.H * w.Dv))
    return _quant(w, std * _rng(w.seed, "W_o", 0).standard_normal((w.D_model, w.H * w.Dv), dtype=np.float32))


def make_inputs_prefix(w: Workload, tokens: int) -> dict:
    """make_inputs() restricted to the first ``tokens`` tokens (B = 1): the
    same values as the full draw's first tokens, at a fraction of the cost."""
    heads = [head_inputs(w, h, tokens=tokens) for h in range(w.H)]
    out = {}
    for name in ("q", "k", "v", "z", "gate"):
        out[name] = np.stack([hd[name] for hd in heads], axis=2)
    out["beta"] = np.stack([hd["beta"] for hd in heads], axis=2)
    out["S0"] = None if heads[0]["S0"] is None else np.stack([hd["S0"] for hd in heads], axis=1)
    out["W_o"] = weights(w)
    return out


def make_inputs(w: Workload) -> dict:
    """All tensors in the page's layout (fp32 arrays holding dtype-exact values):
    q,k,z (B,S,H,Dk); v, gate (B,S,H,Dv); beta (B,S,H); W_o (D_model,H*Dv);
    S0 (B,H,Dk,Dv) fp32 or None."""
    heads = [head_inputs(w, h) for h in range(w.H)]
    out = {}
    for name in ("q", "k", "v", "z", "gate"):
        out[name] = np.stack([hd[name] for hd in heads], axis=2)
    out["beta"] = np.stack([hd["beta"] for hd in heads], axis=2)
    out["S0"] = None if heads[0]["S0"] is None else np.stack([hd["S0"] for hd in heads], axis=1)
    out["W_o"] = weights(w)
    return out


# ----------------------------------------------------------------------------- device generator

def _device_seed(seed: int, tensor: str) -> int:
    return (int(seed) * 1000003 + TENSOR_IDS[tensor] * 7919) & 0x7FFFFFFFFFFF


def device_inputs(w: Workload, device, slab_tokens: int = 1 << 15) -> dict:
    """All tensors of workload ``w`` drawn on a CUDA device (torch Philox,
    one generator per tensor seeded from (seed, tensor)), in the page's layout
    and the workload dtype (state fp32): q, k, z (B,S,H,Dk); v, gate (B,S,H,Dv);
    beta (B,S,H); W_o (D_model, H*Dv); S0 (B,H,Dk,Dv) or None.  Same
    distributions as make_inputs(); drawn in fp32 slabs of ``slab_tokens``
    tokens, q and k L2-normalised per (token, head), rounded once (RNE)."""
    import torch
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = torch.device(device)
    out = {}
    shapes = {"q": w.Dk, "k": w.Dk, "z": w.Dk, "v": w.Dv, "gate": w.Dv}
    for name, D in shapes.items():
        t = torch.empty((w.B, w.S, w.H, D), dtype=dt, device=dev)
        g = torch.Generator(device=dev)
        g.manual_seed(_device_seed(w.seed, name))
        for b in range(w.B):
            for t0 in range(0, w.S, slab_tokens):
                n = min(slab_tokens, w.S - t0)
                x = torch.randn((n, w.H, D), generator=g, device=dev, dtype=torch.float32)
                if name in ("q", "k"):
                    x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)
                elif name == "z" and w.z_std != 1.0:
                    x = x * w.z_std
                t[b, t0:t0 + n] = x.to(dt)
        out[name] = t
    g = torch.Generator(device=dev)
    g.manual_seed(_device_seed(w.seed, "beta"))
    out["beta"] = torch.rand((w.B, w.S, w.H), generator=g, device=dev, dtype=torch.float32).to(dt)
    g.manual_seed(_device_seed(w.seed, "W_o"))
    std = 1.0 / float(np.sqrt(w.H * w.Dv))
    out["W_o"] = (torch.randn((w.D_model, w.H * w.Dv), generator=g, device=dev, dtype=torch.float32) * std).to(dt)
    if w.s0_std > 0:
        g.manual_seed(_device_seed(w.seed, "S0"))
        out["S0"] = torch.randn((w.B, w.H, w.Dk, w.Dv), generator=g, device=dev, dtype=torch.float32) * w.s0_std
    else:
        out["S0"] = None
    return out


def host_slice(d: dict, b: int, h: int, t0: int = 0, t1: int | None = None) -> dict:
    """One (batch row, head) of device_inputs() output, tokens [t0, t1), copied
    to the host as fp32 numpy arrays shaped for the oracle: q, k, z, v, gate
    (1, n, 1, D); beta (1, n, 1); S0 (1, 1, Dk, Dv) or None; W_o (D_model, H*Dv)."""
    t1 = d["q"].shape[1] if t1 is None else t1
    out = {}
    for name in ("q", "k", "z", "v", "gate"):
        out[name] = d[name][b:b + 1, t0:t1, h:h + 1].float().cpu().numpy()
    out["beta"] = d["beta"][b:b + 1, t0:t1, h:h + 1].float().cpu().numpy()
    out["S0"] = None if d["S0"] is None else d["S0"][b:b + 1, h:h + 1].float().cpu().numpy()
    out["W_o"] = d["W_o"].float().cpu().numpy()
    return out


def host_rows(d: dict, b: int, t0: int, t1: int) -> dict:
    """Tokens [t0, t1) of batch row b, all heads, copied to the host (fp32
    numpy, the oracle's layout with B = 1)."""
    out = {name: d[name][b:b + 1, t0:t1].float().cpu().numpy() for name in ("q", "k", "z", "v", "gate", "beta")}
    out["S0"] = None if d["S0"] is None else d["S0"][b:b + 1].float().cpu().numpy()
    out["W_o"] = d["W_o"].float().cpu().numpy()
    return out
