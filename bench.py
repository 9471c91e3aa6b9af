#!/usr/bin/env python
"""Throughput of the KDA layer forward on B200: chunkwise prefill and the
single-token decode step, with roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one process per GPU)

Without a launcher, ``--gpus N`` (N > 1) starts the N rank processes itself.

One step = one whole layer forward (chunk engine with the gate, the fused
RMSNorm and sigmoid gate, then the output projection) over one batch of a
workload, inputs resident in HBM, a 256 MiB L2 flush between steps.  The
headline (top-level ``value``) is the largest single-GPU prefill workload,
``long_1m`` (B1 S1,048,576 H16 D128, D_model 2048, bf16, fp32 state from
S0 ~ N(0, 0.02)); ``batch_8x8k``, ``prefill_4k`` and the decode engine on
``decode_256`` are timed in the same run and reported under ``workloads``.
Each rank runs its own independently seeded batch (weak scaling, no
collective on the data path).  Rank 0 prints one JSON line.

Rooflines follow the layer's arithmetic: the chunk engine's fraction is
max(FLOPs / peak FLOP/s, bytes / peak bandwidth) / time with algorithmic
FLOPs and bytes; the layer's adds the projection's FLOPs and output bytes.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
headline workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import socket
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import kda_inputs as ki  # noqa: E402

METRIC = "KDA tokens/s (chunk prefill, decode) on 1 B200; % of tensor/HBM roofline"
HEADLINE = "long_1m"
PREFILL_EXTRA = ("batch_8x8k", "prefill_4k")
DECODE = "decode_256"
ALL_WORKLOADS = (HEADLINE,) + PREFILL_EXTRA + (DECODE,)
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
REF_SAMPLE_TOKENS = 512   # tokens (all heads) per reference-arm step
CHUNK = 64

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one chunk-engine
# call or one decode step, from an ncu capture of the named kernels on the
# named workload, valid only while the kernel source is unchanged (sha256
# prefix of the listed files).  "units" marks a figure taken on a smaller
# workload, scaled by the number of (batch, head, chunk) units of the one timed.
_CHUNK_SRC = {"kimi_delta_attention_21_b200/csrc/chunk_tc.cu": "be071728e8f1c356",
              "kimi_delta_attention_21_b200/csrc/tc_common.cuh": "3897eb1336479212",
              "kimi_delta_attention_21_b200/csrc/sm100_ptx.cuh": "b75f6e1e7fa94863"}
NCU_TRAFFIC = {
    # chunk engine (prep, map pass, combine, chain pass) on prefill_4k, 1,024 units, captured as is
    "chunk_engine@prefill_4k": {"bytes": 249097941, "units": 1024, "src_sha": _CHUNK_SRC},
    # long_1m: the prep and the chain pass of that capture, scaled by units (both move the same bytes per
    # unit at any length); its map pass runs windows of a few dozen chunks per segment and its combine
    # eight steps per head, together under 0.1% of the total, and are left out; none for batch_8x8k,
    # whose single segment runs no map pass
    "chunk_engine@long_1m": {"bytes": 194046762, "units": 1024, "src_sha": _CHUNK_SRC},
    "decode@decode_256": {"bytes": 1024257664,
                          "src_sha": {"kimi_delta_attention_21_b200/csrc/decode.cu": "88b9a3ab7b5af3e2",
                                      "kimi_delta_attention_21_b200/csrc/sm100_ptx.cuh": "b75f6e1e7fa94863"}},
}


# ----------------------------------------------------------------------------- helpers

def src_sha(relpath):
    with open(os.path.join(ROOT, relpath), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(key, units=None):
    """Per-call DRAM bytes for `key` if its sources are unchanged since the capture, else None."""
    rec = NCU_TRAFFIC.get(key)
    if not rec or any(src_sha(p) != h for p, h in rec["src_sha"].items()):
        return None
    if "units" in rec and units is not None:
        return int(round(rec["bytes"] * units / rec["units"]))
    return rec["bytes"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def n_chunks(w):
    return (w.S + CHUNK - 1) // CHUNK


def prefill_bytes(w, scalar_decay=False):
    """Algorithmic HBM bytes of the chunk engine for a whole workload: read q, k,
    z (D_k each; one value for the scalar-decay GDN case), v, gate (D_v each) and
    beta per token-head, write the gated output (D_v) per token-head; read the
    fp32 initial state (when there is one) and write the fp32 final state per
    (b, h)."""
    es = 2 if w.dtype == "bf16" else 4
    per_tok_head = es * ((2 * w.Dk + (1 if scalar_decay else w.Dk)) + 3 * w.Dv + 1)
    n_states = 2 if w.s0_std > 0 else 1
    return w.B * w.S * w.H * per_tok_head + n_states * w.B * w.H * w.Dk * w.Dv * 4


def chunk_flops(w, C=CHUNK):
    """Algorithmic tensor FLOPs of the chunkwise prefill (2 per multiply-add), per chunk of C tokens:
    the causal intra-chunk products A = (beta K) K^T and M = Q K^T, the UT-transform products
    W = T (beta K e^G) and U = T (beta V) and the intra-chunk output M V' (lower triangles: C^2 D
    each), and the three state products W S, (Q e^G) S and K~^T V' (2 C D_k D_v each).  The
    triangular solve itself is not counted."""
    per_chunk = C * C * (2 * w.Dk + w.Dk + 2 * w.Dv) + 3 * 2 * C * w.Dk * w.Dv
    return w.B * w.H * n_chunks(w) * per_chunk


def proj_flops(n_rows, w):
    return 2.0 * n_rows * w.H * w.Dv * w.D_model


def layer_bytes(w):
    """Algorithmic HBM bytes of the whole layer: the chunk engine's inputs and
    states, W_o once, and the projected output y (N x D_model)."""
    es = 2 if w.dtype == "bf16" else 4
    core = prefill_bytes(w) - w.B * w.S * w.H * w.Dv * es   # o is an intermediate of the layer
    return core + w.D_model * w.H * w.Dv * es + w.B * w.S * w.D_model * es


def decode_bytes(w):
    """Algorithmic HBM bytes of one decode step: the fp32 state read and written
    once, q, k, z, v, gate and beta read, the gated output written."""
    es = 2 if w.dtype == "bf16" else 4
    per_bh = 2 * w.Dk * w.Dv * 4 + es * (3 * w.Dk + 3 * w.Dv + 1)
    return w.B * w.H * per_bh


def roofline(flops, nbytes, seconds, peaks, tensor_peak_key="bf16_tflops"):
    """max(flop time, byte time) at the peaks over the measured time.  `bound` is
    the roof that sets the floor; `achieved` is in that roof's unit."""
    t_flop = flops / (peaks[tensor_peak_key] * 1e12)
    t_byte = nbytes / (peaks["hbm_gbs"] * 1e9)
    if t_byte >= t_flop:
        out = {"bound": "hbm", "achieved": round(nbytes / seconds / 1e9, 1), "peak": peaks["hbm_gbs"],
               "unit": "GB/s"}
    else:
        out = {"bound": "tensor", "achieved": round(flops / seconds / 1e12, 2), "peak": peaks[tensor_peak_key],
               "unit": "TFLOP/s"}
    out["frac"] = round(max(t_flop, t_byte) / seconds, 4)
    out.update({"algorithmic_flops": int(flops), "algorithmic_bytes": int(nbytes),
                "flop_time_ms": round(t_flop * 1e3, 4), "byte_time_ms": round(t_byte * 1e3, 4),
                "ms": round(seconds * 1e3, 4),
                "tensor_achieved_tflops": round(flops / seconds / 1e12, 2),
                "tensor_frac": round(flops / seconds / 1e12 / peaks[tensor_peak_key], 4),
                "hbm_achieved_gbs": round(nbytes / seconds / 1e9, 1),
                "hbm_frac": round(nbytes / seconds / 1e9 / peaks["hbm_gbs"], 4)})
    return out


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.01):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
            return self
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def _run(self):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(values, world, device=None):
    """Element-wise max over ranks of a list of floats (identity at world 1)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_workload(name, rank):
    """Each rank runs an independent batch: same shapes, its own seed."""
    w = ki.WORKLOADS[name]
    if rank == 0:
        return w
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 7919 * rank)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_entry(rank, argv, world, port):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), LOCAL_WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    rc = main(argv)
    if rc:
        raise SystemExit(rc)


def launch_ranks(argv, world):
    """Start `world` rank processes on this node (one per GPU), each running
    main(argv) with RANK / LOCAL_RANK / WORLD_SIZE set, and wait for all of
    them; a failing rank fails the launch."""
    import torch.multiprocessing as mp
    mp.start_processes(_rank_entry, args=(list(argv), world, _free_port()), nprocs=world, join=True,
                       start_method="spawn")
    return 0


# ----------------------------------------------------------------------------- our arm

class Timer:
    """CUDA events around the chunk-engine call and the projection of each step."""

    def __init__(self, torch, n):
        self.ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]

    def means(self):
        n = len(self.ev)
        a = sum(e[0].elapsed_time(e[1]) for e in self.ev) / n * 1e-3
        b = sum(e[1].elapsed_time(e[2]) for e in self.ev) / n * 1e-3
        return a, b


def time_prefill(K, torch, w, d, steps, warmup, world, dev, flush, lib, sampler=None, gdn=False, engine="auto"):
    """Times `steps` layer forwards of workload `w` (device inputs `d`).  Returns
    per-step seconds (chunk engine, projection; max over ranks) and launches.
    gdn: the scalar-decay (Gated DeltaNet) engine, one decay logit per token and
    head (the first channel's logit of the same inputs).  engine: "auto" (the
    tensor-core engine inside its envelope) or "simt" (the exact engine the
    library falls back to outside it)."""
    B, S, H = w.B, w.S, w.H
    N = B * S
    x = torch.empty((B, S, H, w.Dv), dtype=d["v"].dtype, device=dev)
    y = torch.empty((N, w.D_model), dtype=d["v"].dtype, device=dev)
    sf = torch.empty((B, H, w.Dk, w.Dv), dtype=torch.float32, device=dev)
    ws = torch.empty(K.chunk_workspace_bytes(B, S, H, w.Dk, w.Dv, scalar_decay=gdn, engine=engine), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    z = d["z"][..., 0].contiguous() if gdn else d["z"]

    def chunk():
        K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=z, g_min=w.g_min, initial_state=d["S0"],
                    gate_logits=d["gate"], eps=w.eps, out=x, final_state=sf, workspace=ws, scalar_decay=gdn,
                    engine=engine)

    def proj():
        K.out_proj(x.view(N, H * w.Dv), d["W_o"], out=y)

    for _ in range(warmup):
        flush.fill_(1.0)
        chunk()
        proj()
    torch.cuda.synchronize(dev)
    tm = Timer(torch, steps)
    barrier(world)
    torch.cuda.synchronize(dev)
    n0 = lib.kda_launch_count()
    t_wall0 = time.perf_counter()
    if sampler is not None:
        sampler.__enter__()
    for i in range(steps):
        flush.fill_(float(i))
        tm.ev[i][0].record(stream)
        chunk()
        tm.ev[i][1].record(stream)
        proj()
        tm.ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    if sampler is not None:
        sampler.__exit__(None, None, None)
    barrier(world)
    t_wall = time.perf_counter() - t_wall0
    launches = lib.kda_launch_count() - n0
    t_chunk, t_proj = tm.means()
    t_step_max, t_chunk_max, t_proj_max = reduce_max([t_chunk + t_proj, t_chunk, t_proj], world, dev)
    del x, y, sf, ws, z
    return {"t_step": t_step_max, "t_chunk": t_chunk_max, "t_proj": t_proj_max, "launches": launches,
            "wall": t_wall}


def prefill_record(w, tm, peaks, world, traffic_key):
    N = w.B * w.S
    units = w.B * w.H * n_chunks(w)
    chunk = roofline(chunk_flops(w), prefill_bytes(w), tm["t_chunk"], peaks)
    chunk["kernel"] = "kda_chunk_fwd (chunk engine: prep, segment maps, combine, segment chains)"
    chunk["traffic"] = traffic_for(traffic_key, units)
    layer = roofline(chunk_flops(w) + proj_flops(N, w), layer_bytes(w), tm["t_step"], peaks)
    layer_s = roofline(chunk_flops(w) + proj_flops(N, w), layer_bytes(w), tm["t_step"], peaks,
                       "bf16_tflops_sustained")
    layer["kernel"] = "layer forward (kda_chunk_fwd + kda_out_proj)"
    layer["frac_vs_sustained_tensor_peak"] = layer_s["frac"]
    proj_t = proj_flops(N, w) / tm["t_proj"] / 1e12
    return {
        "workload": w.name, "value": round(N * world / tm["t_step"], 1), "unit": "tokens/s",
        "ms_per_step": round(tm["t_step"] * 1e3, 4),
        "config": {"B": w.B, "S": w.S, "H": w.H, "D_k": w.Dk, "D_v": w.Dv, "D_model": w.D_model, "chunk": CHUNK,
                   "g_min": w.g_min, "z_std": w.z_std, "initial_state": f"N(0, {w.s0_std})" if w.s0_std else "zeros",
                   "state": "fp32", "units_b_h_chunk": units},
        "kernels_ms": {"chunk_engine": round(tm["t_chunk"] * 1e3, 4), "out_proj": round(tm["t_proj"] * 1e3, 4)},
        "roofline": chunk,
        "layer_roofline": layer,
        "out_proj": {"achieved_tflops": round(proj_t, 1), "frac": round(proj_t / peaks["bf16_tflops"], 4)},
        "chunk_engine_tokens_per_s": round(N * world / tm["t_chunk"], 1),
    }


def cpu_baseline_prefill(w, d, target_s):
    """The oracle as it stands, on this host's cores, on the first n tokens of
    batch row 0 (all heads) of the same device-generated inputs: fp64
    recurrence + norm/gate + projection.  n is calibrated so that the timed
    call takes about `target_s` seconds."""
    import oracle
    cores = oracle.default_threads()

    def run(n):
        h = ki.host_rows(d, 0, 0, n)
        t0 = time.perf_counter()
        oracle.forward(h["q"], h["k"], h["v"], h["z"], h["beta"], h["gate"], h["W_o"], h["S0"],
                       g_min=w.g_min, eps=w.eps, threads=cores)
        return time.perf_counter() - t0

    n = min(w.S, 256)
    dt = run(n)
    n = int(min(w.S, max(n, n * target_s / max(dt, 1e-3))))
    dt = run(n)
    return {"value": round(n / dt, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} of {w.S} tokens x {w.H} heads of batch row 0 of {w.name} (same device-generated "
                      f"inputs, copied to the host): fp64 recurrence + norm/gate + projection, {dt:.2f} s"}


def cpu_baseline_decode(w, d, target_s):
    """The oracle on the first m sequences (all heads, all decode steps) of the
    decode workload: its recurrence over the steps from each sequence's state."""
    import oracle
    cores = oracle.default_threads()

    def run(m):
        h = {n: d[n][:m].float().cpu().numpy() for n in ("q", "k", "z", "v", "gate", "beta")}
        s0 = d["S0"][:m].float().cpu().numpy()
        W = d["W_o"].float().cpu().numpy()
        t0 = time.perf_counter()
        oracle.forward(h["q"], h["k"], h["v"], h["z"], h["beta"], h["gate"], W, s0, g_min=w.g_min, eps=w.eps,
                       threads=cores)
        return time.perf_counter() - t0

    m = 2
    dt = run(m)
    m = int(min(w.B, max(m, m * target_s / max(dt, 1e-3))))
    dt = run(m)
    return {"value": round(m * w.S / dt, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{m} of {w.B} sequences x {w.H} heads x {w.S} decode steps of {w.name} (same device-generated "
                      f"inputs): fp64 recurrence + norm/gate + projection, {dt:.2f} s"}


def run_e2e(K, torch, w, d, steps, world, dev):
    """The headline metric through the public API with HOST buffers: every step
    copies the step's inputs from pinned host memory to the device, runs the
    layer and copies the outputs and the final state back (kda_forward)."""
    names = ("q", "k", "v", "z", "beta", "gate")
    hin = {}
    for n in names:
        t = torch.empty(d[n].shape, dtype=d[n].dtype, pin_memory=True)
        t.copy_(d[n])
        hin[n] = t
    s0 = None
    if d["S0"] is not None:
        s0 = torch.empty(d["S0"].shape, dtype=torch.float32, pin_memory=True)
        s0.copy_(d["S0"])
    W = d["W_o"]
    for n in names:
        d[n] = None   # the device copies of the timing run are not needed any more
    torch.cuda.empty_cache()
    y_h = torch.empty((w.B, w.S, w.D_model), dtype=hin["q"].dtype, pin_memory=True)
    s_h = torch.empty((w.B, w.H, w.Dk, w.Dv), dtype=torch.float32, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in hin.values()) + (0 if s0 is None else s0.numel() * 4)
    d2h = y_h.numel() * y_h.element_size() + s_h.numel() * 4

    def one():
        K.kda_forward(hin["q"], hin["k"], hin["v"], hin["z"], hin["beta"], hin["gate"], W, s0, g_min=w.g_min,
                      eps=w.eps, state_dtype=torch.float32, outputs=y_h, final_state_out=s_h)

    one()
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(steps):
        one()
    torch.cuda.synchronize(dev)
    t = (time.perf_counter() - t0) / steps
    (t_max,) = reduce_max([t], world, dev)
    return {"value": round(w.B * w.S * world / t_max, 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps, "ms_per_step": round(t_max * 1e3, 2),
            "api": "kimi_delta_attention_21_b200.kda_forward (pinned host tensors in and out)"}


BACKWARD_ENTRY = {
    "recurrent_bwd": "kda_recurrent_bwd (exact fp32, recurrent form with 64-token checkpoints)",
    "chunk_bwd": "kda_chunk_bwd (exact fp32, chunk form: chunks in parallel, state and its gradient in order)",
}


def time_backward(K, torch, w, d, warmup, world, dev, flush, lib, steps=3, engine="recurrent_bwd"):
    """A backward entry point on the workload: gradients of the core recurrence
    w.r.t. q, k, v, beta, z and the initial state from a seeded dL/do~ and
    dL/dS_T, by the recurrent form (kda_recurrent_bwd) or the chunk form
    (kda_chunk_bwd)."""
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 99)
    d_o = torch.randn((w.B, w.S, w.H, w.Dv), generator=g, device=dev).to(d["q"].dtype)
    d_st = torch.randn((w.B, w.H, w.Dk, w.Dv), generator=g, device=dev)
    ws = None  # (the binding allocates the outputs and the workspace per call)

    def one():
        return getattr(K, engine)(d["q"], d["k"], d["v"], d["beta"], d_o, z=d["z"], g_min=w.g_min,
                                  initial_state=d["S0"], d_final_state=d_st, workspace=ws)

    for _ in range(max(1, warmup // 3)):
        one()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    n0 = lib.kda_launch_count()
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    (t,) = reduce_max([e0.elapsed_time(e1) / steps * 1e-3], world, dev)
    return {"entry_point": BACKWARD_ENTRY[engine], "ms": round(t * 1e3, 3), "tokens_per_s": round(w.B * w.S * world / t, 1),
            "gpu_launches_per_call": int((lib.kda_launch_count() - n0) // steps)}


def time_dplr(K, torch, w, d, warmup, world, dev, rec, steps=3):
    """The general DPLR transition (free erase directions; here random unit
    directions drawn on the device) on the workload, token by token and in
    chunk form, against the KDA chunk engine's time on the same workload: what
    KDA's binding (two decayed products per chunk instead of four, a state-only
    chain, tensor-core operands) is worth on this GPU."""
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 7)
    shp = (w.B, w.S, w.H, w.Dk)
    a = torch.nn.functional.normalize(torch.randn(shp, generator=g, device=dev), dim=-1).to(d["q"].dtype)
    b = torch.nn.functional.normalize(torch.randn(shp, generator=g, device=dev), dim=-1).to(d["q"].dtype)
    o = torch.empty((w.B, w.S, w.H, w.Dv), dtype=d["q"].dtype, device=dev)
    sf = torch.empty((w.B, w.H, w.Dk, w.Dv), dtype=torch.float32, device=dev)

    ws = torch.empty(K.api.dplr_chunk_workspace_bytes(w.B, w.S, w.H, w.Dk, w.Dv), dtype=torch.uint8, device=dev)

    def recurrent():
        K.dplr_recurrent_fwd(d["q"], d["k"], d["v"], a, b, z=d["z"], g_min=w.g_min, initial_state=d["S0"], out=o,
                             final_state=sf)

    def chunked():
        K.dplr_chunk_fwd(d["q"], d["k"], d["v"], a, b, z=d["z"], g_min=w.g_min, initial_state=d["S0"], out=o,
                         final_state=sf, workspace=ws)

    def timed(one):
        for _ in range(max(1, warmup // 3)):
            one()
        torch.cuda.synchronize(dev)
        stream = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        e0.record(stream)
        for _ in range(steps):
            one()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        (t,) = reduce_max([e0.elapsed_time(e1) / steps * 1e-3], world, dev)
        return t

    t, tc = timed(recurrent), timed(chunked)
    out = {"entry_point": "kda_dplr_recurrent_fwd (general DPLR, token by token, exact fp32)",
           "ms": round(t * 1e3, 3), "tokens_per_s": round(w.B * w.S * world / t, 1),
           "chunk": {"entry_point": "kda_dplr_chunk_fwd (general DPLR in chunk form, exact fp32 SIMT)",
                     "ms": round(tc * 1e3, 3), "tokens_per_s": round(w.B * w.S * world / tc, 1),
                     "recurrent_over_chunk_time": round(t / tc, 2)}}
    if rec and "kernels_ms" in rec:
        out["dplr_over_kda_chunk_engine_time"] = round(t * 1e3 / rec["kernels_ms"]["chunk_engine"], 2)
        out["chunk"]["dplr_chunk_over_kda_chunk_engine_time"] = round(tc * 1e3 / rec["kernels_ms"]["chunk_engine"], 2)
    return out


def run_decode(K, torch, w, d, warmup, world, dev, peaks, lib):
    dt = d["q"].dtype
    T = w.decode_steps
    steps = {n: d[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "z", "beta", "gate")}
    state = d["S0"].clone()
    x = torch.empty((w.B, w.H, w.Dv), dtype=dt, device=dev)
    y = torch.empty((w.B, w.D_model), dtype=dt, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one(t):
        K.decode_step(steps["q"][t], steps["k"][t], steps["v"][t], steps["beta"][t], state, z=steps["z"][t],
                      g_min=w.g_min, gate_logits=steps["gate"][t], eps=w.eps, out=x)

    for t in range(min(warmup, T)):
        one(t)
        K.out_proj(x.view(w.B, w.H * w.Dv), d["W_o"], out=y)
    state.copy_(d["S0"])
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(T)]
    barrier(world)
    n0 = lib.kda_launch_count()
    for t in range(T):
        ev[t][0].record(stream)
        one(t)
        ev[t][1].record(stream)
        K.out_proj(x.view(w.B, w.H * w.Dv), d["W_o"], out=y)
        ev[t][2].record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    launches = lib.kda_launch_count() - n0
    t_dec = sum(e[0].elapsed_time(e[1]) for e in ev) / T * 1e-3
    t_prj = sum(e[1].elapsed_time(e[2]) for e in ev) / T * 1e-3
    t_dec_m, t_prj_m = reduce_max([t_dec, t_prj], world, dev)
    nb = decode_bytes(w)
    ach = nb / t_dec_m / 1e9
    return {"workload": w.name, "value": round(w.B * world / (t_dec_m + t_prj_m), 1), "unit": "tokens/s",
            "steps": T, "ms_per_step": round((t_dec_m + t_prj_m) * 1e3, 4),
            "config": {"B": w.B, "H": w.H, "D_k": w.Dk, "D_v": w.Dv, "D_model": w.D_model,
                       "initial_state": f"N(0, {w.s0_std}) fp32, {w.B * w.H * w.Dk * w.Dv * 4 >> 20} MiB"},
            "kernels_ms": {"decode_step": round(t_dec_m * 1e3, 4), "out_proj": round(t_prj_m * 1e3, 4)},
            "roofline": {"kernel": "kda_decode_step", "bound": "hbm", "achieved": round(ach, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                         "traffic": traffic_for(f"decode@{DECODE}"), "algorithmic_bytes": nb},
            "gpu_launches": int(launches),
            "l2": "state (512 MiB) larger than L2"}


def run_ours(args, rank, world, local):
    import torch
    import kimi_delta_attention_21_b200 as K

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    lib = K.load_library()
    peaks, peak_src = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    only = set(ALL_WORKLOADS) if args.only == "all" else {args.only}
    records, baselines = {}, {}
    head_tm, e2e, sampler = None, None, ClockSampler(local)

    for name in (HEADLINE,) + PREFILL_EXTRA:
        if name not in only:
            continue
        w = rank_workload(name, rank)
        d = ki.device_inputs(w, dev)
        torch.cuda.synchronize(dev)
        tm = time_prefill(K, torch, w, d, args.steps, args.warmup, world, dev, flush, lib,
                          sampler if name == HEADLINE else None)
        records[name] = prefill_record(w, tm, peaks, world, f"chunk_engine@{name}")
        records[name]["gpu_launches"] = int(tm["launches"])
        # the scalar-decay (Gated DeltaNet) engine on the same inputs: what the per-channel decay costs
        tg = time_prefill(K, torch, w, d, max(3, args.steps // 2), args.warmup, world, dev, flush, lib, gdn=True)
        gr = roofline(chunk_flops(w), prefill_bytes(w, scalar_decay=True), tg["t_chunk"], peaks)
        records[name]["gdn"] = {
            "engine": "kda_gdn_chunk_fwd (scalar decay per token and head)",
            "chunk_engine_ms": round(tg["t_chunk"] * 1e3, 4),
            "layer_tokens_per_s": round(w.B * w.S * world / tg["t_step"], 1),
            "chunk_engine_tokens_per_s": round(w.B * w.S * world / tg["t_chunk"], 1),
            "roofline": {k: gr[k] for k in ("bound", "achieved", "peak", "unit", "frac")},
            "kda_over_gdn_chunk_time": round(tm["t_chunk"] / tg["t_chunk"], 3)}
        if name == "prefill_4k":
            # the exact SIMT engine, which the library uses outside the tensor-core engine's envelope
            ts = time_prefill(K, torch, w, d, max(3, args.steps // 4), args.warmup, world, dev, flush, lib,
                              engine="simt")
            records[name]["simt_engine"] = {
                "engine": "kda_chunk_fwd with engine = SIMT (exact; fp64 G and accumulation for fp32 inputs)",
                "used_when": "auto: inputs not bf16, D_k or D_v not 128, chunk not 64, g_min < -5.5, or a pointer "
                             "not 16-byte aligned",
                "chunk_engine_ms": round(ts["t_chunk"] * 1e3, 4),
                "chunk_engine_tokens_per_s": round(w.B * w.S * world / ts["t_chunk"], 1),
                "simt_over_tc_chunk_time": round(ts["t_chunk"] / tm["t_chunk"], 2)}
        if name == HEADLINE:
            head_tm = tm
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            baselines[name] = cpu_baseline_prefill(w, d, 12.0 if name == HEADLINE else 5.0)
        if name == HEADLINE and not args.no_e2e:
            e2e = run_e2e(K, torch, w, d, max(2, min(args.steps, 3)), world, dev)
        del d
        torch.cuda.empty_cache()

    if "prefill_4k" in only and not args.no_backward:
        w = rank_workload("prefill_4k", rank)
        d = ki.device_inputs(w, dev)
        rb = records.setdefault("prefill_4k", {})
        rb["backward"] = time_backward(K, torch, w, d, args.warmup, world, dev, flush, lib)
        rb["chunk_backward"] = time_backward(K, torch, w, d, args.warmup, world, dev, flush, lib, engine="chunk_bwd")
        rb["chunk_backward"]["recurrent_over_chunk_time"] = round(rb["backward"]["ms"] / rb["chunk_backward"]["ms"], 2)
        del d
        torch.cuda.empty_cache()

    if "prefill_4k" in only and not args.no_backward:
        w = rank_workload("prefill_4k", rank)
        d = ki.device_inputs(w, dev)
        records.setdefault("prefill_4k", {})["dplr_comparator"] = time_dplr(K, torch, w, d, args.warmup, world, dev,
                                                                            records.get("prefill_4k"))
        del d
        torch.cuda.empty_cache()

    if DECODE in only:
        w = rank_workload(DECODE, rank)
        d = ki.device_inputs(w, dev)
        records[DECODE] = run_decode(K, torch, w, d, args.warmup, world, dev, peaks, lib)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            baselines[DECODE] = cpu_baseline_decode(w, d, 5.0)
        del d
        torch.cuda.empty_cache()

    if rank != 0:
        return None
    for name, b in baselines.items():
        records[name]["cpu_baseline"] = b
    if head_tm is None:   # a partial run for profiling: print what ran
        return {"metric": METRIC, "partial": True, "n_gpus": world, "workloads": records}
    w = ki.WORKLOADS[HEADLINE]
    rec = records.pop(HEADLINE)
    line = {
        "metric": METRIC, "value": rec["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, generated on the device)",
        "config": dict(rec["config"], workload=HEADLINE, global_batch=w.B * world, seq_len=w.S,
                       parallelism=f"dp{world} (independent sequences)",
                       l2=f"inputs ({prefill_bytes(w) / 1e9:.1f} GB) larger than L2, and a {L2_FLUSH_BYTES >> 20} "
                          f"MiB write between steps (untimed)"),
        "roofline": dict(rec["roofline"], peak_source=f"{peak_src} (burst)"),
        "layer_roofline": rec["layer_roofline"],
        "kernels_ms": rec["kernels_ms"],
        "out_proj": rec["out_proj"],
        "chunk_engine_tokens_per_s": rec["chunk_engine_tokens_per_s"],
        "e2e": e2e,
        "gpu_launches": rec["gpu_launches"],
        "clocks": sampler.summary(),
        "wall_s_timed_region": round(head_tm["wall"], 4),
        "workloads": records,
    }
    if "gdn" in rec:
        line["gdn"] = rec["gdn"]
    if "cpu_baseline" in rec:
        line["cpu_baseline"] = rec["cpu_baseline"]
    return line


# ----------------------------------------------------------------------------- reference arm (the oracle)

def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    w = ki.WORKLOADS[HEADLINE]
    n = min(REF_SAMPLE_TOKENS, w.S)
    inp = ki.make_inputs_prefix(w, n)
    cores = oracle.default_threads()

    def one():
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["z"], inp["beta"], inp["gate"], inp["W_o"], inp["S0"],
                       g_min=w.g_min, eps=w.eps, threads=cores)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / args.steps
    value = round(w.B * n / dt, 1)
    sample = (f"the first {n} tokens x {w.H} heads of {HEADLINE} per step, from its initial state "
              f"(fp64 oracle, whole layer)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": HEADLINE, "B": w.B, "S": w.S, "H": w.H, "D_k": w.Dk,
                                            "D_v": w.Dv, "D_model": w.D_model, "sample_tokens": n},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing on prefill_4k")
    ap.add_argument("--only", choices=("all",) + ALL_WORKLOADS, default="all",
                    help="time one workload only (for profiling); the default runs all of them")
    ap.add_argument("--ranks-log", default=None, help="append one line per rank (rank world pid) to this file")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return launch_ranks(argv, args.gpus)
    rank, world, local = dist_env()
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
        return 2
    if args.ranks_log:
        with open(args.ranks_log, "a") as f:
            f.write(f"{rank} {world} {os.getpid()}\n")
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1 and args.impl == "ours":
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
