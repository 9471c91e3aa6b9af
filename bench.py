#!/usr/bin/env python
"""Throughput of the KDA layer forward on B200: chunkwise prefill (headline)
and the single-token decode step, with roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one process per GPU)

One step = one whole layer forward (gate, chunk engine with the fused
RMSNorm and sigmoid gate, output projection) over one batch of the
``prefill_4k`` workload (B1 S4096 H16 D128, D_model 2048, bf16, fp32 state),
inputs resident in HBM, L2 flushed between steps.  Each rank runs its own
independent sequence (weak scaling, no collective on the data path).  The
decode engine is timed in the same run on the ``decode_256`` workload and
reported under "decode".  Rank 0 prints one JSON line.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
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
PREFILL = "prefill_4k"
DECODE = "decode_256"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
REF_SAMPLE_TOKENS = 512   # tokens (all heads) per reference-arm step

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# the committed ncu summaries under profiles/, keyed by kernel and workload,
# valid only while the kernel's source file is unchanged (sha256 prefix).
NCU_TRAFFIC = {
    # prefill_4k_chunk_engine.md: prep 129.4 + segment maps 43.9 + combine 7.4 + segment chains 104.6 MB
    "chunk_engine@prefill_4k": {"bytes": 285193728, "src_sha": "062ca38e894c9ecc"},
    # decode_256_step.md: decode128_stream_kernel, 547.4 MB read + 479.8 MB written
    "decode@decode_256": {"bytes": 1027173120, "src_sha": "079db3bd726bd665"},
}


# ----------------------------------------------------------------------------- helpers

def src_sha(relpath):
    with open(os.path.join(ROOT, relpath), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(kernel, workload, src):
    rec = NCU_TRAFFIC.get(f"{kernel}@{workload}")
    if rec and rec["src_sha"] == src_sha(src):
        return rec["bytes"]
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def prefill_bytes(w):
    """Algorithmic HBM bytes of the chunk engine for a whole workload: read q, k,
    z (D_k each), v, gate (D_v each) and beta per token-head, write the gated
    output (D_v) per token-head, write the fp32 final state per (b, h)."""
    es = 2 if w.dtype == "bf16" else 4
    per_tok_head = es * (3 * w.Dk + 3 * w.Dv + 1)
    return w.B * w.S * w.H * per_tok_head + w.B * w.H * w.Dk * w.Dv * 4


def chunk_flops(w, C=64):
    """Algorithmic tensor FLOPs of the chunkwise prefill (2 per multiply-add), per chunk of C tokens:
    the causal intra-chunk products A = (beta K) K^T and M = Q K^T, the UT-transform products
    W = T (beta K e^G) and U = T (beta V) and the intra-chunk output M V' (lower triangles: C^2 D
    each), and the three state products W S, (Q e^G) S and K~^T V' (2 C D_k D_v each).  The
    triangular solve itself is not counted."""
    per_chunk = C * C * (2 * w.Dk + w.Dk + 2 * w.Dv) + 3 * 2 * C * w.Dk * w.Dv
    return w.B * w.H * ((w.S + C - 1) // C) * per_chunk


def proj_flops(n_rows, w):
    return 2.0 * n_rows * w.H * w.Dv * w.D_model


def decode_bytes(w):
    """Algorithmic HBM bytes of one decode step: the fp32 state read and written
    once, q, k, z, v, gate and beta read, the gated output written."""
    es = 2 if w.dtype == "bf16" else 4
    per_bh = 2 * w.Dk * w.Dv * 4 + es * (3 * w.Dk + 3 * w.Dv + 1)
    return w.B * w.H * per_bh


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


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local):
    import torch
    import kimi_delta_attention_21_b200 as K

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    lib = K.load_library()
    peaks, peak_src = load_peaks()
    if args.only == "decode":
        dec = run_decode(args, rank, world, local, K, dev, peaks)
        return {"metric": METRIC, "decode": dec, "n_gpus": world} if rank == 0 else None

    # ---------------- prefill inputs, resident in HBM
    w = rank_workload(PREFILL, rank)
    inp = ki.make_inputs(w)
    dt = torch.bfloat16
    dv = {n: torch.from_numpy(inp[n]).to(dev).to(dt).contiguous() for n in ("q", "k", "v", "z", "beta", "gate", "W_o")}
    B, S, H = w.B, w.S, w.H
    N = B * S
    x = torch.empty((B, S, H, w.Dv), dtype=dt, device=dev)
    y = torch.empty((N, w.D_model), dtype=dt, device=dev)
    sf = torch.empty((B, H, w.Dk, w.Dv), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        K.chunk_fwd(dv["q"], dv["k"], dv["v"], dv["beta"], z=dv["z"], g_min=w.g_min, gate_logits=dv["gate"],
                    eps=w.eps, out=x, final_state=sf)
        K.out_proj(x.view(N, H * w.Dv), dv["W_o"], out=y)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize(dev)

    n_ev = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_ev)]
    sampler = ClockSampler(local)
    launches0 = lib.kda_launch_count()
    with sampler:
        barrier(world)
        torch.cuda.synchronize(dev)
        t_wall0 = time.perf_counter()
        for i in range(n_ev):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            K.chunk_fwd(dv["q"], dv["k"], dv["v"], dv["beta"], z=dv["z"], g_min=w.g_min,
                        gate_logits=dv["gate"], eps=w.eps, out=x, final_state=sf)
            ev[i][1].record(stream)
            K.out_proj(x.view(N, H * w.Dv), dv["W_o"], out=y)
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        t_wall = time.perf_counter() - t_wall0
    launches = lib.kda_launch_count() - launches0
    t_chunk = sum(e[0].elapsed_time(e[1]) for e in ev) / n_ev * 1e-3
    t_proj = sum(e[1].elapsed_time(e[2]) for e in ev) / n_ev * 1e-3
    t_step = t_chunk + t_proj
    t_step_max, t_chunk_max, t_proj_max = reduce_max([t_step, t_chunk, t_proj], world, dev)

    if args.only == "prefill":
        return {"metric": METRIC, "value": round(N * world / t_step_max, 1), "unit": "tokens/s",
                "kernels_ms": {"chunk_engine": round(t_chunk * 1e3, 4), "out_proj": round(t_proj * 1e3, 4)},
                "gpu_launches": int(launches)} if rank == 0 else None

    # ---------------- end to end through the public API, host buffers
    hin = {n: torch.from_numpy(inp[n]).to(dt).pin_memory() for n in ("q", "k", "v", "z", "beta", "gate")}
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    for _ in range(2):
        out = K.kda_forward(hin["q"], hin["k"], hin["v"], hin["z"], hin["beta"], hin["gate"], dv["W_o"],
                            None, g_min=w.g_min, eps=w.eps, state_dtype=torch.float32)
    d2h = out["outputs"].numel() * out["outputs"].element_size() + \
        out["final_state"].numel() * out["final_state"].element_size()
    e2e_steps = max(3, min(args.steps, 20))
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        out = K.kda_forward(hin["q"], hin["k"], hin["v"], hin["z"], hin["beta"], hin["gate"], dv["W_o"],
                            None, g_min=w.g_min, eps=w.eps, state_dtype=torch.float32)
    torch.cuda.synchronize(dev)
    t_e2e = (time.perf_counter() - t0) / e2e_steps
    (t_e2e_max,) = reduce_max([t_e2e], world, dev)

    # ---------------- decode engine (decode_256), state larger than L2
    dec = run_decode(args, rank, world, local, K, dev, peaks)

    if rank != 0:
        return None
    tokens_all = N * world
    value = tokens_all / t_step_max
    chunk_bytes = prefill_bytes(w)
    cflops = chunk_flops(w)
    pflops = proj_flops(N, w)
    chunk_ach = chunk_bytes / t_chunk / 1e9
    chunk_tach = cflops / t_chunk / 1e12
    proj_ach = pflops / t_proj / 1e12
    chunk_frac = chunk_ach / peaks["hbm_gbs"]
    chunk_tfrac = chunk_tach / peaks["bf16_tflops"]
    proj_frac = proj_ach / peaks["bf16_tflops"]
    if t_chunk >= t_proj:
        # the chunk products are the path's dense contractions: tensor-pipe roofline, with the HBM view
        # (algorithmic bytes, DRAM traffic from the ncu capture) beside it
        roof = {"kernel": "kda_chunk_fwd (chunk engine)", "bound": "tensor", "achieved": round(chunk_tach, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(chunk_tfrac, 4),
                "traffic": traffic_for("chunk_engine", PREFILL, "kimi_delta_attention_21_b200/csrc/chunk_tc.cu"),
                "algorithmic_flops": cflops, "algorithmic_bytes": chunk_bytes,
                "hbm_achieved_gbs": round(chunk_ach, 1), "hbm_frac": round(chunk_frac, 4),
                "ms": round(t_chunk * 1e3, 4)}
    else:
        roof = {"kernel": "kda_out_proj", "bound": "tensor", "achieved": round(proj_ach, 1),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(proj_frac, 4),
                "traffic": traffic_for("proj", PREFILL, "kimi_delta_attention_21_b200/csrc/proj_tc.cu"),
                "algorithmic_flops": pflops, "ms": round(t_proj * 1e3, 4)}
    roof["peak_source"] = f"{peak_src} (burst)"
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_step_max * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": PREFILL, "B": w.B, "S": w.S, "H": w.H, "D_k": w.Dk, "D_v": w.Dv,
                   "D_model": w.D_model, "chunk": 64, "g_min": w.g_min, "state": "fp32",
                   "global_batch": w.B * world, "seq_len": w.S, "parallelism": f"dp{world} (independent sequences)",
                   "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, untimed)"},
        "roofline": roof,
        "kernels_ms": {"chunk_engine": round(t_chunk * 1e3, 4), "out_proj": round(t_proj * 1e3, 4),
                       "chunk_engine_tensor_frac": round(chunk_tfrac, 4), "chunk_engine_hbm_frac": round(chunk_frac, 4),
                       "out_proj_tensor_frac": round(proj_frac, 4)},
        "e2e": {"value": round(tokens_all / t_e2e_max, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "api": "kimi_delta_attention_21_b200.kda_forward (pinned host tensors)"},
        "gpu_launches": int(launches),
        "clocks": sampler.summary(),
        "wall_s_timed_region": round(t_wall, 4),
        "decode": dec,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, inp)
    return line


def run_decode(args, rank, world, local, K, dev, peaks):
    import torch
    w = rank_workload(DECODE, rank)
    inp = ki.make_inputs(w)
    dt = torch.bfloat16
    T = w.decode_steps
    dv = {n: torch.from_numpy(inp[n]).to(dev).to(dt) for n in ("q", "k", "v", "z", "beta", "gate", "W_o")}
    # per-step contiguous inputs (B, H, D) laid out step-major
    steps = {n: dv[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "z", "beta", "gate")}
    state0 = torch.from_numpy(inp["S0"]).to(dev)
    state = state0.clone()
    x = torch.empty((w.B, w.H, w.Dv), dtype=dt, device=dev)
    y = torch.empty((w.B, w.D_model), dtype=dt, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one(t):
        K.decode_step(steps["q"][t], steps["k"][t], steps["v"][t], steps["beta"][t], state, z=steps["z"][t],
                      g_min=w.g_min, gate_logits=steps["gate"][t], eps=w.eps, out=x)

    for t in range(min(args.warmup, T)):
        one(t)
        K.out_proj(x.view(w.B, w.H * w.Dv), dv["W_o"], out=y)
    state.copy_(state0)
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(T)]
    barrier(world)
    for t in range(T):
        ev[t][0].record(stream)
        one(t)
        ev[t][1].record(stream)
        K.out_proj(x.view(w.B, w.H * w.Dv), dv["W_o"], out=y)
        ev[t][2].record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    t_dec = sum(e[0].elapsed_time(e[1]) for e in ev) / T * 1e-3
    t_prj = sum(e[1].elapsed_time(e[2]) for e in ev) / T * 1e-3
    t_dec_m, t_prj_m = reduce_max([t_dec, t_prj], world, dev)
    nb = decode_bytes(w)
    ach = nb / t_dec / 1e9
    return {"workload": DECODE, "value": round(w.B * world / (t_dec_m + t_prj_m), 1), "unit": "tokens/s",
            "steps": T, "ms_per_step": round((t_dec_m + t_prj_m) * 1e3, 4),
            "kernels_ms": {"decode_step": round(t_dec * 1e3, 4), "out_proj": round(t_prj * 1e3, 4)},
            "roofline": {"kernel": "kda_decode_step", "bound": "hbm", "achieved": round(ach, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                         "traffic": traffic_for("decode", DECODE, "kimi_delta_attention_21_b200/csrc/decode.cu"),
                         "algorithmic_bytes": nb},
            "l2": "state (512 MiB) larger than L2"}


def cpu_baseline(w, inp, max_seconds=20.0):
    """The oracle as it stands on this host's cores, on a bounded sample: the
    first n tokens (all heads) of the same workload, whole layer forward."""
    import oracle
    cores = oracle.default_threads()
    n = min(w.S, 512)
    while True:
        t0 = time.perf_counter()
        oracle.forward(inp["q"][:, :n], inp["k"][:, :n], inp["v"][:, :n], inp["z"][:, :n], inp["beta"][:, :n],
                       inp["gate"][:, :n], inp["W_o"], None, g_min=w.g_min, eps=w.eps, threads=cores)
        dt = time.perf_counter() - t0
        if n >= w.S or dt * (w.S / n) > max_seconds:
            break
        n = w.S
    return {"value": round(w.B * n / dt, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} of {w.S} tokens x {w.H} heads of {w.name}, fp64 recurrence + norm/gate + "
                      f"projection, {dt:.2f} s"}


# ----------------------------------------------------------------------------- reference arm (the oracle)

def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    w = ki.WORKLOADS[PREFILL]
    n = min(REF_SAMPLE_TOKENS, w.S)
    inp = ki.make_inputs(ki.custom("ref_sample", w.B, n, w.H, w.Dk, w.Dv, w.D_model, w.dtype, seed=w.seed))
    cores = oracle.default_threads()

    def one():
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["z"], inp["beta"], inp["gate"], inp["W_o"], None,
                       g_min=w.g_min, eps=w.eps, threads=cores)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / args.steps
    value = round(w.B * n / dt, 1)
    sample = f"{n} tokens x {w.H} heads of {PREFILL} per step (fp64 oracle, whole layer)"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": PREFILL, "B": w.B, "S": w.S, "H": w.H, "D_k": w.Dk,
                                            "D_v": w.Dv, "D_model": w.D_model, "sample_tokens": n},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                    help="run one engine only (for profiling); the default runs both plus e2e")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
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
