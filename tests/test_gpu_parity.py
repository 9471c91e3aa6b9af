"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded
inputs.  fp32: atol 1e-6 / rtol 1e-5 ("KDA Recurrence" page, Requirements).
bf16: max-abs output error <= 2e-2, final-state relative Frobenius <= 1e-2."""
import json
import os

import numpy as np
import pytest

import kda_inputs as ki
import oracle
from kda_testlib import (rel_fro, assert_bf16_outputs, assert_bf16_state, assert_f32_close, oracle_layer, small,
                         to_dev, to_np, upload)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "kda_recurrence_examples.json")))


@pytest.fixture(scope="module")
def K():
    import kimi_delta_attention_21_b200 as K
    K.load_library()
    return K


ENGINES = ["simt", "tc"]


# ------------------------------------------------------------------ the page's examples

def test_worked_example(K):
    i = GOLD["worked_example"]["inputs"]
    t = {n: torch.tensor(i[n], dtype=torch.float32, device="cuda") for n in
         ("query", "key", "value", "decay_logits", "write_strength", "output_gate_logits",
          "output_projection", "initial_state")}
    out = K.kda_forward(**t, g_min=i["g_min"], eps=i["eps"])
    assert set(out) == {"outputs", "final_state"}
    assert out["outputs"].dtype == torch.float32 and out["outputs"].is_cuda
    y = to_np(out["outputs"])
    s = to_np(out["final_state"])
    assert_f32_close(y, np.array(GOLD["worked_example"]["outputs"]), "outputs")
    assert_f32_close(s, np.array(GOLD["worked_example"]["final_state"]), "final_state")


def test_worked_example_from_host_tensors(K):
    i = GOLD["worked_example"]["inputs"]
    t = {n: torch.tensor(i[n], dtype=torch.float32) for n in
         ("query", "key", "value", "decay_logits", "write_strength", "output_gate_logits",
          "output_projection", "initial_state")}
    before = {n: v.clone() for n, v in t.items()}
    out = K.kda_forward(**t, g_min=i["g_min"], eps=i["eps"])
    assert not out["outputs"].is_cuda          # device preserved
    assert_f32_close(out["outputs"].numpy(), np.array(GOLD["worked_example"]["outputs"]))
    for n in t:                                 # inputs not mutated
        assert torch.equal(t[n], before[n])


@pytest.mark.parametrize("case", GOLD["shape_examples"], ids=lambda c: c["cite"])
def test_shape_examples(K, case):
    B, S, H, Dk = case["query_key_decay_shape"]
    Dv = case["value_shape"][-1]
    rng = np.random.default_rng(5)
    q = rng.standard_normal((B, S, H, Dk)).astype(np.float32)
    k = rng.standard_normal((B, S, H, Dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, S, H, Dv)).astype(np.float32)
    z = rng.standard_normal((B, S, H, Dk)).astype(np.float32)
    beta = rng.random((B, S, H, 1)).astype(np.float32)
    gl = rng.standard_normal((B, S, H, Dv)).astype(np.float32)
    W = rng.standard_normal(case["output_projection_shape"]).astype(np.float32)
    S0 = (0.3 * rng.standard_normal(case["initial_state_shape"])).astype(np.float32)
    f32 = torch.float32
    out = K.kda_forward(to_dev(q, f32), to_dev(k, f32), to_dev(v, f32), to_dev(z, f32), to_dev(beta, f32),
                        to_dev(gl, f32), to_dev(W, f32), to_dev(S0, f32))
    assert list(out["outputs"].shape) == case["outputs_shape"]
    assert list(out["final_state"].shape) == case["final_state_shape"]
    want = oracle.forward(q, k, v, z, beta, gl, W, S0)
    assert_f32_close(to_np(out["outputs"]), want["outputs"], "outputs")
    assert_f32_close(to_np(out["final_state"]), want["final_state"], "final_state")


# ------------------------------------------------------------------ small fp32 (exact path)

def test_tiny_fp32_workload(K):
    w = ki.WORKLOADS["tiny_fp32"]
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    out = K.kda_forward(d["q"], d["k"], d["v"], d["z"], d["beta"], d["gate"], d["W_o"], d["S0"],
                        g_min=w.g_min, eps=w.eps)
    want = oracle_layer(inp, w)
    assert_f32_close(to_np(out["outputs"]), want["outputs"], "outputs")
    assert_f32_close(to_np(out["final_state"]), want["final_state"], "final_state")


@pytest.mark.parametrize("B,S,H,Dk,Dv,chunk", [
    (1, 1, 1, 16, 16, 64), (2, 63, 2, 16, 8, 64), (1, 65, 3, 8, 16, 64), (2, 130, 2, 33, 20, 64),
    (1, 100, 1, 128, 128, 64), (1, 77, 2, 64, 48, 16), (3, 40, 1, 1, 1, 8), (1, 200, 2, 16, 16, 1),
])
def test_fp32_core_ragged(K, B, S, H, Dk, Dv, chunk):
    w = small("r", B, S, H, Dk, Dv, 8, "f32", seed=S * 7 + Dk, s0_std=0.3)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, initial_state=d["S0"],
                        chunk=chunk, engine="simt")
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min,
                                     initial_state=inp["S0"])
    assert_f32_close(to_np(o), o_ref, "o~")
    assert_f32_close(to_np(sf), s_ref, "final_state")


def test_fp32_norm_gate_fused_into_prefill(K):
    w = small("ng", 2, 70, 3, 16, 24, 8, "f32", seed=3)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    x, _ = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, gate_logits=d["gate"],
                       eps=w.eps, engine="simt")
    o_ref, _ = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min)
    assert_f32_close(to_np(x), oracle.norm_gate(o_ref, inp["gate"], w.eps))


# ------------------------------------------------------------------ special cases on the device

def test_beta_zero_and_unit_decay(K):
    w = small("s", 1, 50, 2, 16, 16, 8, "f32", seed=4, s0_std=0.5)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    ld = torch.zeros_like(d["z"], dtype=torch.float32)
    zero_beta = torch.zeros_like(d["beta"])
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], zero_beta, log_decay=ld, g_min=-5.0, initial_state=d["S0"])
    # alpha = 1, beta = 0: nothing changes; o_t = S_0^T q_t
    assert_f32_close(to_np(sf), inp["S0"].astype(np.float64))
    assert_f32_close(to_np(o), np.einsum("bshc,bhcj->bshj", inp["q"].astype(np.float64),
                                         inp["S0"].astype(np.float64)))
    # alpha = 1 with writes: DeltaNet
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], log_decay=ld, g_min=-5.0, initial_state=d["S0"])
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], log_decay=np.zeros_like(inp["z"]),
                                     initial_state=inp["S0"])
    assert_f32_close(to_np(o), o_ref)
    assert_f32_close(to_np(sf), s_ref)


def test_empty_sequence_and_batch(K):
    w = small("e", 2, 0, 2, 16, 16, 8, "f32", seed=1, s0_std=0.5)
    S0 = torch.randn(2, 2, 16, 16, device="cuda")
    z = torch.empty(2, 0, 2, 16, device="cuda")
    o, sf = K.chunk_fwd(z, z, z, torch.empty(2, 0, 2, device="cuda"), z=z, initial_state=S0)
    assert o.shape == (2, 0, 2, 16)
    assert torch.equal(sf, S0)
    z0 = torch.empty(0, 5, 2, 16, device="cuda")
    o, sf = K.chunk_fwd(z0, z0, z0, torch.empty(0, 5, 2, device="cuda"), z=z0)
    assert o.shape == (0, 5, 2, 16) and sf.shape == (0, 2, 16, 16)


def test_in_place_state_handoff(K):
    w = small("h", 2, 150, 2, 32, 32, 8, "f32", seed=8, s0_std=0.2)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    o_all, s_all = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"])
    st = d["S0"].clone()
    outs = []
    for a, b in ((0, 37), (37, 64), (64, 150)):
        sl = lambda t: t[:, a:b].contiguous()
        o, _ = K.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["beta"]), z=sl(d["z"]), initial_state=st,
                           final_state=st)
        outs.append(o)
    assert_f32_close(to_np(torch.cat(outs, 1)), to_np(o_all))
    assert_f32_close(to_np(st), to_np(s_all))


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("dtype,Dk,Dv", [("f32", 128, 128), ("f32", 16, 24), ("bf16", 128, 128), ("bf16", 7, 5)])
def test_decode_steps_match_oracle(K, dtype, Dk, Dv):
    T = 12
    w = small("d", 5, T, 3, Dk, Dv, 16, dtype, seed=Dk + Dv, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    state = d["S0"].clone()
    xs = []
    for t in range(T):
        xs.append(K.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                                d["beta"][:, t].contiguous(), state, z=d["z"][:, t].contiguous(), g_min=w.g_min,
                                gate_logits=d["gate"][:, t].contiguous(), eps=w.eps))
    x = to_np(torch.stack(xs, 1))
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min,
                                     initial_state=inp["S0"])
    x_ref = oracle.norm_gate(o_ref, inp["gate"], w.eps)
    if dtype == "f32":
        assert_f32_close(x, x_ref, "x")
        assert_f32_close(to_np(state), s_ref, "state")
    else:
        assert_bf16_outputs(x, x_ref, "x")
        assert_bf16_state(to_np(state), s_ref, "state")


def test_decode_then_prefill_agree(K):
    # 40 decode steps == one 40-token prefill on the same inputs
    w = small("dp", 2, 40, 2, 128, 128, 16, "bf16", seed=21, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    st = d["S0"].clone()
    xs = [K.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                        d["beta"][:, t].contiguous(), st, z=d["z"][:, t].contiguous()) for t in range(40)]
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"])
    assert_bf16_outputs(to_np(torch.stack(xs, 1)), to_np(o))
    assert_bf16_state(to_np(st), to_np(sf))


# ------------------------------------------------------------------ projection and gate kernels

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,H,Dv,Dm", [(1, 1, 1, 1), (37, 2, 16, 40), (300, 4, 32, 96), (256, 16, 128, 512)])
def test_norm_gate_projection(K, dtype, N, H, Dv, Dm):
    rng = np.random.default_rng(N + Dm)
    o = rng.standard_normal((N, H, Dv)).astype(np.float32)
    gl = rng.standard_normal((N, H, Dv)).astype(np.float32)
    W = (rng.standard_normal((Dm, H * Dv)) / np.sqrt(H * Dv)).astype(np.float32)
    if dtype == "bf16":
        o, gl, W = ki.round_bf16(o), ki.round_bf16(gl), ki.round_bf16(W)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    y = K.out_norm_gate_proj(to_dev(o, tdt), to_dev(gl, tdt), to_dev(W, tdt), eps=1e-6)
    want = oracle.project(oracle.norm_gate(o, gl, 1e-6), W)
    if dtype == "f32":
        assert_f32_close(to_np(y), want)
    else:
        assert_bf16_outputs(to_np(y), want)


def test_gate_kernel(K):
    rng = np.random.default_rng(2)
    z = ki.round_bf16(2 * rng.standard_normal(1000 + 3).astype(np.float32))
    for dt in (torch.float32, torch.bfloat16):
        g = K.gate(to_dev(z, dt), -5.0)
        np.testing.assert_allclose(to_np(g), oracle.log_decay(z, -5.0), rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------ bf16 layer at a real size

@pytest.mark.parametrize("engine", ENGINES)
def test_prefill_4k_layer(K, engine):
    w = ki.WORKLOADS["prefill_4k"]
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    out = K.kda_forward(d["q"], d["k"], d["v"], d["z"], d["beta"], d["gate"], d["W_o"], d["S0"],
                        g_min=w.g_min, eps=w.eps, state_dtype=torch.float32, engine=engine)
    want = oracle_layer(inp, w)
    assert_bf16_outputs(to_np(out["outputs"]), want["outputs"], "outputs")
    assert_bf16_state(to_np(out["final_state"]), want["final_state"], "final_state")


@pytest.mark.parametrize("N,K,Dm", [(1, 8, 8), (128, 64, 256), (129, 64, 264), (300, 200, 96), (4096, 2048, 2048),
                                    (256, 4096, 4096), (77, 4096, 520), (100, 1024, 2048)])
def test_projection_tensor_core_shapes(K, N, Dm):
    rng = np.random.default_rng(N * 3 + K)
    x = ki.round_bf16(rng.standard_normal((N, K)).astype(np.float32))
    W = ki.round_bf16((rng.standard_normal((Dm, K)) / np.sqrt(K)).astype(np.float32))
    import kimi_delta_attention_21_b200 as KK
    y = KK.out_proj(to_dev(x, torch.bfloat16), to_dev(W, torch.bfloat16))
    want = oracle.project(x[:, None, :], W)  # one "head" of width K
    # bf16 output rounding dominates: |y| <~ 5, half an ulp of bf16 at 4..8 is 1.6e-2
    err = np.abs(to_np(y) - want)
    assert float(err.max()) <= 2e-2
    assert float(np.median(err)) <= 2e-3


def test_unaligned_views_take_exact_paths(K):
    # token slices of (B, S, H, .) tensors start at element offsets that are not
    # 16-byte aligned: decode and the gate must still run and agree
    w = small("u", 1, 5, 1, 128, 128, 16, "bf16", seed=33, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    st = d["S0"].clone()
    xs = [K.decode_step(d["q"][:, t], d["k"][:, t], d["v"][:, t], d["beta"][:, t], st, z=d["z"][:, t],
                        gate_logits=d["gate"][:, t]) for t in range(5)]
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], initial_state=inp["S0"])
    assert_bf16_outputs(to_np(torch.stack(xs, 1)), oracle.norm_gate(o_ref, inp["gate"], 1e-6))
    assert_bf16_state(to_np(st), s_ref)
    zz = d["z"].flatten()[3:1000]
    np.testing.assert_allclose(to_np(K.gate(zz, -5.0)), oracle.log_decay(to_np(zz), -5.0), rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------ head-sharded layer

@pytest.mark.parametrize("world", [2, 3])
def test_head_sharded_layer_on_one_gpu(K, world):
    """Each rank's share of the head-sharded layer (its heads through the chunk engine and its W_o
    column block through the projection), run one after another on this GPU; the fp32 sum of the
    partial outputs is the layer output and each rank keeps its heads' final states.  The ranks never
    wait on one another, so one GPU can run them in turn.  The sum is checked against the oracle at
    the output tolerance, and against the whole layer through the same engine at the bf16 rounding of
    one partial per rank (the only arithmetic the split changes).  16 heads, as in the prefill
    workloads."""
    from kimi_delta_attention_21_b200.tensor_parallel import head_range, kda_forward_tp, shard, wo_columns
    w = small("tpg", 1, 512, 16, 128, 128, 2048, "bf16", seed=77, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    want = oracle_layer(inp, w)
    whole = K.kda_forward(d["q"], d["k"], d["v"], d["z"], d["beta"], d["gate"], d["W_o"], d["S0"], g_min=w.g_min,
                          eps=w.eps, state_dtype=torch.float32)
    total = 0
    for rank in range(world):
        h0, h1 = head_range(w.H, world, rank)
        c0, c1 = wo_columns(h0, h1, w.Dv)
        sl = lambda t: shard(t, h0, h1)
        y_r, s_r = kda_forward_tp(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["z"]), sl(d["beta"]), sl(d["gate"]),
                                  d["W_o"][:, c0:c1].contiguous(), shard(d["S0"], h0, h1, head_axis=1),
                                  g_min=w.g_min, eps=w.eps, H=w.H, rank=rank, world=world, out_dtype=torch.float32)
        torch.cuda.synchronize()
        total = total + to_np(y_r)
        assert_bf16_state(to_np(s_r), want["final_state"][:, h0:h1], f"rank {rank} final states")
        assert rel_fro(to_np(s_r), to_np(whole["final_state"][:, h0:h1])) <= 1e-3   # same engine, same heads
    assert_bf16_outputs(total, want["outputs"], f"summed partial outputs ({world} ranks)")
    ref = to_np(whole["outputs"])
    bound = world * 2.0 ** -8 * max(1.0, float(np.max(np.abs(ref))))
    assert float(np.max(np.abs(total - ref))) <= bound, "split changes more than the partials' rounding"
