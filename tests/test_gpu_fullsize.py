"""Parity at the full workload sizes, in the launch configuration bench.py
times (default engine choice, device-generated inputs), on outputs the oracle
can compute one head at a time from the device's own input bytes, plus
properties that hold at any size."""
import numpy as np
import pytest

import kda_inputs as ki
import oracle
from kda_testlib import (BF16_OUT_ATOL, assert_bf16_outputs, assert_bf16_state, oracle_heads_dev, rel_fro,
                         to_np)

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def K():
    import kimi_delta_attention_21_b200 as K
    K.load_library()
    return K


def _check_projection_rows(x, y, W, rows):
    # y = concat_h(x) W_o^T, checked in fp64 on sampled rows of the device's own x
    idx = torch.as_tensor(np.asarray(rows), device=x.device)
    xs = to_np(x.reshape(x.shape[0] * x.shape[1], -1).index_select(0, idx))
    want = xs @ to_np(W).T
    assert_bf16_outputs(to_np(y.reshape(-1, y.shape[-1]).index_select(0, idx)), want, "projection rows")


def _check_heads(w, d, x, sf, pairs, t_rec, states_only=()):
    """x[b, t_rec, h] and sf[b, h] against the oracle for every (b, h) in pairs
    (final state only for the pairs in states_only)."""
    ref = oracle_heads_dev(w, d, list(pairs) + list(states_only), t_rec=t_rec)
    idx = torch.as_tensor(np.asarray(t_rec), device=x.device)
    for (b, h), (o_ref, s_ref, gate) in ref.items():
        assert_bf16_state(to_np(sf[b, h]), s_ref, f"final state (b={b}, h={h})")
        if (b, h) in pairs:
            x_ref = oracle.norm_gate(o_ref, gate, w.eps)
            assert_bf16_outputs(to_np(x[b, :, h].index_select(0, idx)), x_ref, f"x (b={b}, h={h})")


def _tokens(S, n, seed):
    rng = np.random.default_rng(seed)
    edge = [0, 1, 63, 64, 65, S // 2, S - 65, S - 64, S - 1]
    return np.unique(np.concatenate([[t for t in edge if 0 <= t < S], rng.integers(0, S, n)]))


def test_full_size_prefill_4k(K):
    w = ki.WORKLOADS["prefill_4k"]
    d = ki.device_inputs(w, "cuda")
    x, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, initial_state=d["S0"],
                        gate_logits=d["gate"], eps=w.eps)
    y = K.out_proj(x.view(w.B, w.S, w.H * w.Dv), d["W_o"])
    torch.cuda.synchronize()
    t_rec = _tokens(w.S, 120, 0)
    _check_heads(w, d, x, sf, [(0, h) for h in range(w.H)], t_rec)          # every head
    rows = np.unique(np.concatenate([[0, w.S - 1], np.random.default_rng(1).integers(0, w.S, 200)]))
    _check_projection_rows(x, y, d["W_o"], rows)


def test_full_size_batch_8x8k(K):
    w = ki.WORKLOADS["batch_8x8k"]
    d = ki.device_inputs(w, "cuda")
    x, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, initial_state=d["S0"],
                        gate_logits=d["gate"], eps=w.eps)
    y = K.out_proj(x.view(w.B, w.S, w.H * w.Dv), d["W_o"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    pairs = {(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)}
    while len(pairs) < 16:
        pairs.add((int(rng.integers(0, w.B)), int(rng.integers(0, w.H))))
    _check_heads(w, d, x, sf, sorted(pairs), _tokens(w.S, 64, 3))
    rows = np.unique(np.concatenate([[0, w.B * w.S - 1], rng.integers(0, w.B * w.S, 200)]))
    _check_projection_rows(x, y, d["W_o"], rows)
    assert np.isfinite(to_np(y.float().view(-1)[:: 9973])).all()


def test_full_size_long_context(K):
    w = ki.WORKLOADS["long_1m"]
    d = ki.device_inputs(w, "cuda")
    x, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, initial_state=d["S0"],
                        gate_logits=d["gate"], eps=w.eps)
    torch.cuda.synchronize()
    # every head's final state; o~ on 72+ tokens of four heads
    t_rec = _tokens(w.S, 64, 4)
    out_heads = [(0, 0), (0, 5), (0, 10), (0, 15)]
    _check_heads(w, d, x, sf, out_heads, t_rec, states_only=[(0, h) for h in range(w.H) if (0, h) not in out_heads])
    # property at full size: a split at an unaligned token with the state handed over
    cut = 700001
    sl = lambda t, a, b: t[:, a:b].contiguous()
    x1, s1 = K.chunk_fwd(*(sl(d[n], 0, cut) for n in ("q", "k", "v", "beta")), z=sl(d["z"], 0, cut),
                         g_min=w.g_min, initial_state=d["S0"], gate_logits=sl(d["gate"], 0, cut), eps=w.eps)
    x2, s2 = K.chunk_fwd(*(sl(d[n], cut, w.S) for n in ("q", "k", "v", "beta")), z=sl(d["z"], cut, w.S),
                         g_min=w.g_min, initial_state=s1, gate_logits=sl(d["gate"], cut, w.S), eps=w.eps)
    torch.cuda.synchronize()
    assert rel_fro(to_np(s2), to_np(sf)) <= 1e-2
    for t in (cut - 1, cut, cut + 1, w.S - 1):
        got = to_np(x1[:, t]) if t < cut else to_np(x2[:, t - cut])
        assert float(np.max(np.abs(got - to_np(x[:, t])))) <= BF16_OUT_ATOL


def test_full_size_decode(K):
    w = ki.WORKLOADS["decode_256"]
    d = ki.device_inputs(w, "cuda")
    steps = {n: d[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "z", "beta", "gate")}
    state = d["S0"].clone()
    xs = []
    for t in range(w.decode_steps):
        xs.append(K.decode_step(steps["q"][t], steps["k"][t], steps["v"][t], steps["beta"][t], state,
                                z=steps["z"][t], g_min=w.g_min, gate_logits=steps["gate"][t], eps=w.eps))
    y_last = K.out_proj(xs[-1].view(w.B, w.H * w.Dv), d["W_o"])
    torch.cuda.synchronize()
    x = torch.stack(xs, 1)  # (B, T, H, Dv)
    rng = np.random.default_rng(5)
    pairs = {(0, 0), (255, 31), (100, 7), (17, 20)}
    while len(pairs) < 16:
        pairs.add((int(rng.integers(0, w.B)), int(rng.integers(0, w.H))))
    _check_heads(w, d, x, state, sorted(pairs), np.arange(w.decode_steps))
    _check_projection_rows(x[:, -1:], y_last, d["W_o"], np.arange(0, 256, 17))
