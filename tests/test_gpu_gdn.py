"""The Gated DeltaNet (scalar-decay) chunk engine against the oracle's GDN
recurrence: the tensor-core engine (bf16, D_k = D_v = 128) on ragged, segmented
and gated shapes, with decays far below the KDA engine's g_min bound, and the
exact SIMT engine (fp32, other head sizes)."""
import numpy as np
import pytest

import kda_inputs as ki
import oracle
from kda_testlib import (assert_bf16_outputs, assert_bf16_state, assert_f32_close, rel_fro, small, to_dev,
                         to_np, upload)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    import kimi_delta_attention_21_b200 as K
    K.load_library()
    return K


def _timeouts(K):
    import ctypes
    n = ctypes.c_uint32(0)
    assert K.load_library().kda_device_timeouts(ctypes.byref(n), 1) == 0
    return n.value


def _case(name, B, S, H, D, dtype, seed, **kw):
    w = small(name, B, S, H, D, D, 256 if D == 128 else 32, dtype, seed=seed, **kw)
    inp = ki.make_inputs(w)
    inp["zh"] = np.ascontiguousarray(inp["z"][..., 0])            # one decay logit per token and head
    d = upload(inp, w)
    d["zh"] = to_dev(inp["zh"], d["z"].dtype)
    return w, inp, d


@pytest.mark.parametrize("B,S,H,g_min,s0", [(1, 1, 1, -5.0, 0.0), (1, 64, 2, -5.0, 0.02), (2, 130, 3, -20.0, 0.02),
                                            (1, 777, 2, -0.5, 0.02), (3, 257, 5, -60.0, 0.0),
                                            (1, 2560, 2, -5.0, 0.02)])
def test_gdn_tc_matches_oracle(K, B, S, H, g_min, s0):
    w, inp, d = _case("gdn", B, S, H, 128, "bf16", seed=S + H, s0_std=s0, g_min=g_min)
    o, sf = K.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["zh"], g_min=g_min, initial_state=d["S0"],
                            engine="tc")
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    o_ref, s_ref = oracle.gdn_recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["zh"], g_min=g_min,
                                         initial_state=inp["S0"])
    assert_bf16_outputs(to_np(o), o_ref, "o~")
    assert_bf16_state(to_np(sf), s_ref, "final_state")


def test_gdn_tc_log_decay_and_gate(K):
    w, inp, d = _case("gdng", 2, 500, 4, 128, "bf16", seed=5, s0_std=0.02)
    ld = (-5.0 / (1.0 + np.exp(-inp["zh"].astype(np.float64)))).astype(np.float32)
    x, sf = K.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], log_decay=torch.from_numpy(ld).cuda(), g_min=-5.0,
                            initial_state=d["S0"], gate_logits=d["gate"], eps=w.eps, engine="tc")
    y = K.out_proj(x.reshape(w.B * w.S, w.H * w.Dv), d["W_o"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.gdn_recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], log_decay=ld, g_min=-5.0,
                                         initial_state=inp["S0"])
    want = oracle.project(oracle.norm_gate(o_ref, inp["gate"], w.eps), inp["W_o"])
    assert_bf16_outputs(to_np(y).reshape(want.shape), want, "layer outputs")
    assert_bf16_state(to_np(sf), s_ref, "final_state")


@pytest.mark.parametrize("dtype,D", [("f32", 16), ("f32", 128), ("bf16", 48)])
def test_gdn_simt_matches_oracle(K, dtype, D):
    w, inp, d = _case("gdns", 2, 150, 3, D, dtype, seed=D, s0_std=0.02)
    o, sf = K.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["zh"], g_min=-5.0, initial_state=d["S0"],
                            engine="simt")
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.gdn_recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["zh"], g_min=-5.0,
                                         initial_state=inp["S0"])
    if dtype == "f32":
        assert_f32_close(to_np(o), o_ref, "o~")
        assert_f32_close(to_np(sf), s_ref, "final_state")
    else:
        assert_bf16_outputs(to_np(o), o_ref, "o~")
        assert_bf16_state(to_np(sf), s_ref, "final_state")


def test_gdn_tc_agrees_with_kda_engine_on_a_channel_constant_decay(K):
    """With the decay logits constant across channels, the KDA tensor-core engine computes the same
    recurrence; the two engines agree within the bf16 tolerances."""
    w, inp, d = _case("gdnk", 1, 900, 3, 128, "bf16", seed=8, s0_std=0.02)
    zc = d["zh"][..., None].expand(w.B, w.S, w.H, w.Dk).contiguous()
    o1, s1 = K.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["zh"], initial_state=d["S0"], engine="tc")
    o2, s2 = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=zc, initial_state=d["S0"], engine="tc")
    assert_bf16_outputs(to_np(o1), to_np(o2), "GDN vs KDA engines")
    assert rel_fro(to_np(s1), to_np(s2)) <= 1e-2


def test_gdn_rejects_a_per_channel_decay_shape(K):
    w, inp, d = _case("gdnr", 1, 70, 2, 128, "bf16", seed=9)
    with pytest.raises(ValueError):
        K.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"])   # (B,S,H,D_k) is the KDA shape
