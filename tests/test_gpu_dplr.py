"""The general DPLR comparator, token by token (kda_dplr_recurrent_fwd) and in
chunk form (kda_dplr_chunk_fwd), against the fp64 DPLR oracle on free erase
directions, and with KDA's binding (a = beta k, b = k * alpha, write key
beta k) against the KDA oracle and the KDA chunk engine."""
import numpy as np
import pytest

import kda_inputs as ki
import oracle
from kda_testlib import (assert_bf16_outputs, assert_bf16_state, assert_f32_close, small, to_dev, to_np, upload)
from oracle.dplr import dplr_recurrence

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    import kimi_delta_attention_21_b200 as K
    K.load_library()
    return K


def _free_directions(w, seed):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((w.B, w.S, w.H, w.Dk)).astype(np.float32)
    a /= np.linalg.norm(a, axis=-1, keepdims=True)
    b = rng.standard_normal((w.B, w.S, w.H, w.Dk)).astype(np.float32)
    b /= np.linalg.norm(b, axis=-1, keepdims=True)
    a *= rng.random((w.B, w.S, w.H, 1)).astype(np.float32)            # |a_t b_t^T| <= 1
    if w.dtype == "bf16":
        a, b = ki.round_bf16(a), ki.round_bf16(b)
    return a, b


ENGINES = ("dplr_recurrent_fwd", "dplr_chunk_fwd")


def _f32_close(engine, got, want, what):
    """fp32 inputs: the token-by-token form to the exact-path tolerance; the chunk form, whose outputs
    are sums of C + D_k fp32 products through T = (I + Ba)^{-1} with the hardware exponential, to 2e-4 of
    the largest magnitude (a wrong term shows at the scale of the outputs themselves)."""
    if engine == "dplr_recurrent_fwd":
        assert_f32_close(got, want, what)
    else:
        scale = max(1e-30, float(np.max(np.abs(want))))
        np.testing.assert_allclose(got, want, rtol=1e-4, atol=2e-4 * scale, err_msg=what)


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("B,S,H,D,dtype", [(1, 1, 1, 16, "f32"), (2, 70, 2, 24, "f32"), (1, 130, 3, 128, "f32"),
                                           (2, 200, 2, 128, "bf16"), (1, 65, 2, 40, "bf16"), (1, 330, 2, 18, "f32")])
def test_dplr_matches_oracle(K, engine, B, S, H, D, dtype):
    w = small("dplr", B, S, H, D, D, 16, dtype, seed=S + D, s0_std=0.05)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    a, b = _free_directions(w, S)
    o, sf = getattr(K, engine)(d["q"], d["k"], d["v"], to_dev(a, d["q"].dtype), to_dev(b, d["q"].dtype), z=d["z"],
                               g_min=w.g_min, initial_state=d["S0"])
    torch.cuda.synchronize()
    o_ref, s_ref = dplr_recurrence(inp["q"], inp["k"], inp["v"], a, b, z=inp["z"], g_min=w.g_min,
                                   initial_state=inp["S0"])
    if dtype == "f32":
        _f32_close(engine, to_np(o), o_ref, "o")
        _f32_close(engine, to_np(sf), s_ref, "final state")
    else:
        assert_bf16_outputs(to_np(o), o_ref, "o")
        assert_bf16_state(to_np(sf), s_ref, "final state")


@pytest.mark.parametrize("engine", ENGINES)
def test_dplr_with_kda_binding_matches_kda(K, engine):
    w = small("dplrk", 2, 300, 3, 128, 128, 16, "bf16", seed=12, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    la = oracle.log_decay(inp["z"], w.g_min)
    bk = (inp["beta"][..., None].astype(np.float64) * inp["k"]).astype(np.float32)
    ka = (inp["k"] * np.exp(la)).astype(np.float32)
    # fp32 inputs for the comparator (the bound vectors are not bf16 values)
    f = lambda x: to_dev(x, torch.float32)
    o, sf = getattr(K, engine)(f(inp["q"]), f(bk), f(inp["v"]), f(bk), f(ka), z=f(inp["z"]), g_min=w.g_min,
                               initial_state=d["S0"])
    o_kda, s_kda = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, initial_state=d["S0"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min,
                                     initial_state=inp["S0"])
    _f32_close(engine, to_np(o), o_ref, "DPLR with the KDA binding vs the KDA oracle")
    assert_bf16_outputs(to_np(o_kda), to_np(o), "KDA chunk engine vs DPLR with the KDA binding")
    assert_bf16_state(to_np(s_kda), to_np(sf), "final states")
