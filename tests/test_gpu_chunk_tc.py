"""The tcgen05 chunk engine (bf16, D_k = D_v = 128, chunk 64) against the oracle,
the fp64 chunk mirror (its workspace intermediates) and the exact SIMT engine."""
import numpy as np
import pytest

import kda_inputs as ki
import oracle
from oracle import chunk_mirror
from kda_testlib import (assert_bf16_outputs, assert_bf16_state, oracle_layer, rel_fro, small, to_np, upload)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REC = 74240  # workspace record bytes per (b, h, chunk)
SIG = 0      # (the gate logits are read by the state pass directly; no per-chunk gate tile)


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


def _bf16_view(ws_bytes):
    return np.frombuffer(ws_bytes.tobytes(), dtype=np.uint16)


def _bf(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _kmajor_image(buf, rows=64):
    """[2 atoms][rows][128 B] 128-byte-swizzled bf16 image -> (rows, 128)."""
    u = np.frombuffer(buf, dtype=np.uint16)
    out = np.zeros((rows, 128))
    for r in range(rows):
        for c in range(128):
            atom, chunk, e = c // 64, (c % 64) // 8, c % 8
            off = atom * rows * 128 + r * 128 + ((chunk ^ (r % 8)) * 16) + e * 2
            out[r, c] = _bf(u[off // 2:off // 2 + 1])[0]
    return out


def _atom_image(buf, rows):
    """One 128-byte-swizzled atom column [rows][128 B] of bf16 -> (rows, 64)."""
    u = np.frombuffer(buf, dtype=np.uint16)
    out = np.zeros((rows, 64))
    for r in range(rows):
        for c in range(64):
            off = r * 128 + (((c // 8) ^ (r % 8)) * 16) + (c % 8) * 2
            out[r, c] = _bf(u[off // 2:off // 2 + 1])[0]
    return out


def _mt_image(buf):
    u = np.frombuffer(buf, dtype=np.uint16)
    out = np.zeros((64, 64))
    for i in range(64):
        for r in range(64):
            off = i * 128 + (((r // 8) ^ (i % 8)) * 16) + (r % 8) * 2
            out[i, r] = _bf(u[off // 2:off // 2 + 1])[0]
    return out


def _close(got, want, what, tol=2e-2):
    scale = max(1.0, float(np.max(np.abs(want))))
    err = float(np.max(np.abs(got - want)))
    assert err <= tol * scale, f"{what}: max-abs {err:.3e} (scale {scale:.3e})"


def _rel(got, want, what, tol):
    """Max-abs error relative to the tensor's own largest entry (the images are bf16: 2^-9 rounding)."""
    scale = max(float(np.max(np.abs(want))), 1e-30)
    err = float(np.max(np.abs(got - want)))
    assert err <= tol * scale, f"{what}: max-abs {err:.3e} against largest |entry| {scale:.3e}"


@pytest.mark.parametrize("s0_std", [0.0, 0.05])
def test_workspace_intermediates_match_chunk_mirror(K, s0_std):
    """The records the prep writes (W, Q e^G, K e^{G_C - G}, M, U, e^{G_C}) against the fp64 mirror of
    the chunk algebra, each to a few bf16 roundings of its own scale; then, from a nonzero initial
    state, the state-corrected values V' = U - W S_0 formed from the record and the known S_0, and the
    outputs and final state of the whole two-chunk sequence, against the mirror chained chunk by chunk."""
    w = small("wsi", 1, 100, 2, 128, 128, 16, "bf16", seed=41, s0_std=s0_std)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    nb = K.chunk_workspace_bytes(1, 100, 2, 128, 128)
    assert nb == 1 * 2 * 2 * (REC + SIG)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"], engine="tc",
                        workspace=ws)
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    wsh = ws.cpu().numpy()
    la = oracle.log_decay(inp["z"], w.g_min)
    o_np, sf_np = to_np(o), to_np(sf)
    for h in range(2):
        S = np.zeros((128, 128)) if inp["S0"] is None else inp["S0"][0, h].astype(np.float64)
        for n in range(2):
            t0, t1 = 64 * n, min(100, 64 * n + 64)
            L = t1 - t0
            pad = lambda a: np.concatenate([a, np.zeros((64 - L,) + a.shape[1:])]) if L < 64 else a
            q = pad(inp["q"][0, t0:t1, h].astype(np.float64)); k = pad(inp["k"][0, t0:t1, h].astype(np.float64))
            v = pad(inp["v"][0, t0:t1, h].astype(np.float64)); beta = pad(inp["beta"][0, t0:t1, h].astype(np.float64))
            g = pad(la[0, t0:t1, h])
            mir = chunk_mirror.matrix_chunk(q, k, v, beta, g, S)
            G = mir["G"]
            rec = wsh[(h * 2 + n) * REC:(h * 2 + n + 1) * REC]
            wq = _kmajor_image(rec[0:32768], rows=128)  # stacked [-W; Q e^G]
            W_rec, U_rec = -wq[:64], _atom_image(rec[57344:73728], 128).T  # U stored as U^T
            tag = f"h{h} n{n} S0 std {s0_std}"
            _rel(wq[64:], q * np.exp(G), f"Q e^G {tag}", 8e-3)
            _rel(W_rec, mir["W"], f"W {tag}", 8e-3)
            _rel(_kmajor_image(rec[32768:49152]), k * np.exp(G[-1] - G), f"K~ {tag}", 8e-3)
            _rel(_mt_image(rec[49152:57344]), mir["M"].T, f"M {tag}", 8e-3)
            _rel(U_rec, mir["U"], f"U {tag}", 8e-3)
            gam = np.frombuffer(rec[73728:74240].tobytes(), dtype=np.float32)
            np.testing.assert_allclose(gam, np.exp(G[-1]), rtol=1e-4, atol=1e-30)
            # V' from the record and the exact entering state, against the mirror's
            _rel(U_rec - W_rec @ S, mir["Vp"], f"V' {tag}", 1.6e-2)
            # the engine's outputs of this chunk against the mirror's O (o~ of the chunk's tokens)
            _rel(o_np[0, t0:t1, h], mir["O"][:L], f"O {tag}", 1.6e-2)
            S = mir["S_next"]
        _rel(sf_np[0, h], S, f"final state h{h} S0 std {s0_std}", 1e-2)


@pytest.mark.parametrize("B,S,H", [(1, 1, 1), (1, 64, 1), (1, 65, 2), (2, 130, 3), (1, 200, 2), (3, 257, 27),
                                   (2, 300, 80)])
def test_tc_core_matches_oracle(K, B, S, H):
    w = small("tc", B, S, H, 128, 128, 16, "bf16", seed=S + 3 * H, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"], engine="tc")
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min,
                                     initial_state=inp["S0"])
    assert_bf16_outputs(to_np(o), o_ref, "o~")
    assert_bf16_state(to_np(sf), s_ref, "final_state")


# segment counts 10, 8, 8, 2 (no combine step) and 3 (one combine step)
@pytest.mark.parametrize("B,S,H,g_min", [(1, 2560, 2, -5.0), (2, 1999, 1, -5.0), (1, 2048, 1, -0.5),
                                         (1, 600, 1, -5.0), (1, 768, 2, -5.0)])
def test_tc_segmented_state_pass(K, B, S, H, g_min):
    """Sequences long enough for the state pass to be split into segments (each segment's affine
    map computed in parallel, the maps chained by the combine pass, the segments then run from
    their entering states); g_min = -0.5 keeps a long memory across segment boundaries."""
    w = small("seg", B, S, H, 128, 128, 16, "bf16", seed=S + 7 * H, s0_std=0.02, g_min=g_min)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    nc = (S + 63) // 64
    assert K.chunk_workspace_bytes(B, S, H, 128, 128) > B * H * nc * (REC + SIG)  # segments in use
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=g_min, initial_state=d["S0"],
                        engine="tc")
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=g_min,
                                     initial_state=inp["S0"])
    assert_bf16_outputs(to_np(o), o_ref, "o~")
    assert_bf16_state(to_np(sf), s_ref, "final_state")


def test_tc_matches_simt_engine(K):
    w = small("ts", 2, 333, 4, 128, 128, 16, "bf16", seed=5, s0_std=0.02, z_std=2.0)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    o1, s1 = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"], engine="tc")
    o2, s2 = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"], engine="simt")
    assert_bf16_outputs(to_np(o1), to_np(o2), "tc vs simt o~")
    assert rel_fro(to_np(s1), to_np(s2)) <= 1e-2


def test_tc_special_cases(K):
    w = small("sp", 1, 150, 2, 128, 128, 16, "bf16", seed=9, s0_std=0.1)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    zero_ld = torch.zeros(d["z"].shape, dtype=torch.float32, device="cuda")
    # alpha = 1, beta = 0: the state never changes and o_t = S_0^T q_t
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], torch.zeros_like(d["beta"]), log_decay=zero_ld,
                        initial_state=d["S0"], engine="tc")
    assert rel_fro(to_np(sf), inp["S0"]) <= 1e-6
    assert_bf16_outputs(to_np(o), np.einsum("bshc,bhcj->bshj", inp["q"].astype(np.float64),
                                            inp["S0"].astype(np.float64)))
    # alpha = 1 with writes (DeltaNet)
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], log_decay=zero_ld, initial_state=d["S0"], engine="tc")
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], log_decay=np.zeros_like(inp["z"]),
                                     initial_state=inp["S0"])
    assert_bf16_outputs(to_np(o), o_ref)
    assert_bf16_state(to_np(sf), s_ref)
    # empty sequence: final state = initial state
    e = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    o, sf = K.chunk_fwd(e, e, e, torch.empty(1, 0, 2, dtype=torch.bfloat16, device="cuda"), z=e,
                        initial_state=d["S0"], engine="tc")
    assert torch.equal(sf, d["S0"])


def test_tc_state_handoff_in_place(K):
    w = small("ho", 1, 300, 2, 128, 128, 16, "bf16", seed=12, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    o_all, s_all = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"], engine="tc")
    st = d["S0"].clone()
    outs = []
    for a, b in ((0, 64), (64, 100), (100, 300)):
        sl = lambda t: t[:, a:b].contiguous()
        o, _ = K.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["beta"]), z=sl(d["z"]), initial_state=st,
                           final_state=st, engine="tc")
        outs.append(o)
    assert_bf16_outputs(to_np(torch.cat(outs, 1)), to_np(o_all))
    assert rel_fro(to_np(st), to_np(s_all)) <= 1e-2


def test_tc_segmented_variants(K):
    """The segmented state pass with precomputed log-decay input, several batch rows and heads,
    and an in-place split-sequence handoff whose parts are themselves segmented, with the fused
    norm and gate (checked on the projected layer output)."""
    w = small("segv", 2, 1536, 3, 128, 128, 256, "bf16", seed=91, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    nc = (w.S + 63) // 64
    assert K.chunk_workspace_bytes(w.B, w.S, w.H, 128, 128) > w.B * w.H * nc * (REC + SIG)
    la = oracle.log_decay(inp["z"], w.g_min)
    ld = torch.from_numpy(np.ascontiguousarray(la, dtype=np.float32)).cuda()
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min,
                                     initial_state=inp["S0"])
    # precomputed log-decay (fp32) instead of z
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], log_decay=ld, g_min=w.g_min,
                        initial_state=d["S0"], engine="tc")
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    assert_bf16_outputs(to_np(o), o_ref, "o~ (log-decay input)")
    assert_bf16_state(to_np(sf), s_ref, "final_state (log-decay input)")
    # split-sequence handoff in place, with the fused gate; each part is long enough to be segmented
    st = d["S0"].clone()
    outs = []
    for a, b in ((0, 640), (640, 1536)):
        sl = lambda t: t[:, a:b].contiguous()
        og, _ = K.chunk_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["beta"]), z=sl(d["z"]), initial_state=st,
                            final_state=st, gate_logits=sl(d["gate"]), eps=w.eps, engine="tc")
        outs.append(og)
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    # the tolerance is stated on the layer output: project the normalised, gated rows (a row whose
    # o~ has a small norm is amplified by the normalisation, and the projection averages it)
    x = torch.cat(outs, 1).reshape(w.B * w.S, w.H * w.Dv)
    y = K.out_proj(x, d["W_o"])
    want = oracle.project(oracle.norm_gate(o_ref, inp["gate"], w.eps), inp["W_o"])
    assert_bf16_outputs(to_np(y).reshape(want.shape), want, "layer outputs (handoff)")
    assert_bf16_state(to_np(st), s_ref, "final_state (handoff)")


def test_tc_layer_with_fused_gate(K):
    w = ki.custom("lay", 2, 500, 4, 128, 128, 256, "bf16", seed=77)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    out = K.kda_forward(d["q"], d["k"], d["v"], d["z"], d["beta"], d["gate"], d["W_o"], None,
                        g_min=w.g_min, eps=w.eps, state_dtype=torch.float32, engine="tc")
    want = oracle_layer(inp, w)
    assert_bf16_outputs(to_np(out["outputs"]), want["outputs"], "outputs")
    assert_bf16_state(to_np(out["final_state"]), want["final_state"], "final_state")


def _random_case(seed):
    import random
    r = random.Random(seed)
    return dict(B=r.choice([1, 1, 2, 3]), S=r.randint(1, 3000), H=r.choice([1, 2, 3, 4]),
                g_min=r.choice([-5.0, -1.0, -0.3]), gated=r.random() < 0.5, s0=r.choice([0.0, 0.02]))


@pytest.mark.parametrize("seed", range(12))
def test_tc_random_shapes(K, seed):
    """Seeded random batch sizes, lengths (ragged tails, one to many segments), head counts, decay
    bounds, initial states and with or without the fused gate.  Gated rows are checked on the
    projected layer output, where the tolerance is stated (a row whose o~ is close to zero is
    amplified by the normalisation before the projection averages it); o~ otherwise."""
    c = _random_case(seed)
    B, S, H = c["B"], c["S"], c["H"]
    w = small("rnd", B, S, H, 128, 128, 256, "bf16", seed=4000 + seed, s0_std=c["s0"], g_min=c["g_min"])
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, initial_state=d["S0"],
                        gate_logits=d["gate"] if c["gated"] else None, eps=w.eps, engine="tc")
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min,
                                     initial_state=inp["S0"])
    what = f"B{B} S{S} H{H} g_min {w.g_min} gated {c['gated']}"
    if c["gated"]:
        y = K.out_proj(o.reshape(B * S, H * w.Dv), d["W_o"])
        want = oracle.project(oracle.norm_gate(o_ref, inp["gate"], w.eps), inp["W_o"])
        assert_bf16_outputs(to_np(y).reshape(want.shape), want, "layer outputs, " + what)
    else:
        assert_bf16_outputs(to_np(o), o_ref, "o~, " + what)
    assert_bf16_state(to_np(sf), s_ref, "final_state, " + what)


def test_tc_segment_windows(K):
    """Strong decay (z shifted by +5): every chunk's log-bound of the transition norm is below -100 (checked
    here from the same inputs: 64 tokens of at most the chunk's largest log(alpha); unit keys and beta < 1
    add nothing), so each segment's map runs a window of its last two or three chunks and writes A_g = 0.
    The segmented state pass (8 segments of 8 chunks) still matches the oracle."""
    w = small("win", 1, 4096, 16, 128, 128, 16, "bf16", seed=77, s0_std=0.5)
    inp = ki.make_inputs(w)
    inp["z"] = ki.round_bf16(inp["z"].astype(np.float64) + 5.0).astype(inp["z"].dtype)
    g = w.g_min / (1.0 + np.exp(-inp["z"].astype(np.float64)))            # (B, S, H, D_k)
    per_chunk = 64 * g.reshape(1, 64, 64, 16, 128).max(axis=(2, 4))        # (B, chunks, H)
    assert per_chunk.max() < -100.0
    d = upload(inp, w)
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"], engine="tc")
    torch.cuda.synchronize()
    assert _timeouts(K) == 0
    o_ref, s_ref = oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["beta"], z=inp["z"], g_min=w.g_min,
                                     initial_state=inp["S0"])
    assert_bf16_outputs(to_np(o), o_ref, "o~")
    assert_bf16_state(to_np(sf), s_ref, "final_state")
