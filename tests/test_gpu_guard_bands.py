"""Guard bands around every output and workspace: each entry point runs with
4 KiB of a known byte pattern directly before and after each buffer it writes
(outputs, in-place state, workspaces), and no byte of the pattern may change.
This is the host-side check for out-of-bounds stores that an address sanitizer
would otherwise catch."""
import ctypes

import numpy as np
import pytest

import kda_inputs as ki
from kda_testlib import small, upload

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A device buffer of `nbytes` with GUARD bytes of PATTERN on each side."""

    def __init__(self, nbytes):
        self.n = int(nbytes)
        self.raw = torch.full((GUARD + max(self.n, 1) + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")

    def view(self, dtype, shape):
        return self.raw[GUARD:GUARD + self.n].view(dtype).view(shape)

    def bytes_view(self):
        return self.raw[GUARD:GUARD + self.n]

    def check(self, what):
        torch.cuda.synchronize()
        lo = self.raw[:GUARD].cpu().numpy()
        hi = self.raw[GUARD + self.n:].cpu().numpy()
        bad_lo = np.flatnonzero(lo != PATTERN)
        bad_hi = np.flatnonzero(hi != PATTERN)
        assert bad_lo.size == 0, f"{what}: {bad_lo.size} bytes written before the buffer (last at -{GUARD - bad_lo[-1]})"
        assert bad_hi.size == 0, f"{what}: {bad_hi.size} bytes written after the buffer (first at +{bad_hi[0]})"


def _tensor(shape, dtype):
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    g = Guarded(n)
    return g, g.view(dtype, shape)


@pytest.fixture(scope="module")
def K():
    import kimi_delta_attention_21_b200 as K
    K.load_library()
    return K


def _chunk_case(K, w, engine, with_s0):
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    dt = d["q"].dtype
    s0 = torch.randn((w.B, w.H, w.Dk, w.Dv), device="cuda") * 0.02 if with_s0 else None
    go, o = _tensor((w.B, w.S, w.H, w.Dv), dt)
    gs, sf = _tensor((w.B, w.H, w.Dk, w.Dv), torch.float32)
    nws = K.chunk_workspace_bytes(w.B, w.S, w.H, w.Dk, w.Dv, dt, engine=engine)
    gw = Guarded(nws)
    K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], g_min=w.g_min, initial_state=s0,
                gate_logits=d["gate"], eps=w.eps, engine=engine, out=o, final_state=sf,
                workspace=gw.bytes_view() if nws else None)
    go.check(f"o ({engine})")
    gs.check(f"final_state ({engine})")
    gw.check(f"workspace ({engine}, {nws} bytes)")
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("S", [1, 63, 200, 4099])
def test_chunk_tc_writes_stay_inside(K, S):
    w = small(f"gb_tc{S}", 2, S, 3, 128, 128, 64, "bf16", seed=600 + S)
    _chunk_case(K, w, "tc", with_s0=True)


@pytest.mark.parametrize("dtype,Dk,Dv", [("f32", 16, 24), ("bf16", 128, 128), ("f32", 100, 36)])
def test_chunk_simt_writes_stay_inside(K, dtype, Dk, Dv):
    w = small(f"gb_simt{Dk}", 2, 77, 2, Dk, Dv, 32, dtype, seed=610 + Dk)
    _chunk_case(K, w, "simt", with_s0=True)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 128), ("bf16", 48)])
def test_decode_writes_stay_inside(K, dtype, D):
    w = small(f"gb_dec{D}", 150, 1, 4, D, D, 32, dtype, seed=620 + D)
    d = upload(ki.make_inputs(w), w)
    dt = d["q"].dtype
    gst, state = _tensor((w.B, w.H, w.Dk, w.Dv), torch.float32)
    state.copy_(torch.randn(state.shape, device="cuda") * 0.02)
    go, o = _tensor((w.B, w.H, w.Dv), dt)
    sl = lambda t: t[:, 0].contiguous()
    K.decode_step(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["beta"]), state, z=sl(d["z"]), g_min=w.g_min,
                  gate_logits=sl(d["gate"]), eps=w.eps, out=o)
    gst.check("decode state (in place)")
    go.check("decode o")


@pytest.mark.parametrize("dtype,N,Kd,Dm", [(torch.bfloat16, 300, 512, 256), (torch.bfloat16, 5, 2048, 2048),
                                           (torch.float32, 77, 96, 40)])
def test_projection_writes_stay_inside(K, dtype, N, Kd, Dm):
    x = (torch.randn((N, Kd), device="cuda")).to(dtype)
    W = (torch.randn((Dm, Kd), device="cuda") / Kd ** 0.5).to(dtype)
    gy, y = _tensor((N, Dm), dtype)
    K.out_proj(x, W, out=y)
    gy.check("out_proj y")


def test_norm_gate_and_gate_writes_stay_inside(K):
    from kimi_delta_attention_21_b200 import _lib
    lib = _lib.load()
    o = torch.randn((99, 3, 128), device="cuda").to(torch.bfloat16)
    gl = torch.randn((99, 3, 128), device="cuda").to(torch.bfloat16)
    gx, x = _tensor((99, 3, 128), torch.bfloat16)
    K.norm_gate(o, gl, out=x)
    gx.check("norm_gate x")
    z = torch.randn((1001,), device="cuda").to(torch.bfloat16)
    ga, la = _tensor((1001,), torch.float32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.kda_gate(ctypes.c_void_p(z.data_ptr()), _lib.KDA_BF16, 1001, -5.0, ctypes.c_void_p(la.data_ptr()),
                        stream) == 0
    ga.check("gate log_alpha")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_out_norm_gate_proj_writes_stay_inside(K, dtype):
    from kimi_delta_attention_21_b200 import _lib
    lib = _lib.load()
    N, H, Dv, Dm = 130, 4, 64, 192
    code = _lib.KDA_BF16 if dtype == torch.bfloat16 else _lib.KDA_F32
    o = torch.randn((N, H, Dv), device="cuda").to(dtype)
    gl = torch.randn((N, H, Dv), device="cuda").to(dtype)
    W = (torch.randn((Dm, H * Dv), device="cuda") / (H * Dv) ** 0.5).to(dtype)
    n = ctypes.c_size_t(0)
    assert lib.kda_out_norm_gate_proj_workspace_size(N, H, Dv, code, ctypes.byref(n)) == 0
    gw = Guarded(n.value)
    gy, y = _tensor((N, Dm), dtype)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.kda_out_norm_gate_proj(p(o), p(gl), p(W), N, H, Dv, Dm, 1e-6, p(y), code, p(gw.bytes_view()),
                                      n.value, stream) == 0
    gy.check("out_norm_gate_proj y")
    gw.check("out_norm_gate_proj workspace")
    gy2, y2 = _tensor((N, Dm), dtype)
    assert lib.kda_out_norm_gate_proj_noalloc(p(o), p(gl), p(W), N, H, Dv, Dm, 1e-6, p(y2), code, stream) == 0
    gy2.check("out_norm_gate_proj_noalloc y")


@pytest.mark.parametrize("engine,dtype,D", [("tc", "bf16", 128), ("simt", "f32", 24)])
def test_gdn_chunk_writes_stay_inside(K, engine, dtype, D):
    w = small(f"gb_gdn{D}", 2, 333, 3, D, D, 32, dtype, seed=640 + D)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    dt = d["q"].dtype
    zh = d["z"][..., 0].contiguous()
    s0 = torch.randn((w.B, w.H, w.Dk, w.Dv), device="cuda") * 0.02
    go, o = _tensor((w.B, w.S, w.H, w.Dv), dt)
    gs, sf = _tensor((w.B, w.H, w.Dk, w.Dv), torch.float32)
    nws = K.chunk_workspace_bytes(w.B, w.S, w.H, w.Dk, w.Dv, dt, engine=engine, scalar_decay=True)
    gw = Guarded(nws)
    K.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=zh, g_min=w.g_min, initial_state=s0,
                    gate_logits=d["gate"], eps=w.eps, engine=engine, out=o, final_state=sf,
                    workspace=gw.bytes_view() if nws else None)
    go.check(f"GDN o ({engine})")
    gs.check(f"GDN final_state ({engine})")
    gw.check(f"GDN workspace ({engine})")
