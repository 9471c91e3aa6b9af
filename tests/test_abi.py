"""The C-ABI library on the host: it loads, exports every declared symbol, its
struct layouts match the header, and argument validation rejects bad calls
before launching anything (no compute runs here)."""
import ctypes
import os
import re
import subprocess

import pytest

from kimi_delta_attention_21_b200 import _lib
from kimi_delta_attention_21_b200._lib import ChunkArgs, DecodeArgs, DplrArgs, RecBwdArgs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared()
    assert "kda_chunk_fwd" in names and "kda_decode_step" in names
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"{n} has no Python signature"
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (kda_\w+)", out))
    assert set(names) <= exported


def test_struct_layout_matches_header(tmp_path):
    structs = {"c": ("kda_chunk_args", ChunkArgs), "d": ("kda_decode_args", DecodeArgs),
               "r": ("kda_recurrent_bwd_args", RecBwdArgs), "p": ("kda_dplr_args", DplrArgs)}
    prog = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void){"]
    for tag, (cname, S) in structs.items():
        lines.append(f'printf("{tag} sizeof %zu\\n", sizeof({cname}));')
        for f, _ in S._fields_:
            lines.append(f'printf("{tag} {f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0;}")
    prog.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-o", str(exe), str(prog)])
    out = subprocess.check_output([str(exe)], text=True).split("\n")
    for line in out:
        if not line:
            continue
        tag, f, off = line.split()
        S = structs[tag][1]
        if f == "sizeof":
            assert ctypes.sizeof(S) == int(off), structs[tag][0]
        else:
            assert getattr(S, f).offset == int(off), (tag, f)


def test_status_strings():
    lib = _lib.load()
    names = [lib.kda_status_string(i).decode() for i in range(6)]
    assert names == ["KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_WORKSPACE",
                     "KDA_ERR_CUDA", "KDA_ERR_TIMEOUT"]
    assert lib.kda_status_string(99).decode() == "KDA_ERR_UNKNOWN"


# Fake device addresses: never dereferenced, because every call below fails
# validation before anything is launched.
BASE = 1 << 40


def _args(**kw):
    B, S, H, Dk, Dv = kw.pop("shape", (1, 8, 2, 16, 16))
    nk = B * S * H * Dk * 2
    a = ChunkArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_lib.KDA_BF16, g_min=-5.0, eps=1e-6)
    a.q = BASE
    a.k = BASE + 1 * (1 << 30)
    a.v = BASE + 2 * (1 << 30)
    a.z = BASE + 3 * (1 << 30)
    a.beta = BASE + 4 * (1 << 30)
    a.o = BASE + 5 * (1 << 30)
    a.final_state = BASE + 6 * (1 << 30)
    for k_, v_ in kw.items():
        setattr(a, k_, v_)
    assert nk < (1 << 30)
    return a


def _chunk_status(a):
    return _lib.load().kda_chunk_fwd(ctypes.byref(a))


@pytest.mark.parametrize("mut,status", [
    (dict(g_min=0.0), _lib.KDA_ERR_INVALID_ARG),
    (dict(g_min=float("nan")), _lib.KDA_ERR_INVALID_ARG),
    (dict(q=None), _lib.KDA_ERR_INVALID_ARG),
    (dict(q=BASE + 1), _lib.KDA_ERR_INVALID_ARG),            # misaligned for bf16
    (dict(z=None), _lib.KDA_ERR_INVALID_ARG),                # neither z nor log_decay
    (dict(o=BASE + 256), _lib.KDA_ERR_INVALID_ARG),          # o overlaps q (512 bytes)
    (dict(final_state=BASE + 2 * (1 << 30)), _lib.KDA_ERR_INVALID_ARG),  # state overlaps v
    (dict(shape=(1, 8, 2, 256, 16)), _lib.KDA_ERR_UNSUPPORTED),
    (dict(chunk=128), _lib.KDA_ERR_UNSUPPORTED),
    (dict(chunk=-1), _lib.KDA_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.KDA_ERR_UNSUPPORTED),
    (dict(engine=9), _lib.KDA_ERR_INVALID_ARG),
    (dict(H=0), _lib.KDA_ERR_INVALID_ARG),
    (dict(gate_logits=BASE + 7 * (1 << 30), eps=-1.0), _lib.KDA_ERR_INVALID_ARG),
])
def test_chunk_validation(mut, status):
    a = _args(**mut)
    assert _chunk_status(a) == status
    assert _lib.load().kda_last_error().decode() != ""


def test_tc_engine_refuses_uncovered_shapes():
    a = _args(shape=(1, 8, 2, 64, 64), engine=_lib.ENGINE_TC)
    assert _chunk_status(a) == _lib.KDA_ERR_UNSUPPORTED
    a = _args(shape=(1, 8, 2, 128, 128), engine=_lib.ENGINE_TC, dtype=_lib.KDA_F32)
    assert _chunk_status(a) == _lib.KDA_ERR_UNSUPPORTED
    a = _args(shape=(1, 8, 2, 128, 128), engine=_lib.ENGINE_TC, g_min=-8.0)
    assert _chunk_status(a) == _lib.KDA_ERR_UNSUPPORTED


def test_decode_and_gate_validation():
    lib = _lib.load()
    d = DecodeArgs(B=2, H=2, D_k=16, D_v=16, dtype=_lib.KDA_BF16, g_min=1.0, eps=1e-6,
                   q=BASE, k=BASE + (1 << 30), v=BASE + 2 * (1 << 30), z=BASE + 3 * (1 << 30),
                   beta=BASE + 4 * (1 << 30), state=BASE + 5 * (1 << 30), o=BASE + 6 * (1 << 30))
    assert lib.kda_decode_step(ctypes.byref(d)) == _lib.KDA_ERR_INVALID_ARG   # g_min > 0
    d.g_min = -5.0
    d.o = d.state                                                              # o overlaps state
    assert lib.kda_decode_step(ctypes.byref(d)) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_gate(BASE, _lib.KDA_BF16, 16, 0.5, BASE + (1 << 30), None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_gate(BASE, _lib.KDA_BF16, -1, -5.0, BASE + (1 << 30), None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_gate(BASE, _lib.KDA_BF16, 16, -5.0, BASE + 2, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_gate(BASE, _lib.KDA_BF16, 0, -5.0, None, None) == _lib.KDA_OK  # empty: nothing to do


def test_projection_validation():
    lib = _lib.load()
    assert lib.kda_out_proj(BASE, BASE + (1 << 30), 4, 0, 8, BASE + 2 * (1 << 30), 1, None) == _lib.KDA_ERR_INVALID_ARG
    # y overlapping x
    assert lib.kda_out_proj(BASE, BASE + (1 << 30), 4, 8, 8, BASE, 1, None) == _lib.KDA_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    assert lib.kda_out_norm_gate_proj_workspace_size(10, 2, 4, 1, ctypes.byref(n)) == _lib.KDA_OK
    assert n.value == 10 * 2 * 4 * 2
    assert lib.kda_out_norm_gate_proj(BASE, BASE + (1 << 30), BASE + 2 * (1 << 30), 10, 2, 4, 8, 1e-6,
                                      BASE + 3 * (1 << 30), 1, BASE + 4 * (1 << 30), 8, None) == _lib.KDA_ERR_WORKSPACE


def test_workspace_query_needs_no_device():
    a = _args(shape=(2, 100, 3, 32, 32))
    n = ctypes.c_size_t(123)
    assert _lib.load().kda_chunk_workspace_size(ctypes.byref(a), ctypes.byref(n)) == _lib.KDA_OK


def _expected_tc_workspace(B, S, H, sms=148):
    """Workspace of the tensor-core chunk engine, from the rule it follows: per-chunk records, and,
    with G segments, BH (G - 1) map slots (A image + Y), BH G entering states and a 4-byte log-bound
    per chunk, G the
    largest count for which the chain pass (BH G CTAs, so also the map pass, BH (G - 1) CTAs) fits
    in one wave, at least 4 chunks per segment, and no empty segment."""
    rec = 74240
    bh, nc = B * H, (S + 63) // 64
    per_sm = sms // bh
    g = min(per_sm, nc // 4)
    g = max(g, 1)
    L = (nc + g - 1) // g
    g = (nc + L - 1) // L
    ws = bh * nc * rec
    if g > 1:  # segment maps (A image + Y), entering states, per-chunk log-bounds for the map windows
        ws += bh * (g - 1) * (32768 + 65536) + bh * g * 128 * 128 * 4 + bh * nc * 4
    return ws, g


@pytest.mark.parametrize("B,S,H,G", [(1, 4096, 16, 8),      # prefill_4k: 8 segments of 8 chunks
                                     (8, 8192, 32, 1),      # batch_8x8k: one segment
                                     (1, 600, 1, 2), (1, 768, 2, 3), (1, 2560, 2, 10)])
def test_tc_workspace_and_segment_count(B, S, H, G):
    a = _args(shape=(B, S, H, 128, 128))
    n = ctypes.c_size_t(0)
    assert _lib.load().kda_chunk_workspace_size(ctypes.byref(a), ctypes.byref(n)) == _lib.KDA_OK
    want, g = _expected_tc_workspace(B, S, H)
    assert g == G
    assert n.value == want


def test_noalloc_size_check_cannot_be_wrapped():
    """A row count whose byte size wraps 64 bits is rejected on the host before
    any CUDA call (fake, aligned, non-NULL pointers: nothing is dereferenced)."""
    lib = _lib.load()
    H, Dv, Dm = 16, 128, 64
    N = (1 << 64) // (H * Dv * 2) + 1            # N * H * Dv * 2 wraps to 4096
    fake = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(4)]
    n0 = lib.kda_launch_count()
    st = lib.kda_out_norm_gate_proj_noalloc(fake[0], fake[1], fake[2], N, H, Dv, Dm, 1e-6, fake[3], _lib.KDA_BF16,
                                            None)
    assert st == _lib.KDA_ERR_UNSUPPORTED
    assert "scratch" in lib.kda_last_error().decode()
    assert lib.kda_launch_count() == n0


def test_checked_build_reports_itself():
    """build() makes a bounds-checked variant beside the library; each reports which one it is before
    any CUDA call (here, without a GPU, the counter read itself then fails with KDA_ERR_CUDA)."""
    import os
    pkg = os.path.dirname(_lib.LIB_PATH)
    for name, want in (("libkda.so", 0), ("libkda_checked.so", 1)):
        path = os.path.join(pkg, name)
        assert os.path.exists(path), f"{name} missing: run the build"
        lib = ctypes.CDLL(path)
        f = lib.kda_device_bounds_errors
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, ctypes.c_void_p]
        n, chk = ctypes.c_uint32(7), ctypes.c_int(-1)
        st = f(ctypes.byref(n), 0, ctypes.cast(ctypes.pointer(chk), ctypes.c_void_p))
        assert chk.value == want
        assert st in (_lib.KDA_OK, _lib.KDA_ERR_CUDA)
        assert f(None, 0, None) == _lib.KDA_ERR_INVALID_ARG


@pytest.mark.parametrize("B,S,H,Dk,Dv", [(1, 4096, 16, 128, 128), (2, 100, 3, 18, 13)])
def test_chunk_backward_and_dplr_workspace_rules(B, S, H, Dk, Dv):
    """The two SIMT chunk paths size their workspace as one record per (b, h, chunk): the chunkwise
    backward's C (4 Dk + 3 Dv + 3 C) + 2 Dk Dv + ceil(Dv / 16) Dk floats, the chunked DPLR's
    (Dk rounded to 4) + C (3 Dk + C + 2 Dv) + Dk Dv floats, each rounded up to 4 floats (C = 64)."""
    lib = _lib.load()
    C, nc = 64, (S + 63) // 64
    r4 = lambda x: (x + 3) // 4 * 4
    want_bwd = B * H * nc * r4(C * (4 * Dk + 3 * Dv + 3 * C) + 2 * Dk * Dv + (Dv + 15) // 16 * Dk) * 4
    want_dplr = B * H * nc * r4(r4(Dk) + C * (3 * Dk + C + 2 * Dv) + Dk * Dv) * 4
    n = ctypes.c_size_t(0)
    rb = _lib.RecBwdArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_lib.KDA_BF16, g_min=-5.0)
    assert lib.kda_chunk_bwd_workspace_size(ctypes.byref(rb), ctypes.byref(n)) == _lib.KDA_OK
    assert n.value == want_bwd
    da = _lib.DplrArgs(B=B, S=S, H=H, D_k=Dk, D_v=Dv, dtype=_lib.KDA_BF16, g_min=-5.0)
    assert lib.kda_dplr_chunk_workspace_size(ctypes.byref(da), ctypes.byref(n)) == _lib.KDA_OK
    assert n.value == want_dplr


def test_chunked_dplr_refuses_a_short_workspace():
    """Validated on the host before any launch (fake, aligned, non-NULL device pointers)."""
    lib = _lib.load()
    B, S, H, D = 1, 130, 2, 32
    fake = [ctypes.c_void_p(0x1000000 * (i + 1)) for i in range(8)]
    da = _lib.DplrArgs(B=B, S=S, H=H, D_k=D, D_v=D, dtype=_lib.KDA_BF16, q=fake[0], k=fake[1], v=fake[2], a=fake[3],
                       b=fake[4], z=fake[5], g_min=-5.0, o=fake[6])
    n = ctypes.c_size_t(0)
    assert lib.kda_dplr_chunk_workspace_size(ctypes.byref(da), ctypes.byref(n)) == _lib.KDA_OK
    n0 = lib.kda_launch_count()
    assert lib.kda_dplr_chunk_fwd(ctypes.byref(da), fake[7], n.value - 16) == _lib.KDA_ERR_WORKSPACE
    assert lib.kda_dplr_chunk_fwd(ctypes.byref(da), None, n.value) == _lib.KDA_ERR_WORKSPACE
    assert lib.kda_launch_count() == n0


def test_chunk_backward_validation():
    """Host-side refusals of kda_chunk_bwd before any launch (fake, aligned, non-NULL device pointers)."""
    lib = _lib.load()
    fake = [ctypes.c_void_p(0x1000000 * (i + 1)) for i in range(13)]
    B, S, H, D = 1, 130, 2, 32

    def args(**kw):
        base = dict(B=B, S=S, H=H, D_k=D, D_v=D, dtype=_lib.KDA_BF16, q=fake[0], k=fake[1], v=fake[2], z=fake[3],
                    g_min=-5.0, beta=fake[4], d_o=fake[5], dq=fake[6], dk=fake[7], dv=fake[8], dbeta=fake[9],
                    dz=fake[10])
        base.update(kw)
        return _lib.RecBwdArgs(**base)

    n = ctypes.c_size_t(0)
    a = args()
    assert lib.kda_chunk_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == _lib.KDA_OK
    n0 = lib.kda_launch_count()
    a.workspace, a.workspace_bytes = fake[11], n.value - 16
    assert lib.kda_chunk_bwd(ctypes.byref(a)) == _lib.KDA_ERR_WORKSPACE
    big = args(D_k=129)
    assert lib.kda_chunk_bwd_workspace_size(ctypes.byref(big), ctypes.byref(n)) == _lib.KDA_ERR_UNSUPPORTED
    assert lib.kda_chunk_bwd(ctypes.byref(big)) == _lib.KDA_ERR_UNSUPPORTED
    pos = args(g_min=0.5)
    assert lib.kda_chunk_bwd(ctypes.byref(pos)) == _lib.KDA_ERR_INVALID_ARG
    nodo = args(d_o=None)
    nodo.workspace, nodo.workspace_bytes = fake[11], 1 << 40
    assert lib.kda_chunk_bwd(ctypes.byref(nodo)) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_launch_count() == n0


def test_simt_chunk_paths_refuse_too_many_chunks():
    """One CTA per (b, h, chunk): a size query past 2^31 - 1 of them is refused, not wrapped."""
    lib = _lib.load()
    n = ctypes.c_size_t(0)
    S = 64 * (1 << 28)                                    # 2^28 chunks per sequence, 16 heads
    rb = _lib.RecBwdArgs(B=1, S=S, H=16, D_k=128, D_v=128, dtype=_lib.KDA_BF16, g_min=-5.0)
    assert lib.kda_chunk_bwd_workspace_size(ctypes.byref(rb), ctypes.byref(n)) == _lib.KDA_ERR_UNSUPPORTED
    da = _lib.DplrArgs(B=1, S=S, H=16, D_k=128, D_v=128, dtype=_lib.KDA_BF16, g_min=-5.0)
    assert lib.kda_dplr_chunk_workspace_size(ctypes.byref(da), ctypes.byref(n)) == _lib.KDA_ERR_UNSUPPORTED
    ok = _lib.RecBwdArgs(B=1, S=64 * (1 << 20), H=16, D_k=128, D_v=128, dtype=_lib.KDA_BF16, g_min=-5.0)
    assert lib.kda_chunk_bwd_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == _lib.KDA_OK
