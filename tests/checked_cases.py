"""The calls the checked-build test runs, shared by the test and the child
process that runs them on libkda_checked.so: the tensor-core chunk engine on
segmented sequences (maps, combine, chains; z and log-decay inputs, gate), the
GDN engine, the recurrent and chunkwise backward and the DPLR comparator (both forms).  As a script:
`python tests/checked_cases.py OUT.npz` runs them on the library the binding
loads (KDA_LIBRARY picks it) and saves the results with the device counters."""
import ctypes
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def run_cases():
    import torch

    import kda_inputs as ki
    import kimi_delta_attention_21_b200 as K
    from kda_testlib import small, upload
    from kimi_delta_attention_21_b200 import _lib as L
    out = {}

    def keep(name, t):
        out[name] = t.detach().float().cpu().numpy()

    # segmented tensor-core forward: 10 segments (maps, combine and chains), gated output
    w = small("chk1", 1, 2560, 2, 128, 128, 16, "bf16", seed=41, s0_std=0.02)
    d = upload(ki.make_inputs(w), w)
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"], initial_state=d["S0"],
                        gate_logits=d["gate"], engine="tc")
    keep("tc_o", o)
    keep("tc_sf", sf)
    # log-decay input, two batch rows, ragged length (8 segments)
    w = small("chk2", 2, 1999, 1, 128, 128, 16, "bf16", seed=43, s0_std=0.02)
    inp = ki.make_inputs(w)
    d = upload(inp, w)
    ld = torch.from_numpy(ki.round_bf16(-5.0 / (1.0 + np.exp(-inp["z"].astype(np.float64))))).float().cuda()
    o, sf = K.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], log_decay=ld, initial_state=d["S0"], engine="tc")
    keep("tcl_o", o)
    keep("tcl_sf", sf)
    # GDN engine
    w = small("chk3", 1, 1000, 2, 128, 128, 16, "bf16", seed=45, s0_std=0.02)
    d = upload(ki.make_inputs(w), w)
    o, sf = K.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], z=d["z"][..., 0].contiguous(), initial_state=d["S0"])
    keep("gdn_o", o)
    keep("gdn_sf", sf)
    # recurrent backward (three chunks, ragged)
    w = small("chk4", 1, 150, 2, 128, 128, 16, "bf16", seed=47, s0_std=0.1)
    d = upload(ki.make_inputs(w), w)
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    d_o = torch.randn((1, 150, 2, 128), generator=g, device="cuda").to(torch.bfloat16)
    d_st = torch.randn((1, 2, 128, 128), generator=g, device="cuda")
    grads = K.recurrent_bwd(d["q"], d["k"], d["v"], d["beta"], d_o, z=d["z"], initial_state=d["S0"],
                            d_final_state=d_st)
    for n, t in grads.items():
        if t is not None:
            keep("bwd_" + n, t)
    # chunkwise backward on the same inputs (three chunks, ragged)
    grads = K.chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d_o, z=d["z"], initial_state=d["S0"],
                        d_final_state=d_st)
    for n, t in grads.items():
        if t is not None:
            keep("bwd_chunk_" + n, t)
    # DPLR comparator (two chunks, ragged)
    w = small("chk5", 1, 100, 2, 128, 128, 16, "bf16", seed=49, s0_std=0.1)
    d = upload(ki.make_inputs(w), w)
    o, sf = K.dplr_recurrent_fwd(d["q"], d["k"], d["v"], d["k"], d["q"], z=d["z"], initial_state=d["S0"])
    keep("dplr_o", o)
    keep("dplr_sf", sf)
    o, sf = K.dplr_chunk_fwd(d["q"], d["k"], d["v"], d["k"], d["q"], z=d["z"], initial_state=d["S0"])
    keep("dplrc_o", o)
    keep("dplrc_sf", sf)
    torch.cuda.synchronize()
    lib = K.load_library()
    n, chk = ctypes.c_uint32(0), ctypes.c_int(-1)
    assert lib.kda_device_bounds_errors(ctypes.byref(n), 0, ctypes.byref(chk)) == 0
    t = ctypes.c_uint32(0)
    assert lib.kda_device_timeouts(ctypes.byref(t), 0) == 0
    return out, {"bounds_errors": n.value, "checked_build": chk.value, "timeouts": t.value,
                 "library": os.path.basename(L.LIB_PATH)}


if __name__ == "__main__":
    res, counters = run_cases()
    np.savez(sys.argv[1], **res, **{"_" + k: np.array(str(v)) for k, v in counters.items()})
