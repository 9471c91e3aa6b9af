"""The bounds-checked build (libkda_checked.so, compiled with -DKDA_CHECKED):
in a child process that loads it, the segmented tensor-core forward, the GDN
engine, the recurrent and chunkwise backward passes and the DPLR comparator
find no write outside its buffer, and give the results the normal library
gives on the same inputs (bit for bit where no floating-point atomics are
involved)."""
import os
import subprocess
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_checked_build_runs_clean_and_matches(tmp_path):
    import kimi_delta_attention_21_b200 as K
    lib_checked = os.path.join(os.path.dirname(K.__file__), "libkda_checked.so")
    assert os.path.exists(lib_checked), "build it: python -m kimi_delta_attention_21_b200.build --checked"
    out = tmp_path / "checked.npz"
    env = dict(os.environ, KDA_LIBRARY="libkda_checked.so")
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_cases.py"), str(out)], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-4000:]
    got = np.load(out)
    assert str(got["_library"]) == "libkda_checked.so" and str(got["_checked_build"]) == "1"
    assert str(got["_bounds_errors"]) == "0", "the checked build skipped writes outside their buffers"
    assert str(got["_timeouts"]) == "0"

    import checked_cases
    want, counters = checked_cases.run_cases()  # the normal library, in this process
    assert counters["checked_build"] == 0 and counters["bounds_errors"] == 0
    assert set(want) == {k for k in got.files if not k.startswith("_")}
    for k, v in want.items():
        g = got[k]
        if k.startswith("bwd_"):  # fp32 atomics add in any order (value-column slices, dbeta terms)
            scale = max(1e-30, float(np.abs(v).max()))
            np.testing.assert_allclose(g, v, rtol=1e-5, atol=1e-6 * scale, err_msg=k)
        else:
            assert np.array_equal(g, v), f"{k}: checked and normal builds differ"
