"""Failure detection without a GPU fault: a bounded device wait that nothing
completes gives up after its limit, reports KDA_ERR_TIMEOUT to the host, and
the context keeps working afterwards."""
import ctypes

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import kimi_delta_attention_21_b200 as K
    from kimi_delta_attention_21_b200 import _lib
    lib = K.load_library()
    n = ctypes.c_uint32(0)
    assert lib.kda_device_timeouts(ctypes.byref(n), 1) == 0          # reset
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = lib.kda_selftest_wait_timeout(ctypes.c_void_p(status.data_ptr()), 20000, None)  # 20 ms
    assert st == _lib.KDA_OK
    torch.cuda.synchronize()
    assert int(status.item()) == _lib.KDA_ERR_TIMEOUT
    assert lib.kda_device_timeouts(ctypes.byref(n), 1) == 0 and n.value == 1
    # the context is still usable: an ordinary call runs and is correct
    z = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    g = K.gate(z, -4.0)
    torch.cuda.synchronize()
    assert torch.allclose(g, torch.full_like(g, -2.0))
    assert lib.kda_device_timeouts(ctypes.byref(n), 0) == 0 and n.value == 0


def test_selftest_validation():
    import kimi_delta_attention_21_b200 as K
    from kimi_delta_attention_21_b200 import _lib
    lib = K.load_library()
    assert lib.kda_selftest_wait_timeout(None, 10, None) == _lib.KDA_ERR_INVALID_ARG
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.kda_selftest_wait_timeout(ctypes.c_void_p(status.data_ptr()), 0, None) == _lib.KDA_ERR_INVALID_ARG
