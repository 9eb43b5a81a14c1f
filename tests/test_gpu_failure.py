"""The device-side failure path without any fault: the library's bounded wait,
run on a barrier that nothing completes, gives up, records CR_ERR_TIMEOUT in
the workspace status word, and the context keeps working afterwards."""

import ctypes
import time

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_records_timeout_and_context_survives():
    from w4a8_rotated_quantized_b200 import binding
    import w4a8_rotated_quantized_b200 as cr

    ws = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    binding.cr_selftest_wait_timeout(ws)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    st = ctypes.c_int(-1)
    assert binding._lib.cr_read_device_status(binding._ptr(ws), ctypes.byref(st), binding._stream(ws.device)) == 0
    assert st.value == 7  # CR_ERR_TIMEOUT
    assert 1.0 < elapsed < 30.0  # the wait gave up after its limit, not at once and not never
    # the context is intact: a normal call on a fresh workspace runs and reports no error
    X = torch.randn((64, 512), device="cuda").to(torch.bfloat16)
    Xq, s = cr.cr_rotate_quant_act(X)
    torch.cuda.synchronize()
    assert np.isfinite(s.item()) and s.item() > 0
