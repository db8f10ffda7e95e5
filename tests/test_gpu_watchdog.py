"""Failure detection without a GPU fault: a kernel's bounded wait on a
barrier that nothing signals runs out after a short limit, the library's
watchdog word records it, the host reads FP4_ERR_DEVICE_TIMEOUT, and the
context keeps working (a normal quantize + GEMM still matches the oracle)."""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import fp4lib as L
from mxfp4_block_scaled_fp4_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(orc):
    from mxfp4_block_scaled_fp4_b200 import ops
    st, code = ops.device_status()                  # start clean
    assert st == L.FP4_OK and code == 0
    s = torch.cuda.current_stream().cuda_stream
    assert L.fp4_watchdog_selftest(50_000_000, s) == L.FP4_OK      # 50 ms limit
    st, code = L.fp4_device_status(s)
    assert st == L.FP4_ERR_DEVICE_TIMEOUT
    assert code & (1 << 6)
    st, code = L.fp4_device_status(s)               # reading clears the word
    assert st == L.FP4_OK and code == 0
    # the context is still usable
    a, w = inputs.pr1_tiny()
    c = ops.gemm(ops.quantize(a.cuda(), 0), ops.quantize_weights(w.cuda(), 0), torch.float32)
    torch.cuda.synchronize()
    c_ref, _ = orc.w4a4_reference(a, w, 0)
    err = np.abs(c.cpu().numpy() - c_ref)
    assert np.all(err <= 1e-4 * np.maximum(np.abs(c_ref), np.sqrt(np.mean(c_ref ** 2))))


def test_selftest_rejects_bad_limits():
    assert L.fp4_watchdog_selftest(0, None) == L.FP4_ERR_INVALID_ARG
    assert L.fp4_watchdog_selftest(5_000_000_000, None) == L.FP4_ERR_INVALID_ARG
