"""The device status word on the GPU: a DYNAMIC global-scale reduction that
meets an Inf or NaN input reports FP4_ERR_NONFINITE through
fp4_device_status, keeps g finite (the largest finite bf16 / 2688), and the
next call on finite data is clean again.  Non-finite inputs are a value
test here (host-built tensors), nothing faults.  "Hardware FP4 inference for
speech on Blackwell", section "NVFP4, and the two ways it fails": the
format saturates, it never produces NaN."""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import fp4lib as L
from mxfp4_block_scaled_fp4_b200 import inputs

pytestmark = pytest.mark.gpu

BF16_MAX = float(np.frombuffer(np.uint32(0x7F7F0000).tobytes(), np.float32)[0])


@pytest.fixture(scope="module")
def ops():
    from mxfp4_block_scaled_fp4_b200 import ops as o
    return o


def _poisoned(M, K, seed):
    x = inputs.random_bf16(seed, (M, K)).clone()
    x[0, 3] = float("inf")
    x[M - 1, K - 5] = float("nan")
    return x


def _clean(ops):
    st, code = ops.device_status()
    assert st == L.FP4_OK and code == 0, (st, code)


# 2 x 2880 (11 KiB) takes the self-amax path, 512 x 4096 the amax pass
@pytest.mark.parametrize("M,K", [(2, 2880), (512, 4096)])
def test_quantize_dynamic_reports_nonfinite(ops, M, K):
    _clean(ops)
    q = ops.quantize(_poisoned(M, K, 11).cuda(), ops.NVFP4, ops.SCALES_MMA)
    st, code = ops.device_status()
    assert st == L.FP4_ERR_NONFINITE
    assert code == L.FP4_STATUS_NONFINITE_BIT
    g = q.g.item()
    assert np.isfinite(g) and np.float32(g) == np.float32(BF16_MAX) / np.float32(2688.0)
    # reading cleared the word; a finite input leaves it clear
    ops.quantize(inputs.random_bf16(12, (M, K)).cuda(), ops.NVFP4, ops.SCALES_MMA)
    _clean(ops)


def test_static_and_mxfp4_do_not_reduce(ops):
    """Only the DYNAMIC reduction looks at the whole tensor; STATIC and
    MXFP4 quantize element by element and report nothing."""
    _clean(ops)
    x = _poisoned(64, 1024, 13).cuda()
    ops.quantize(x, ops.NVFP4, ops.SCALES_MMA, g=torch.tensor([0.5], device="cuda"))
    ops.quantize(x, ops.MXFP4, ops.SCALES_MMA)
    _clean(ops)


# one-kernel path (M*K <= 32K values) and the chain
@pytest.mark.parametrize("M,N,K", [(1, 256, 4096), (32, 256, 4096)])
def test_fused_dynamic_reports_nonfinite(ops, M, N, K):
    _clean(ops)
    wq = ops.quantize_weights(inputs.random_bf16(14, (N, K), 0.02).cuda(), ops.NVFP4)
    g_out = torch.zeros(1, dtype=torch.float32, device="cuda")
    ops.gemm_fused(_poisoned(M, K, 15).cuda(), wq, torch.float32, g_out=g_out)
    st, code = ops.device_status()
    assert st == L.FP4_ERR_NONFINITE and code == L.FP4_STATUS_NONFINITE_BIT
    assert np.isfinite(g_out.item())
    ops.gemm_fused(inputs.random_bf16(16, (M, K)).cuda(), wq, torch.float32)
    _clean(ops)


def test_status_exchange_keeps_both_kinds(ops):
    """A timeout and a non-finite input in the same interval: the word holds
    both bits and the timeout decides the status."""
    _clean(ops)
    s = torch.cuda.current_stream().cuda_stream
    ops.quantize(_poisoned(2, 2880, 17).cuda(), ops.NVFP4, ops.SCALES_MMA)
    assert L.fp4_watchdog_selftest(20_000_000, s) == L.FP4_OK
    st, code = L.fp4_device_status(s)
    assert st == L.FP4_ERR_DEVICE_TIMEOUT
    assert code & L.FP4_STATUS_NONFINITE_BIT and code & (1 << 6)
    _clean(ops)
