"""fp4_quantize_act_noalloc against fp4_quantize_act (GPU).

The allocation-free entry point serves callers that cannot allocate device
memory (engines that reserve all memory at start-up, plug-ins inside a host
framework that owns the allocator, latency-critical paths that cannot pay
for cudaMalloc's implicit synchronization); its scratch is a fixed device
array inside the library.  Its outputs must equal those of the workspace entry point bit for
bit (quantized codes, scales and the global scale are compared exactly, as
in every quantizer test), on two calls in a row, so that the array's
leftover contents from the first call cannot change the second.

This file is collected last so that a failure here cannot hide others.
"""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import fp4lib as L
from mxfp4_block_scaled_fp4_b200 import inputs

pytestmark = pytest.mark.gpu


def _run(entry, x, fmt, layout, gmode, g_in=None):
    rows, K = x.shape
    dev = x.device
    codes = torch.full((rows, K // 2), 0xAB, dtype=torch.uint8, device=dev)
    scales = torch.full((L.fp4_scale_bytes(rows, K, fmt, layout),), 0xCD, dtype=torch.uint8,
                        device=dev)
    g = torch.tensor([g_in if g_in is not None else -1.0], dtype=torch.float32, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    if entry == "ws":
        nbytes = L.fp4_workspace_bytes(rows, 0, K, fmt)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        st = L.fp4_quantize_act(x.data_ptr(), rows, K, fmt, layout, gmode, g.data_ptr(),
                                codes.data_ptr(), scales.data_ptr(), ws.data_ptr(), nbytes, s)
    else:
        st = L.fp4_quantize_act_noalloc(x.data_ptr(), rows, K, fmt, layout, gmode, g.data_ptr(),
                                        codes.data_ptr(), scales.data_ptr(), s)
    assert st == L.FP4_OK, L.fp4_status_string(st)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), g.cpu().numpy()


@pytest.mark.parametrize("fmt,gmode", [(L.FP4_NVFP4, L.FP4_GLOBAL_DYNAMIC),
                                       (L.FP4_NVFP4, L.FP4_GLOBAL_STATIC),
                                       (L.FP4_MXFP4, L.FP4_GLOBAL_DYNAMIC)])
@pytest.mark.parametrize("layout", [L.FP4_SCALES_MMA, L.FP4_SCALES_ROWMAJOR])
def test_noalloc_matches_workspace_entry_two_calls(fmt, gmode, layout):
    L.lib()
    # two different inputs in a row: the second call must not see the first's scratch
    # (16 x 512 is small enough that the DYNAMIC path skips the amax pass)
    shapes = [(512, 8192), (32, 2880), (16, 512)]
    for i, (M, K) in enumerate(shapes):
        x = inputs.act_sweep(M, K).cuda()
        g_in = 0.05 if gmode == L.FP4_GLOBAL_STATIC else None
        ref = _run("ws", x, fmt, layout, gmode, g_in)
        got = _run("noalloc", x, fmt, layout, gmode, g_in)
        assert np.array_equal(got[0], ref[0]), f"codes differ on call {i + 1}"
        assert np.array_equal(got[1], ref[1]), f"scales differ on call {i + 1}"
        assert got[2].tobytes() == ref[2].tobytes(), f"global scale differs on call {i + 1}"


def test_noalloc_rejects_bad_arguments_before_launch():
    L.lib()
    fake = 1 << 20
    assert L.fp4_quantize_act_noalloc(fake, 4, 100, 0, 0, 0, fake, fake, fake, None) == \
        L.FP4_ERR_UNSUPPORTED_SHAPE
    assert L.fp4_quantize_act_noalloc(fake, 4, 256, 9, 0, 0, fake, fake, fake, None) == \
        L.FP4_ERR_INVALID_ARG
