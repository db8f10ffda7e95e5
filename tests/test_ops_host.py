"""Host-side checks of the torch wrappers (ops.py), on CPU.  A caller's
output tensor must be exactly [M, N] with unit stride along N (rows may be
strided, as the column slices the decoder writes into), bf16 or fp32 and on
the operands' device, since the kernels write M x N values through it; a
quantized operand must hold the codes, scale bytes, global scale and
macro-block scales the kernels read, on that device."""
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import ops

CPU = torch.device("cpu")


def test_accepts_exact_and_row_strided_outputs():
    ops._check_out(torch.empty(4, 16, dtype=torch.bfloat16), 4, 16, CPU)
    ops._check_out(torch.empty(4, 16, dtype=torch.float32), 4, 16, CPU)
    wide = torch.empty(4, 64, dtype=torch.bfloat16)
    ops._check_out(wide[:, 16:32], 4, 16, CPU)       # ldc 64
    ops._check_out(torch.empty(0, 16, dtype=torch.bfloat16), 0, 16, CPU)


@pytest.mark.parametrize("bad", [
    lambda: torch.empty(3, 16, dtype=torch.bfloat16),          # too few rows
    lambda: torch.empty(4, 8, dtype=torch.bfloat16),           # too few columns
    lambda: torch.empty(16, 4, dtype=torch.bfloat16).t(),      # column-major
    lambda: torch.empty(4, 32, dtype=torch.bfloat16)[:, ::2],  # strided along N
    lambda: torch.empty(64, dtype=torch.bfloat16),             # 1-D
    lambda: torch.empty(4, 16, dtype=torch.float16),           # dtype
    lambda: torch.empty(4, 16, dtype=torch.bfloat16, device="meta"),   # device
])
def test_rejects_outputs_the_kernels_would_overrun(bad):
    with pytest.raises(ValueError):
        ops._check_out(bad(), 4, 16, CPU)


@pytest.fixture(scope="module")
def built():
    from mxfp4_block_scaled_fp4_b200 import build
    build.build()


def _q(rows=256, K=128, fmt=ops.NVFP4, **over):
    from mxfp4_block_scaled_fp4_b200 import fp4lib as L
    parts = dict(codes=torch.empty(rows, K // 2, dtype=torch.uint8),
                 scales=torch.empty(L.fp4_scale_bytes(rows, K, fmt, ops.SCALES_MMA),
                                    dtype=torch.uint8),
                 g=torch.ones(1, dtype=torch.float32), sigma=None)
    parts.update(over)
    return ops.Quantized(parts["codes"], parts["scales"], parts["g"], fmt, ops.SCALES_MMA,
                         rows, K, sigma=parts["sigma"])


def test_accepts_well_formed_operands(built):
    ops._check_quantized(_q(), "a", CPU)
    ops._check_quantized(_q(fmt=ops.MXFP4, sigma=torch.ones(256)), "a", CPU)
    ops._check_quantized(_q(rows=0), "a", CPU)
    ops._check_scalar(torch.ones(1), "g", CPU)


@pytest.mark.parametrize("over", [
    dict(codes=torch.empty(256, 32, dtype=torch.uint8)),                 # K/2 wrong
    dict(codes=torch.empty(255, 64, dtype=torch.uint8)),                 # rows wrong
    dict(codes=torch.empty(64, 256, dtype=torch.uint8).t()),             # not contiguous
    dict(codes=torch.empty(256, 64, dtype=torch.int8)),                  # dtype
    dict(scales=torch.empty(100, dtype=torch.uint8)),                    # too few scale bytes
    dict(g=torch.ones(1, dtype=torch.float64)),                          # g dtype
    dict(g=torch.ones(0)),                                               # g empty
    dict(sigma=torch.ones(100)),                                         # too few sigma
    dict(codes=torch.empty(256, 64, dtype=torch.uint8, device="meta")),  # device
])
def test_rejects_operands_the_kernels_would_overread(built, over):
    with pytest.raises(ValueError):
        ops._check_quantized(_q(**over), "a", CPU)
