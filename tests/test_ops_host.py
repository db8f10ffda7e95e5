"""Host-side checks of the torch wrappers (ops.py), on CPU: a caller's
output tensor must be exactly [M, N] with unit stride along N (rows may be
strided, as the column slices the decoder writes into), bf16 or fp32 and on
the operands' device, since the kernels write M x N values through it."""
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
