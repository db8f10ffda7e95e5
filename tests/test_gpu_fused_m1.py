"""fp4_gemm_fused with one activation row (the decode step of one token)
against the oracle: ragged K (a partial last 256-value step), rows longer
than one K slice, the largest K of the fused path, N below and above the
SM count, both formats and output types, STATIC and DYNAMIC global scales,
rotations, the overflow-aware MXFP4 rule, shared-SM launches (max_sms)
that change the K split, and the degenerate inputs."""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import inputs
from tests.parity import gemm_close

pytestmark = pytest.mark.gpu
DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module")
def ops():
    from mxfp4_block_scaled_fp4_b200 import ops as o
    return o


def _case(ops, orc, a, w, fmt, dt, had=0, rule=0, g=None, max_sms=0):
    ca, sa, ga = orc.quantize_ex(a, fmt, g, hadamard_n=had, operand="act", rule=rule)
    cw, sw, gw = orc.quantize_ex(w, fmt, None, hadamard_n=had, operand="w", rule=rule)
    c_ref = orc.gemm(orc.dequant(ca, sa, fmt, ga), orc.dequant(cw, sw, fmt, gw))
    wq = ops.quantize_weights(w.cuda(), fmt, hadamard=had, mx_rule=rule)
    g_in = None if g is None else torch.tensor([g], dtype=torch.float32, device="cuda")
    g_out = torch.zeros(1, dtype=torch.float32, device="cuda")
    c = ops.gemm_fused(a.cuda(), wq, DT[dt], g_a=g_in, g_out=None if g is not None else g_out,
                       max_sms=max_sms, mx_rule=rule)
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    ok, worst, where = gemm_close(c, c_ref, DT[dt])
    assert ok, f"worst err/bound {worst:.3g} at {where}"
    if fmt == 0 and g is None:
        assert np.float32(g_out.item()).tobytes() == np.float32(ga).tobytes()
    return c


# (N, K): K = 32, 96, 1056 and 2880 (a partial last step), 4096, 7680 and
# 14336 (several slices of a split K), 65536 (beyond the one-kernel path:
# the amax -> quantize -> GEMM chain); N a multiple of 8, as the entry point
# requires, from 8 to more 128-row tiles than SMs
SHAPES = [(8, 32), (8, 96), (40, 1056), (264, 2880), (2880, 2880), (4096, 4096), (720, 7680),
          (136, 14336), (8, 65536), (4104, 1024)]


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_m1_shapes(ops, orc, N, K, fmt, dt):
    a = inputs.random_bf16(700 + K, (1, K))
    w = inputs.random_bf16(800 + N, (N, K), 0.02)
    _case(ops, orc, a, w, fmt, dt)


@pytest.mark.parametrize("fmt,had,rule", [(0, 16, 0), (0, 32, 0), (1, 16, 1), (1, 32, 0)])
def test_m1_rotated(ops, orc, fmt, had, rule):
    a = inputs.random_bf16(71, (1, 2880))
    w = inputs.random_bf16(72, (1000, 2880), 0.02)
    _case(ops, orc, a, w, fmt, "f32", had=had, rule=rule)


def test_m1_overflow_aware_rule(ops, orc):
    a = inputs.random_bf16(73, (1, 4096))
    w = inputs.random_bf16(74, (520, 4096), 0.02)
    _case(ops, orc, a, w, 1, "f32", rule=1)


@pytest.mark.parametrize("g", [1.0, 0.01])
def test_m1_static_global_scale(ops, orc, g):
    a = inputs.random_bf16(75, (1, 2048))
    w = inputs.random_bf16(76, (512, 2048), 0.02)
    _case(ops, orc, a, w, 0, "f32", g=g)


@pytest.mark.parametrize("max_sms", [1, 3, 37])
def test_m1_few_ctas(ops, orc, max_sms):
    """Shared-SM launches: the K split is chosen for a handful of SMs."""
    a = inputs.random_bf16(77, (1, 7680))
    w = inputs.random_bf16(78, (2888, 7680), 0.02)
    _case(ops, orc, a, w, 0, "f32", max_sms=max_sms)


def test_m1_degenerate_inputs(ops, orc):
    """All-zero activation (g = 1, zero output), an outlier block and bf16
    subnormals in one row, and a weight row of zeros."""
    K, N = 1024, 304
    w = inputs.random_bf16(79, (N, K), 0.02)
    w[5] = 0
    c = _case(ops, orc, torch.zeros(1, K, dtype=torch.bfloat16), w, 0, "f32")
    assert torch.count_nonzero(c) == 0
    a = inputs.random_bf16(80, (1, K))
    a[0, 16:32] = 0
    a[0, 32] = 1000.0
    a[0, 64:80] = torch.tensor(1e-40, dtype=torch.bfloat16)
    for fmt in (0, 1):
        c = _case(ops, orc, a, w, fmt, "f32")
        assert c[0, 5].item() == 0.0


def test_m1_repeated_calls_are_deterministic(ops):
    a, w = inputs.decode(1, 4096, 14336)
    wq = ops.quantize_weights(w.cuda(), 0)
    x = a.cuda()
    outs = [ops.gemm_fused(x, wq, torch.float32).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
