"""The GEMM epilogue that emits the next layer's FP4 activation
(fp4_gemm_quant) against the oracle: the bf16 C it stores beside the codes
is within the GEMM tolerance of the oracle's binary64 product, and the
emitted codes, scales (both orders, padding included) are bit for bit the
oracle quantizer's output on that same bf16 C (STATIC global scale for
NVFP4; MXFP4 with either scale rule; optionally after the online
rotation).  The emitted activation then feeds a second fp4_gemm.

"FP4 n'existe pas : il existe des FP4, et chaque runtime choisit son
dialecte", section "TensorRT-LLM 1.3 : NVFP4 natif, verrouille NVIDIA":
quantization, scaling, matmul and de-scaling in one launch, with no HBM
round trip between the steps."""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import fp4lib as L
from mxfp4_block_scaled_fp4_b200 import inputs
from tests.parity import bits, gemm_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from mxfp4_block_scaled_fp4_b200 import ops as o
    return o


# the CTA-pair kernel (M > 128 with many tiles) and the 128-row kernel with
# 256-, 128- and 64-wide tiles (few tiles: the quantizing epilogue takes no K
# split); ragged M, N % 32 == 0, K tails
SHAPES = [(1, 256, 256), (130, 288, 2880), (300, 544, 1056), (2048, 4096, 1024),
          (64, 2880, 2880), (8, 736, 7680), (256, 2880, 7680), (129, 4096, 512)]


def _ref_c(orc, a, w, fmt):
    ca, sa, ga = orc.quantize(a, fmt)
    cw, sw, gw = orc.quantize(w, fmt)
    return orc.gemm(orc.dequant(ca, sa, fmt, ga), orc.dequant(cw, sw, fmt, gw))


def _check_emitted(orc, q, c_gpu, out_fmt, g_out, had, rule):
    codes, scales, _ = orc.quantize_ex(c_gpu.cpu(), out_fmt, g_out if out_fmt == 0 else None,
                                       hadamard_n=had, operand="act", rule=rule)
    assert np.array_equal(bits(q.codes), codes)
    if q.layout == L.FP4_SCALES_MMA:
        assert np.array_equal(bits(q.scales), orc.scales_to_mma(scales))
    else:
        assert np.array_equal(bits(q.scales).reshape(scales.shape), scales)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("fmt,out_fmt", [(0, 0), (1, 1), (0, 1)])
def test_emitted_activation_matches_oracle(ops, orc, M, N, K, fmt, out_fmt):
    a = inputs.random_bf16(900 + M, (M, K))
    w = inputs.random_bf16(901 + N, (N, K), 0.02)
    aq = ops.quantize(a.cuda(), fmt, ops.SCALES_MMA)
    wq = ops.quantize_weights(w.cuda(), fmt)
    g_out = torch.tensor([0.004], dtype=torch.float32, device="cuda")
    for layout in (ops.SCALES_MMA, ops.SCALES_ROWMAJOR):
        q, c = ops.gemm_quant(aq, wq, out_fmt, layout, g_out, with_c=True)
        q2, none = ops.gemm_quant(aq, wq, out_fmt, layout, g_out, with_c=False)
        torch.cuda.synchronize()
        st, code = ops.device_status()
        assert st == 0 and code == 0 and none is None
        ok, worst, where = gemm_close(c, _ref_c(orc, a, w, fmt), torch.bfloat16)
        assert ok, f"worst err/bound {worst:.3g} at {where}"
        _check_emitted(orc, q, c, out_fmt, 0.004, 0, 0)
        assert torch.equal(q.codes, q2.codes) and torch.equal(q.scales, q2.scales)


@pytest.mark.parametrize("M,N,K", [(300, 544, 1056), (64, 2880, 2880), (2048, 4096, 1024)])
@pytest.mark.parametrize("out_fmt,had,rule", [(0, 16, 0), (0, 32, 0), (1, 32, 1), (1, 0, 1)])
def test_emitted_activation_rotated_and_oas(ops, orc, M, N, K, out_fmt, had, rule):
    a = inputs.random_bf16(910 + M, (M, K))
    w = inputs.random_bf16(911 + N, (N, K), 0.02)
    aq = ops.quantize(a.cuda(), 0, ops.SCALES_MMA)
    wq = ops.quantize_weights(w.cuda(), 0)
    g_out = torch.tensor([0.002], dtype=torch.float32, device="cuda")
    q, c = ops.gemm_quant(aq, wq, out_fmt, ops.SCALES_MMA, g_out, hadamard=had, mx_rule=rule,
                          with_c=True)
    torch.cuda.synchronize()
    _check_emitted(orc, q, c, out_fmt, 0.002, had, rule)


@pytest.mark.parametrize("fmt", [0, 1])
def test_emitted_activation_feeds_the_next_gemm(ops, orc, fmt):
    """Two layers: C1 = A.W1^T emitted as FP4, then C2 = C1_hat.W2^T."""
    M, N1, N2, K = 200, 1024, 768, 2048
    a = inputs.random_bf16(920, (M, K))
    w1 = inputs.random_bf16(921, (N1, K), 0.02)
    w2 = inputs.random_bf16(922, (N2, N1), 0.02)
    aq = ops.quantize(a.cuda(), fmt, ops.SCALES_MMA)
    w1q, w2q = ops.quantize_weights(w1.cuda(), fmt), ops.quantize_weights(w2.cuda(), fmt)
    g1 = torch.tensor([0.0005], dtype=torch.float32, device="cuda")
    q1, c1 = ops.gemm_quant(aq, w1q, fmt, ops.SCALES_MMA, g1, with_c=True)
    c2 = ops.gemm(q1, w2q, torch.float32)
    torch.cuda.synchronize()
    c1_codes, c1_scales, g1v = orc.quantize(c1.cpu(), fmt, 0.0005 if fmt == 0 else None)
    cw, sw, gw = orc.quantize(w2, fmt)
    ref = orc.gemm(orc.dequant(c1_codes, c1_scales, fmt, g1v), orc.dequant(cw, sw, fmt, gw))
    ok, worst, where = gemm_close(c2, ref, torch.float32)
    assert ok, f"worst err/bound {worst:.3g} at {where}"


def test_gemm_quant_argument_checks(ops):
    fake = 1 << 20
    f = L.fp4_gemm_quant
    # N % 32 (the next layer's K)
    assert f(fake, fake, fake, fake, fake, fake, 4, 48, 256, 0, 0, 0, None, fake, fake, fake, None,
             0, None, 0, 0, None) == L.FP4_ERR_UNSUPPORTED_SHAPE
    # NVFP4 output needs g_out
    assert f(fake, fake, fake, fake, fake, fake, 4, 64, 256, 0, 0, 0, None, None, fake, fake, None,
             0, None, 0, 0, None) == L.FP4_ERR_INVALID_ARG
    # OAS rule with NVFP4 output
    assert f(fake, fake, fake, fake, fake, fake, 4, 64, 256, 0, 0, 0, L.opts(0, 1), fake, fake,
             fake, None, 0, None, 0, 0, None) == L.FP4_ERR_INVALID_ARG
