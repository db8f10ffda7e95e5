"""MXFP4 macro-block scaling on the GPU against the oracle (reading R9: one
binary32 second-level scale per row): the per-row scales, codes and E8M0
scales bit for bit on the activation-sweep shapes (both scale orders, both
MXFP4 rules) and for weights, and fp4_gemm_mbs within the stated tolerance
of the binary64 product of the two-level dequantized operands.

"FP4 n'existe pas : il existe des FP4, et chaque runtime choisit son
dialecte", section "L'ecart de qualite -- et comment il se reduit" (macro
block scaling: a second-level scale over groups of 32-blocks)."""
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


@pytest.mark.parametrize("M,K", [(1, 2880), (32, 8192), (512, 16384), (8192, 2880), (8192, 8192)])
@pytest.mark.parametrize("rule", [0, 1])
def test_mbs_quantize_matches_oracle(ops, orc, M, K, rule):
    x = inputs.act_sweep(M, K)
    xg = x.cuda()
    q_rm = ops.quantize(xg, 1, ops.SCALES_ROWMAJOR, mx_rule=rule, mbs=True)
    q_mma = ops.quantize(xg, 1, ops.SCALES_MMA, mx_rule=rule, mbs=True)
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    codes, scales, sigma = orc.quantize_mxfp4_mbs(x, rule)
    for q in (q_rm, q_mma):
        assert np.array_equal(bits(q.codes), codes)
        assert q.sigma.cpu().numpy().tobytes() == sigma.tobytes()
    assert np.array_equal(bits(q_rm.scales).reshape(scales.shape), scales)
    assert np.array_equal(bits(q_mma.scales), orc.scales_to_mma(scales))


def _ref(orc, a, w, rule):
    ca, sa, ga = orc.quantize_mxfp4_mbs(a, rule)
    cw, sw, gw = orc.quantize_mxfp4_mbs(w, rule)
    a_hat = orc.dequant(ca, sa, 1) * ga[:, None].astype(np.float64)
    w_hat = orc.dequant(cw, sw, 1) * gw[:, None].astype(np.float64)
    return orc.gemm(a_hat, w_hat), cw, gw


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (130, 264, 2880), (300, 520, 1056),
                                   (2048, 4096, 1024), (64, 2880, 2880), (8, 720, 7680)])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rule", [0, 1])
def test_mbs_gemm_matches_oracle(ops, orc, M, N, K, dt, rule):
    a = inputs.random_bf16(800 + M, (M, K))
    w = inputs.random_bf16(801 + N, (N, K), 0.02)
    aq = ops.quantize(a.cuda(), 1, ops.SCALES_MMA, mx_rule=rule, mbs=True)
    wq = ops.quantize_weights(w.cuda(), 1, mx_rule=rule, mbs=True)
    c = ops.gemm(aq, wq, dt)
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    ref, cw, gw = _ref(orc, a, w, rule)
    assert np.array_equal(bits(wq.codes), cw)
    assert wq.sigma.cpu().numpy().tobytes() == gw.tobytes()
    ok, worst, where = gemm_close(c, ref, dt)
    assert ok, f"worst err/bound {worst:.3g} at {where}"


def test_mbs_gemm_prefill_sampled(ops, orc):
    """The large prefill shape (pair kernel), 128 sampled rows x 128 columns."""
    M, N, K = 8192, 8192, 8192
    a, w = inputs.prefill(M, N, K)
    aq = ops.quantize(a.cuda(), 1, ops.SCALES_MMA, mbs=True)
    wq = ops.quantize_weights(w.cuda(), 1, mbs=True)
    c = ops.gemm(aq, wq, torch.bfloat16)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    ri = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 126, replace=False)]))
    ci = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 126, replace=False)]))
    rt, ct = torch.from_numpy(ri), torch.from_numpy(ci)
    ref, _, _ = _ref(orc, a[rt].contiguous(), w[ct].contiguous(), 0)
    ok, worst, where = gemm_close(c[rt.cuda()][:, ct.cuda()], ref, torch.bfloat16)
    assert ok, f"worst err/bound {worst:.3g} at {where}"


def test_mbs_nonfinite_row_is_reported(ops):
    ops.device_status()
    x = inputs.random_bf16(810, (64, 512)).clone()
    x[9, 5] = float("inf")
    q = ops.quantize(x.cuda(), 1, ops.SCALES_MMA, mbs=True)
    st, code = ops.device_status()
    assert st == L.FP4_ERR_NONFINITE and code == L.FP4_STATUS_NONFINITE_BIT
    assert torch.isfinite(q.sigma).all()


def test_mbs_argument_checks(ops):
    fake = 1 << 20
    q = L.fp4_quantize_act_ex
    assert q(fake, 4, 256, 0, 0, 0, L.opts(0, 0, fake), fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_INVALID_ARG                                 # NVFP4
    assert q(fake, 4, 256, 1, 0, 0, L.opts(32, 0, fake), fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_INVALID_ARG                                 # with a rotation
    assert q(fake, 4, 256, 1, 0, 0, L.opts(0, 0, fake + 2), fake, fake, fake, fake, 1 << 16,
             None) == L.FP4_ERR_MISALIGNED
    f = L.fp4_gemm_fused_ex
    assert f(fake, fake, fake, fake, 8, 16, 256, 1, 0, L.opts(0, 0, fake), fake, fake, 16, 0, fake,
             1 << 30, 0, None) == L.FP4_ERR_INVALID_ARG
    g = L.fp4_gemm_mbs
    assert g(fake, fake, None, fake, fake, fake, 4, 16, 256, fake, 16, 0, None, 0, 0, None) == \
        L.FP4_ERR_INVALID_ARG
