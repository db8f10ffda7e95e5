"""GPU W4A4 GEMM (quantize on the GPU, tcgen05 GEMM) against the oracle's
binary64 product of its own dequantized operands, within the stated
tolerance (tests/parity.py), on the tiny outlier problem, ragged shapes
that span several tiles and a K tail, the decode shapes through the fused
entry point, and sampled outputs of the full-size prefill shapes."""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import inputs
from tests.parity import bits, gemm_close

pytestmark = pytest.mark.gpu
DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module")
def ops():
    from mxfp4_block_scaled_fp4_b200 import ops as o
    return o


def run_pair(ops, orc, a, w, fmt, dt, fused=False):
    aq_ref = orc.quantize(a, fmt)
    wq_ref = orc.quantize(w, fmt)
    c_ref = orc.gemm(orc.dequant(aq_ref[0], aq_ref[1], fmt, aq_ref[2]),
                     orc.dequant(wq_ref[0], wq_ref[1], fmt, wq_ref[2]))
    wq = ops.quantize_weights(w.cuda(), fmt)
    if fused:
        g_out = torch.zeros(1, dtype=torch.float32, device="cuda")
        c = ops.gemm_fused(a.cuda(), wq, DT[dt], g_out=g_out)
    else:
        aq = ops.quantize(a.cuda(), fmt, ops.SCALES_MMA)
        c = ops.gemm(aq, wq, DT[dt])
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    assert np.array_equal(bits(wq.codes), wq_ref[0])
    ok, worst, where = gemm_close(c, c_ref, DT[dt])
    assert ok, f"worst err/bound {worst:.3g} at {where}"
    if fused and fmt == 0:
        assert np.float32(g_out.item()).tobytes() == np.float32(aq_ref[2]).tobytes()
    return c, c_ref


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("fused", [False, True])
def test_pr1_tiny_outliers(ops, orc, fmt, dt, fused):
    a, w = inputs.pr1_tiny()
    run_pair(ops, orc, a, w, fmt, dt, fused)


RAGGED = [(1, 8, 32), (16, 256, 64), (130, 264, 2880), (300, 520, 1056), (257, 512, 4096),
          (128, 256, 256), (129, 136, 96), (2304, 2312, 320), (600, 4104, 1056), (1024, 4096, 128),
          # few output tiles: narrow tiles and / or K split across a cluster
          (256, 2880, 2880), (64, 2880, 2880), (8, 720, 7680), (8, 256, 2048),
          (200, 1024, 6400), (200, 4864, 256), (8, 19200, 256), (256, 2880, 7680)]


# Launch classes fp4_gemm can take: (tile rows, tile columns, split along K);
# K is split only with 64- and 128-wide tiles
LAUNCH_CLASSES = {(256, 256, False), (128, 256, False), (128, 128, False), (128, 128, True),
                  (128, 64, False), (128, 64, True)}


def test_ragged_shapes_cover_every_launch_class(ops):
    for fmt in (0, 1):
        seen = set()
        for M, N, K in RAGGED:
            tm, tn, sp = ops.gemm_plan(M, N, K, fmt)
            seen.add((tm, tn, sp > 1))
        assert seen == LAUNCH_CLASSES, LAUNCH_CLASSES - seen


@pytest.mark.parametrize("M,N,K", RAGGED)
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_ragged_shapes(ops, orc, M, N, K, fmt, dt):
    a = inputs.random_bf16(100 + M, (M, K))
    w = inputs.random_bf16(200 + N, (N, K), 0.02)
    run_pair(ops, orc, a, w, fmt, dt)


@pytest.mark.parametrize("M,N,K", [(8, 720, 7680), (256, 2880, 7680), (200, 1024, 6400)])
@pytest.mark.parametrize("fmt", [0, 1])
def test_split_k_is_deterministic(ops, M, N, K, fmt):
    """K split over a cluster: the partial sums are added in split order, so
    repeated calls give identical bits."""
    assert ops.gemm_plan(M, N, K, fmt)[2] > 1
    a = inputs.random_bf16(300 + M, (M, K)).cuda()
    w = inputs.random_bf16(400 + N, (N, K), 0.02).cuda()
    aq = ops.quantize(a, fmt, ops.SCALES_MMA)
    wq = ops.quantize_weights(w, fmt)
    outs = [ops.gemm(aq, wq, torch.float32) for _ in range(4)]
    torch.cuda.synchronize()
    assert all(torch.equal(outs[0], o) for o in outs[1:])


@pytest.mark.parametrize("M,N,K,max_sms", [(256, 2880, 2880, 49), (256, 3840, 2880, 37),
                                           (256, 720, 7680, 37), (2048, 4096, 1024, 40)])
def test_sm_budget_changes_the_shape_not_the_result(ops, orc, M, N, K, max_sms):
    """max_sms picks a launch shape for a share of the device (the CTA-pair
    kernel keeps its tiles and runs fewer persistent pairs); the result
    stays within tolerance of the oracle (only the FP32 summation order may
    change)."""
    if ops.gemm_plan(M, N, K, 0)[0] == 128:
        assert ops.gemm_plan(M, N, K, 0, max_sms) != ops.gemm_plan(M, N, K, 0)
    a = inputs.random_bf16(500 + M, (M, K))
    w = inputs.random_bf16(600 + N, (N, K), 0.02)
    aq_ref, wq_ref = orc.quantize(a, 0), orc.quantize(w, 0)
    c_ref = orc.gemm(orc.dequant(aq_ref[0], aq_ref[1], 0, aq_ref[2]),
                     orc.dequant(wq_ref[0], wq_ref[1], 0, wq_ref[2]))
    aq = ops.quantize(a.cuda(), 0, ops.SCALES_MMA)
    wq = ops.quantize_weights(w.cuda(), 0)
    c = ops.gemm(aq, wq, torch.bfloat16, max_sms=max_sms)
    torch.cuda.synchronize()
    ok, worst, where = gemm_close(c, c_ref, torch.bfloat16)
    assert ok, f"worst err/bound {worst:.3g} at {where}"


@pytest.mark.parametrize("M", [1, 8, 32])
@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 4096), (4096, 14336)])
def test_decode_shapes_fused(ops, orc, M, N, K):
    a, w = inputs.decode(M, N, K)
    run_pair(ops, orc, a, w, 0, "bf16", fused=True)


# The prefill matrix: M in {2048, 8192} x (N, K) in {(8192, 8192), (28672,
# 8192)} x {bf16, fp32} in NVFP4, and MXFP4 at both M (bf16).  Cases of one
# shape are adjacent so that its inputs are generated once.
PREFILL = [(M, N, 8192, fmt, dt)
           for M in (2048, 8192) for N in (8192, 28672)
           for fmt, dt in ((0, "bf16"), (0, "f32"), (1, "bf16"))]
_prefill_cache = {}


def _prefill_inputs(M, N, K):
    if (M, N, K) not in _prefill_cache:
        _prefill_cache.clear()
        _prefill_cache[(M, N, K)] = inputs.prefill(M, N, K)
    return _prefill_cache[(M, N, K)]


@pytest.mark.parametrize("M,N,K,fmt,dt", PREFILL)
def test_prefill_full_size_sampled(ops, orc, M, N, K, fmt, dt):
    """Full-size launch; the oracle computes 128 sampled rows x 128 sampled
    columns (each row quantized with the tensor's own global scale)."""
    a, w = _prefill_inputs(M, N, K)
    wq = ops.quantize_weights(w.cuda(), fmt)
    aq = ops.quantize(a.cuda(), fmt, ops.SCALES_MMA)
    c = ops.gemm(aq, wq, DT[dt])
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    rng = np.random.default_rng(M + N)
    ri = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 126, replace=False)]))
    ci = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 126, replace=False)]))
    g_a = orc.global_scale(orc.amax(a)) if fmt == 0 else None
    g_w = orc.global_scale(orc.amax(w)) if fmt == 0 else None
    if fmt == 0:
        assert np.float32(aq.g.item()).tobytes() == np.float32(g_a).tobytes()
        assert np.float32(wq.g.item()).tobytes() == np.float32(g_w).tobytes()
    rt, ct = torch.from_numpy(ri), torch.from_numpy(ci)
    ca, sa, ga = orc.quantize(a[rt].contiguous(), fmt, g_a)
    cw, sw, gw = orc.quantize(w[ct].contiguous(), fmt, g_w)
    assert np.array_equal(bits(aq.codes[rt.cuda()]), ca)
    assert np.array_equal(bits(wq.codes[ct.cuda()]), cw)
    c_ref = orc.gemm(orc.dequant(ca, sa, fmt, ga), orc.dequant(cw, sw, fmt, gw))
    ok, worst, where = gemm_close(c[rt.cuda()][:, ct.cuda()], c_ref, DT[dt])
    assert ok, f"worst err/bound {worst:.3g} at {where}"
    del c, aq, wq


# M * K <= 128K values take the one-kernel path, larger activations the
# amax -> quantize -> GEMM chain (the last two shapes)
FUSED_RAGGED = [(1, 8, 32), (5, 264, 2880), (16, 520, 1056), (17, 136, 96), (32, 1024, 4096),
                (32, 14336, 256), (3, 4096, 8192), (24, 1032, 8192), (32, 520, 8192)]


@pytest.mark.parametrize("M,N,K", FUSED_RAGGED)
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_fused_ragged_shapes(ops, orc, M, N, K, fmt, dt):
    """Split-K and single-slice grids, padded activation rows, K tails."""
    a = inputs.random_bf16(300 + M, (M, K))
    w = inputs.random_bf16(400 + N, (N, K), 0.02)
    run_pair(ops, orc, a, w, fmt, dt, fused=True)


@pytest.mark.parametrize("g", [1.0, 0.01])
def test_fused_static_global_scale(ops, orc, g):
    M, N, K = 8, 512, 2048
    a = inputs.random_bf16(500, (M, K))
    w = inputs.random_bf16(501, (N, K), 0.02)
    ca, sa, ga = orc.quantize(a, 0, g)
    wq_ref = orc.quantize(w, 0)
    c_ref = orc.gemm(orc.dequant(ca, sa, 0, ga), orc.dequant(*wq_ref[:2], 0, wq_ref[2]))
    wq = ops.quantize_weights(w.cuda(), 0)
    c = ops.gemm_fused(a.cuda(), wq, torch.float32,
                       g_a=torch.tensor([g], dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    ok, worst, where = gemm_close(c, c_ref, torch.float32)
    assert ok, f"worst err/bound {worst:.3g} at {where}"


def test_fused_repeated_calls_are_deterministic(ops):
    """The split-K reduction runs in slice order: repeated calls give identical bits."""
    a, w = inputs.decode(32, 4096, 14336)
    wq = ops.quantize_weights(w.cuda(), 0)
    x = a.cuda()
    outs = [ops.gemm_fused(x, wq, torch.float32).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
