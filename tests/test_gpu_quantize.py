"""GPU quantizers against the oracle, bit for bit (codes, scales, global
scale), on the activation-quantize sweep shapes (M in {1, 32, 512, 8192},
K in {2880, 8192, 16384}, per-row lognormal scales), both formats, both
scale layouts, DYNAMIC and STATIC global scale, and crafted edge blocks."""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import inputs
from tests.parity import bits

pytestmark = pytest.mark.gpu

SWEEP = [(M, K) for M in (1, 32, 512, 8192) for K in (2880, 8192, 16384)]


@pytest.fixture(scope="module")
def ops():
    from mxfp4_block_scaled_fp4_b200 import ops as o
    return o


_cache = {}


def act(M, K):
    if (M, K) not in _cache:
        if len(_cache) > 3:
            _cache.clear()
        _cache[(M, K)] = inputs.act_sweep(M, K)
    return _cache[(M, K)]


def check_quant(ops, orc, x, fmt, g_static=None):
    xg = x.cuda()
    g_t = None if g_static is None else torch.tensor([g_static], dtype=torch.float32, device="cuda")
    q_rm = ops.quantize(xg, fmt, ops.SCALES_ROWMAJOR, g_t)
    q_mma = ops.quantize(xg, fmt, ops.SCALES_MMA, g_t)
    torch.cuda.synchronize()
    codes, scales, g = orc.quantize(x, fmt, g_static)
    assert np.array_equal(bits(q_rm.codes), codes)
    assert np.array_equal(bits(q_rm.scales).reshape(scales.shape), scales)
    assert np.array_equal(bits(q_mma.codes), codes)
    assert np.array_equal(bits(q_mma.scales), orc.scales_to_mma(scales))   # padding = 0 too
    if fmt == 0:
        assert np.float32(q_rm.g.item()).tobytes() == np.float32(g).tobytes()
        assert np.float32(q_mma.g.item()).tobytes() == np.float32(g).tobytes()


@pytest.mark.parametrize("M,K", SWEEP)
def test_nvfp4_dynamic_sweep(ops, orc, M, K):
    check_quant(ops, orc, act(M, K), 0)


@pytest.mark.parametrize("M,K", SWEEP)
def test_mxfp4_sweep(ops, orc, M, K):
    check_quant(ops, orc, act(M, K), 1)


# DYNAMIC tensors of at most 32 KiB skip the amax pass (each quantize CTA
# reads the whole tensor for its global scale); either side of that limit
@pytest.mark.parametrize("M,K", [(1, 16384), (1, 16416), (2, 8192), (2, 8224)])
def test_nvfp4_dynamic_self_amax_limit(ops, orc, M, K):
    check_quant(ops, orc, inputs.act_sweep(M, K), 0)


@pytest.mark.parametrize("M,K", [(32, 2880), (512, 8192)])
@pytest.mark.parametrize("g", [1.0, 0.0123])
def test_nvfp4_static_global_scale(ops, orc, M, K, g):
    check_quant(ops, orc, act(M, K), 0, g_static=g)


def crafted():
    """Rows of edge blocks: a 1000 outlier, the 3616 overflow, zeros and -0,
    bf16 subnormals, values on E2M1 tie points, huge values."""
    rows = []
    r = np.zeros(64, np.float32)
    r[3] = 1000.0
    r[:16][r[:16] == 0] = np.linspace(-39, 39, 15)
    rows.append(r)
    r = np.zeros(64, np.float32)
    r[0] = 3616.0
    r[1:16] = -1.0
    r[16:32] = -0.0
    r[32:48] = 1e-40                        # bf16 subnormal range
    r[48:64] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.75, -1.25, -1.75, -2.5,
                -3.5, -5.0, -6.0]
    rows.append(r)
    r = np.full(64, 3.0e38, np.float32)
    r[1::2] = -2.0e38
    rows.append(r)
    r = np.zeros(64, np.float32)
    rows.append(r)
    return inputs.to_bf16(np.stack(rows))


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("g", [None, 1.0])
def test_crafted_edge_blocks(ops, orc, fmt, g):
    if fmt == 1 and g is not None:
        pytest.skip("MXFP4 has no global scale")
    check_quant(ops, orc, crafted(), fmt, g)


def ladder(top=50):
    """One 16-value block per power of two from 2^-70 to 2^top (mantissas
    drawn at random, signs mixed), so the block maxima straddle both ends of
    the range in which the quantizer computes amax / (6 g) by Markstein's
    method rather than by a division."""
    g = np.random.default_rng(11)
    exps = np.arange(-70, top + 1)
    blocks = (g.uniform(1.0, 2.0, size=(exps.size, 16)) * np.exp2(exps)[:, None]
              * np.where(g.random((exps.size, 16)) < 0.5, -1.0, 1.0))
    flat = blocks.astype(np.float32).reshape(-1)
    K = 256
    flat = np.concatenate([flat, np.zeros((-flat.size) % K, np.float32)])
    return inputs.to_bf16(flat.reshape(-1, K))


@pytest.mark.parametrize("top", [50, 10])
@pytest.mark.parametrize("g", [None, 1e-20, 3.0e-4, 1.0, 1e20])
def test_scale_division_paths(ops, orc, top, g):
    check_quant(ops, orc, ladder(top), 0, g_static=g)


def test_zero_rows_is_a_noop(ops):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q = ops.quantize(x, 0, ops.SCALES_MMA)
    torch.cuda.synchronize()
    assert q.codes.numel() == 0


def test_quantize_weights_matches_act_path(ops, orc):
    w = inputs.random_bf16(9, (300, 1056), 0.02)
    wq = ops.quantize_weights(w.cuda(), 0)
    torch.cuda.synchronize()
    codes, scales, g = orc.quantize(w, 0)
    assert np.array_equal(bits(wq.codes), codes)
    assert np.array_equal(bits(wq.scales), orc.scales_to_mma(scales))
    assert np.float32(wq.g.item()).tobytes() == np.float32(g).tobytes()
