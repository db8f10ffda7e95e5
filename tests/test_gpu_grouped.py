"""Grouped (mixture-of-experts) W4A4 GEMM on the GPU against the oracle's
plain definition (each group's rows times its expert's weights, binary64 on
dequantized operands), within the stated tolerance: routed activations with
empty groups, one-row groups and groups that start on any row; experts
quantized one by one (bit-exact codes); both formats and output types;
offsets kept on the device, including malformed ones (clamped, never read
or written out of bounds).

"FP4 n'existe pas : il existe des FP4, et chaque runtime choisit son
dialecte", section "Les runtimes et leurs dialectes : qui parle quoi"
(fused NVFP4 MoE kernels; W4A4 MegaMoE)."""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import fp4lib as L
from mxfp4_block_scaled_fp4_b200 import inputs
from tests.parity import bits, gemm_close

pytestmark = pytest.mark.gpu
DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module")
def ops():
    from mxfp4_block_scaled_fp4_b200 import ops as o
    return o


def _sizes(seed, E, M):
    """Group sizes summing to M with some empty and some one-row groups."""
    rng = np.random.default_rng(seed)
    w = rng.dirichlet(np.full(E, 0.7))
    sizes = np.floor(w * M).astype(np.int64)
    sizes[0] += M - sizes.sum()
    if E >= 4:
        sizes[1], sizes[0] = 0, sizes[0] + sizes[1]     # an empty group
        if sizes[0] > 1:
            sizes[2] += 1
            sizes[0] -= 1
    return sizes


def _run(ops, orc, E, M, N, K, fmt, dt, seed=0, sizes=None):
    if sizes is None:
        sizes = _sizes(seed, E, M)
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    assert offs[-1] == M
    a = inputs.random_bf16(700 + seed, (M, K))
    w = inputs.random_bf16(701 + seed, (E * N, K), 0.02).view(E, N, K)
    aq = ops.quantize(a.cuda(), fmt, ops.SCALES_MMA)
    wq = ops.quantize_experts(w.cuda().contiguous(), fmt)
    c = ops.gemm_grouped(aq, wq, torch.from_numpy(offs).cuda(), DT[dt])
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    ca, sa, ga = orc.quantize(a, fmt)
    assert np.array_equal(bits(aq.codes), ca)
    w_hats = []
    for e in range(E):
        cw, sw, gw = orc.quantize(w[e].contiguous(), fmt)
        assert np.array_equal(bits(wq.codes[e]), cw)
        if fmt == 0:
            assert np.float32(wq.g[e].item()).tobytes() == np.float32(gw).tobytes()
        w_hats.append(orc.dequant(cw, sw, fmt, gw))
    ref = orc.gemm_grouped(orc.dequant(ca, sa, fmt, ga), w_hats, offs)
    ok, worst, where = gemm_close(c, ref, DT[dt])
    assert ok, f"worst err/bound {worst:.3g} at {where}"


@pytest.mark.parametrize("E,M,N,K", [(1, 300, 256, 256), (4, 513, 264, 2880), (8, 1000, 2048, 1024),
                                     (16, 2048, 1408, 2048), (64, 4096, 512, 768)])
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_grouped_matches_oracle(ops, orc, E, M, N, K, fmt, dt):
    _run(ops, orc, E, M, N, K, fmt, dt, seed=E + M)


# groups of many rows on average take the CTA-pair form (256 x 256 tiles)
@pytest.mark.parametrize("E,M,N,K", [(4, 4096, 2048, 1024), (8, 8192, 1536, 768)])
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_grouped_pair_form_matches_oracle(ops, orc, E, M, N, K, fmt, dt):
    _run(ops, orc, E, M, N, K, fmt, dt, seed=E + M + 1)


def test_groups_of_one_row_and_empty_tail(ops, orc):
    sizes = np.array([1, 0, 1, 129, 0, 127, 1, 0], np.int64)
    _run(ops, orc, 8, int(sizes.sum()), 384, 512, 0, "bf16", seed=5, sizes=sizes)


def test_max_groups(ops, orc):
    sizes = np.full(256, 3, np.int64)
    _run(ops, orc, 256, 768, 128, 256, 0, "f32", seed=6, sizes=sizes)


@pytest.mark.parametrize("fmt", [0, 1])
def test_max_groups_wide_tiles(ops, orc, fmt):
    """256 groups with N > 128: 128 x 256 tiles beside a full group table;
    groups of 1 to 9 rows, so most start inside a 128-row scale block."""
    sizes = (np.arange(256, dtype=np.int64) % 9) + 1
    _run(ops, orc, 256, int(sizes.sum()), 384, 512, fmt, "f32", seed=7, sizes=sizes)


def test_malformed_offsets_are_clamped(ops, orc):
    """Decreasing and out-of-range entries: the kernel clamps them into
    [0, M], keeps the groups disjoint and leaves every other row alone."""
    M, N, K, E = 300, 256, 512, 4
    a = inputs.random_bf16(710, (M, K)).cuda()
    w = inputs.random_bf16(711, (E * N, K), 0.02).view(E, N, K).cuda().contiguous()
    aq = ops.quantize(a, 0, ops.SCALES_MMA)
    wq = ops.quantize_experts(w, 0)
    offs = torch.tensor([-50, 100, 60, 250, 10_000], dtype=torch.int32, device="cuda")
    c = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    ops.gemm_grouped(aq, wq, offs, out=c)
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    # clamped groups: [0, 100), [100, 100), [100, 250), [250, 300)
    ref = torch.full((M, N), 7.0, dtype=torch.float32)
    for e, (lo, hi) in enumerate([(0, 100), (100, 100), (100, 250), (250, 300)]):
        if hi > lo:
            sub = ops.quantize(a[lo:hi].contiguous(), 0, ops.SCALES_MMA,
                               g=aq.g)   # same global scale as the whole tensor
            one = ops.Quantized(wq.codes[e], wq.scales[e], wq.g[e:e + 1], 0, ops.SCALES_MMA, N, K)
            ref[lo:hi] = ops.gemm(sub, one, torch.float32).cpu()
    torch.cuda.synchronize()
    got = c.cpu()
    assert torch.allclose(got, ref, rtol=1e-4, atol=1e-4 * float(ref.abs().max()))


def test_malformed_offsets_pair_form(ops, orc):
    """The same clamping on the CTA-pair form."""
    M, N, K, E = 4096, 1024, 512, 4
    a = inputs.random_bf16(720, (M, K)).cuda()
    w = inputs.random_bf16(721, (E * N, K), 0.02).view(E, N, K).cuda().contiguous()
    aq = ops.quantize(a, 0, ops.SCALES_MMA)
    wq = ops.quantize_experts(w, 0)
    offs = torch.tensor([-50, 1000, 900, 3000, 99_999], dtype=torch.int32, device="cuda")
    c = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    ops.gemm_grouped(aq, wq, offs, out=c)
    torch.cuda.synchronize()
    st, code = ops.device_status()
    assert st == 0 and code == 0
    ref = torch.full((M, N), 7.0, dtype=torch.float32)
    for e, (lo, hi) in enumerate([(0, 1000), (1000, 1000), (1000, 3000), (3000, 4096)]):
        if hi > lo:
            sub = ops.quantize(a[lo:hi].contiguous(), 0, ops.SCALES_MMA, g=aq.g)
            one = ops.Quantized(wq.codes[e], wq.scales[e], wq.g[e:e + 1], 0, ops.SCALES_MMA, N, K)
            ref[lo:hi] = ops.gemm(sub, one, torch.float32).cpu()
    got = c.cpu()
    assert torch.allclose(got, ref, rtol=1e-4, atol=1e-4 * float(ref.abs().max()))


def test_grouped_argument_checks(ops):
    fake = 1 << 20
    f = L.fp4_gemm_grouped
    assert f(fake, fake, fake, fake, fake, fake, fake, 0, 8, 16, 256, 0, fake, 16, 0, None, 0, 0,
             None) == L.FP4_ERR_INVALID_ARG                                   # E = 0
    assert f(fake, fake, fake, fake, fake, fake, fake, 257, 8, 16, 256, 0, fake, 16, 0, None, 0, 0,
             None) == L.FP4_ERR_INVALID_ARG                                   # E > 256
    assert f(fake, fake, fake, fake, fake, fake, None, 2, 8, 16, 256, 0, fake, 16, 0, None, 0, 0,
             None) == L.FP4_ERR_INVALID_ARG                                   # offsets NULL
    assert f(fake, fake, fake, fake, fake, fake, fake, 2, 8, 12, 256, 0, fake, 16, 0, None, 0, 0,
             None) == L.FP4_ERR_UNSUPPORTED_SHAPE                             # N % 8
