"""Pins for the oracle's MXFP4 macro-block scaling (reading R9: one binary32
second-level scale per row, applied by the GEMM's epilogue): the macro scale
is the significand of amax/6 (numpy's frexp, independently), a lone value
comes back within rounding, power-of-two row scalings only move the block
exponents, and the second level multiplies the plain MXFP4 dequantization.

"FP4 n'existe pas : il existe des FP4, et chaque runtime choisit son
dialecte", section "L'ecart de qualite -- et comment il se reduit" (macro
block scaling: a second-level scale over groups of 32-blocks, the base
format unchanged)."""
import numpy as np
import pytest

from mxfp4_block_scaled_fp4_b200 import inputs


def bf16(v):
    v = np.asarray(v, np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)


def test_sigma_is_the_significand_of_amax_over_6(orc):
    rng = np.random.default_rng(1)
    for a in np.concatenate([rng.lognormal(0, 6, 300), [6.0, 3.0, 1e-30, 3e30]]).astype(np.float32):
        t = np.float32(a) / np.float32(6.0)
        m, _ = np.frexp(np.float64(t))                 # t = m 2^e, m in [0.5, 1)
        assert orc.mbs_sigma(float(a)) == 2.0 * m
        assert 1.0 <= orc.mbs_sigma(float(a)) < 2.0
    assert orc.mbs_sigma(0.0) == 1.0


@pytest.mark.parametrize("rule", [0, 1])
def test_lone_value_comes_back(orc, rule):
    """A row holding one value A: its block's code is the top of E2M1 and
    sigma * 2^e * q is A within a few binary32 roundings."""
    rng = np.random.default_rng(2)
    for a in rng.lognormal(0, 5, 200).astype(np.float32):
        a = float((bf16([a]).astype(np.uint32) << 16).view(np.float32)[0])   # bf16-exact
        x = np.zeros((1, 64), np.float32)
        x[0, 37] = a
        c, s, sg = orc.quantize_mxfp4_mbs(bf16(x), rule)
        xh = orc.dequant(c, s, 1) * np.float64(sg[0])
        assert abs(xh[0, 37] - a) <= 2.0 ** -20 * a
        assert np.count_nonzero(xh) == 1


def test_power_of_two_row_scaling_moves_only_exponents(orc):
    x = orc.widen_bf16(inputs.act_sweep(8, 512)).reshape(8, 512)
    c0, s0, g0 = orc.quantize_mxfp4_mbs(bf16(x))
    for j in (-7, 3):
        c1, s1, g1 = orc.quantize_mxfp4_mbs(bf16(x * np.float32(2.0 ** j)))
        assert np.array_equal(c0, c1) and np.array_equal(g0, g1)
        assert np.array_equal(s1.astype(int) - s0.astype(int), np.full(s0.shape, j))


@pytest.mark.parametrize("rule", [0, 1])
def test_second_level_multiplies_the_mxfp4_dequantization(orc, rule):
    """x_hat = sigma * 2^e * q: the codes and E8M0 scales are plain MXFP4 of
    the row divided by (the reciprocal of) sigma."""
    x = inputs.act_sweep(16, 1024)
    c, s, sg = orc.quantize_mxfp4_mbs(x, rule)
    xf = orc.widen_bf16(x).reshape(16, 1024)
    rho = (np.float32(1.0) / sg.astype(np.float32))[:, None]
    c2, s2, _ = orc.quantize_f32((xf * rho).astype(np.float32), 1, rule=rule)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
    # values of at least half the row maximum land on |v| >= 1.5 of E2M1,
    # where a rounding step is at most a quarter of the value
    xh = orc.dequant(c, s, 1) * sg[:, None].astype(np.float64)
    big = np.abs(xf) >= np.abs(xf).max(axis=1, keepdims=True) / 2
    assert np.all(np.abs(xh - xf)[big] <= 0.25 * np.abs(xf)[big] + 1e-30)
