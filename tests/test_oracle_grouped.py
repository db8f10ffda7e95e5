"""Pins for the oracle's grouped GEMM (its plain definition: each group's
rows times its expert's weights): against the naive triple loop of the C
oracle group by group, the dense GEMM when there is one group, and the
dense GEMM of a block-diagonal rewrite."""
import numpy as np


def test_one_group_is_the_dense_gemm(orc):
    rng = np.random.default_rng(1)
    a, w = rng.standard_normal((9, 64)), rng.standard_normal((5, 64))
    assert np.array_equal(orc.gemm_grouped(a, [w], [0, 9]), orc.gemm(a, w))


def test_groups_against_the_naive_loop(orc):
    rng = np.random.default_rng(2)
    offs = [0, 3, 3, 10, 11, 16]                 # one empty group
    a = rng.integers(-3, 4, (16, 32)).astype(np.float64)
    ws = [rng.integers(-3, 4, (6, 32)).astype(np.float64) for _ in range(5)]
    c = orc.gemm_grouped(a, ws, offs)
    for e in range(5):
        lo, hi = offs[e], offs[e + 1]
        if hi > lo:
            assert np.array_equal(c[lo:hi], orc.gemm_naive(a[lo:hi], ws[e]))


def test_block_diagonal_rewrite(orc):
    """Group e's product equals the dense product of A with the e-th slot of
    the stacked weights, read off the matching block."""
    rng = np.random.default_rng(3)
    offs = [0, 4, 9, 12]
    a = rng.integers(-2, 3, (12, 16)).astype(np.float64)
    ws = [rng.integers(-2, 3, (7, 16)).astype(np.float64) for _ in range(3)]
    full = orc.gemm(a, np.concatenate(ws))        # [12, 21]
    c = orc.gemm_grouped(a, ws, offs)
    for e in range(3):
        assert np.array_equal(c[offs[e]:offs[e + 1]], full[offs[e]:offs[e + 1], 7 * e:7 * e + 7])
