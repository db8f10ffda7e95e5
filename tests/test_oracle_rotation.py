"""Pins for the oracle's online rotation (R7), its binary32-input quantizers
and the overflow-aware MXFP4 scale rule (R8), against facts fixed outside
the oracle: the Sylvester Hadamard matrix of scipy, exact integer
arithmetic, the orthogonality H.H^T = n.I, brute-force exponent searches,
and the bf16 quantizers already pinned elsewhere.

Rotation: "FP4 on a consumer RTX 5090: the Blackwell headline loses to
plain int4", section "Finding 3 -- the real-FP4 path (QuTLASS MXFP4)"
(an online Hadamard rotation ahead of activation quantization).  OAS: "FP4
n'existe pas : il existe des FP4, et chaque runtime choisit son dialecte",
section "L'ecart de qualite -- et comment il se reduit" (the block scale is
chosen so that extreme values do not saturate)."""
import numpy as np
import pytest
import scipy.linalg

from mxfp4_block_scaled_fp4_b200 import inputs


def bf16(vals):
    """bf16 bit patterns of values that bf16 holds exactly (or of binary32
    bit patterns whose low half is zero)."""
    v = np.asarray(vals)
    if v.dtype != np.uint32:
        v = v.astype(np.float32).view(np.uint32)
    return (v >> 16).astype(np.uint16)


@pytest.mark.parametrize("n", [16, 32])
@pytest.mark.parametrize("shift", [0, 2, 3])
def test_basis_vectors_give_scipy_hadamard_columns(orc, n, shift):
    """Rotating e_j gives column j of the Sylvester Hadamard matrix (scipy),
    times 2^-shift: pins every butterfly's index and sign."""
    H = scipy.linalg.hadamard(n).astype(np.float64)
    K = 2 * n                       # two blocks: the second must stay zero
    x = np.zeros((n, K), np.float32)
    for j in range(n):
        x[j, n + j] = 1.0           # e_j in the second block
    y = orc.hadamard(bf16(x), n, shift).astype(np.float64)
    assert np.all(y[:, :n] == 0.0)
    assert np.array_equal(y[:, n:], H.T * 2.0 ** -shift)


@pytest.mark.parametrize("n", [16, 32])
def test_small_integers_are_exact(orc, n):
    """Integer inputs: every partial sum is exact in binary32, so the result
    equals the binary64 matrix product (H x) 2^-shift exactly."""
    rng = np.random.default_rng(5)
    x = rng.integers(-64, 65, size=(7, 4 * n)).astype(np.float32)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    for shift in (0, 1, 2, 3):
        y = orc.hadamard(bf16(x), n, shift).astype(np.float64)
        ref = np.concatenate([x[:, b * n:(b + 1) * n].astype(np.float64) @ H.T
                              for b in range(4)], axis=1) * 2.0 ** -shift
        assert np.array_equal(y, ref)


@pytest.mark.parametrize("n", [16, 32])
def test_twice_is_n_times_identity(orc, n):
    """H.H^T = n.I: rotating twice returns n x (integer inputs, exact)."""
    rng = np.random.default_rng(6)
    x = rng.integers(-16, 17, size=(3, 2 * n)).astype(np.float32)
    y = orc.hadamard(bf16(x), n, 0)
    assert np.all(np.abs(y) < 256)          # representable in bf16 exactly
    z = orc.hadamard(bf16(y), n, 0)
    assert np.array_equal(z, n * x)


@pytest.mark.parametrize("n", [16, 32])
def test_random_inputs_within_rounding_of_exact(orc, n):
    """bf16 values over a wide exponent range (so that binary32 sums do
    round): the transform is within log2(n) roundings of the exact binary64
    product (a dropped term or a wrong sign is far off)."""
    rng = np.random.default_rng(7)
    v = (rng.standard_normal((64, 8 * n)) * np.exp2(rng.integers(-30, 30, (64, 8 * n))))
    x = bf16(v.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000))
    xf = orc.widen_bf16(x).reshape(64, 8 * n).astype(np.float64)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    ref = np.concatenate([xf[:, b * n:(b + 1) * n] @ H.T for b in range(8)], axis=1)
    y = orc.hadamard(x, n, 0).astype(np.float64)
    tol = np.log2(n) * 2.0 ** -24 * np.abs(xf).reshape(64, 8, n).sum(-1).repeat(n, axis=1)
    assert np.all(np.abs(y - ref) <= tol)
    assert np.any(y != ref)                # the transform does round (binary32)


def test_rotated_product_equals_plain_product(orc):
    """The shifts of the two operands add up to log2(n): for exactly
    representable data the rotated GEMM equals the plain one."""
    rng = np.random.default_rng(8)
    for n in (16, 32):
        sa, sw = orc.rotation_shifts(n)
        assert sa + sw == int(np.log2(n))
        a = rng.integers(-4, 5, size=(5, 2 * n)).astype(np.float32)
        w = rng.integers(-4, 5, size=(6, 2 * n)).astype(np.float32)
        ra = orc.hadamard(bf16(a), n, sa).astype(np.float64)
        rw = orc.hadamard(bf16(w), n, sw).astype(np.float64)
        assert np.array_equal(ra @ rw.T, a.astype(np.float64) @ w.astype(np.float64).T)


def test_rotation_spreads_a_spike(orc):
    """A lone outlier in a block becomes n values of equal magnitude (the
    point of rotating before a block quantizer)."""
    for n in (16, 32):
        x = np.zeros((1, n), np.float32)
        x[0, 5] = 1024.0
        y = orc.hadamard(bf16(x), n, 2)
        assert np.all(np.abs(y) == 256.0)


@pytest.mark.parametrize("fmt", [0, 1])
def test_f32_quantizers_equal_bf16_quantizers_on_widened_inputs(orc, fmt):
    x = inputs.act_sweep(32, 2880)
    xf = orc.widen_bf16(x).reshape(32, 2880)
    for g in (None, 0.05) if fmt == 0 else (None,):
        c1, s1, g1 = orc.quantize(x, fmt, g)
        c2, s2, g2 = orc.quantize_f32(xf, fmt, g)
        assert np.array_equal(c1, c2) and np.array_equal(s1, s2) and g1 == g2


def test_rotated_dynamic_scale_uses_the_rotated_amax(orc):
    x = inputs.random_bf16(9, (8, 256))
    for n in (16, 32):
        sa, _ = orc.rotation_shifts(n)
        y = orc.hadamard(x, n, sa)
        _, _, g = orc.quantize_ex(x, 0, hadamard_n=n)
        assert np.float32(g) == np.float32(np.abs(y).max()) / np.float32(2688.0)


def _oas_exponent_brute(b):
    """The smallest integer e in [-127, 127] with b <= 6 * 2^e (exact)."""
    if b == 0:
        return -127
    for e in range(-127, 128):
        if b <= 6.0 * 2.0 ** e:
            return e
    return 127


def test_oas_exponent_is_the_smallest_non_clipping_one(orc):
    rng = np.random.default_rng(10)
    vals = np.concatenate([rng.lognormal(0, 4, 400), [6.0, 7.0, 7.5, 8.0, 12.0, 1e-30, 3e30],
                           [6.0 * 2.0 ** k for k in range(-20, 20)],
                           [np.nextafter(np.float32(6.0 * 2.0 ** k), np.float32(np.inf))
                            for k in range(-20, 20)]]).astype(np.float32)
    x = np.zeros((len(vals), 32), np.float32)
    x[:, 7] = vals
    _, s, _ = orc.quantize_f32(x, 1, rule=orc.OAS)
    for v, sc in zip(vals, s[:, 0]):
        assert int(sc) - 127 == _oas_exponent_brute(float(v)), v


def test_oas_never_clips_and_ocp_does(orc):
    """7 in a block: OCP (e = 0) clips it to 6, OAS (e = 1) codes it as 4 * 2
    = 8 (3.5 ties to the even code 4); any block: OAS keeps every |v| <= 6."""
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 7.0
    x[0, 1] = -1.0
    c_ocp, s_ocp, _ = orc.quantize_f32(x, 1, rule=orc.OCP)
    c_oas, s_oas, _ = orc.quantize_f32(x, 1, rule=orc.OAS)
    d_ocp = orc.dequant(c_ocp, s_ocp, 1)
    d_oas = orc.dequant(c_oas, s_oas, 1)
    assert d_ocp[0, 0] == 6.0 and d_oas[0, 0] == 8.0
    assert d_ocp[0, 1] == -1.0 and d_oas[0, 1] == -1.0      # -0.5 at scale 2
    xr = orc.widen_bf16(inputs.act_sweep(64, 2880)).reshape(64, 2880)
    c, s, _ = orc.quantize_f32(xr, 1, rule=orc.OAS)
    e = s.astype(np.int64) - 127
    v = np.abs(xr).reshape(64, -1, 32) / np.exp2(e)[..., None]
    assert np.all(v <= 6.0)
    # where the OCP rule would clip (block max in (6, 8) 2^e), OAS moved up by one
    c2, s2, _ = orc.quantize_f32(xr, 1, rule=orc.OCP)
    assert np.all((s - s2) >= 0) and np.all((s - s2) <= 1) and np.any(s != s2)
