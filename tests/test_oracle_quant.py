"""Pins for the oracle's NVFP4 / MXFP4 quantizers, dequant, GEMM and the
MMA-consumable scale order (CPU only).

The pinned facts come from "Hardware FP4 inference for speech on
Blackwell" (section "NVFP4, and the two ways it fails": x_hat = s*q with
s = E4M3(max|x|/6); one 1000 outlier zeroes the other fifteen values of its
block; the smallest nonzero magnitude is max|x|/12 and anything below
max|x|/24 becomes zero; a block max above 6*448 = 2688 overflows E4M3 and a
per-tensor FP32 scale with saturation handles it; section "Activations are
where it breaks": |3616| gives a block scale 3616/6 = 603 > 448) and from
"FP4 n'existe pas : il existe des FP4, et chaque runtime choisit son
dialecte" (format table: 16 vs 32 values per block, E4M3 vs E8M0 scales,
~4.5 vs ~4.25 bits per value).
"""
import numpy as np
import pytest
import torch

from mxfp4_block_scaled_fp4_b200 import inputs
from tests.golden import load as golden

NV, MX = 0, 1
FACTS = golden.format_facts()


def bf16(vals, shape=None):
    t = torch.tensor(np.asarray(vals, np.float32)).to(torch.bfloat16)
    return t.reshape(shape) if shape else t


def unpack(codes: np.ndarray) -> np.ndarray:
    lo = codes & 15
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


# ------------------------------------------------------------ NVFP4 pins --

def _outlier_block():
    g = np.random.default_rng(5)
    x = g.uniform(-39.0, 39.0, 16).astype(np.float32)
    x[3] = FACTS["outlier"]
    return bf16(x, (1, 16))


def test_outlier_zeroes_its_neighbours_static_g1(orc):
    """g = 1: s = E4M3(1000/6 = 166.7) = 160, 1000/160 = 6.25 clips to 6."""
    x = _outlier_block()
    codes, scales, g = orc.quantize_nvfp4(x, g=1.0)
    q = unpack(codes)[0]
    assert orc.e4m3_decode(scales[0, 0]) == 160.0
    assert q[3] == 7                                     # +6
    assert all((q[i] & 7) == 0 for i in range(16) if i != 3)
    xh = orc.dequant(codes, scales, NV, g)[0]
    assert xh[3] == 960.0
    assert np.count_nonzero(xh) == 1


def test_outlier_zeroes_its_neighbours_dynamic(orc):
    """Dynamic g = 1000/2688: the block scale lands on 448, 1000 -> ~1000."""
    x = _outlier_block()
    codes, scales, g = orc.quantize_nvfp4(x)
    assert g == np.float32(np.float32(1000.0) / np.float32(2688.0))
    assert scales[0, 0] == 0x7E
    q = unpack(codes)[0]
    assert all((q[i] & 7) == 0 for i in range(16) if i != 3)
    xh = orc.dequant(codes, scales, NV, g)[0]
    assert abs(xh[3] - 1000.0) <= 1000.0 * 2.0 ** -22
    assert np.count_nonzero(xh) == 1


@pytest.mark.parametrize("k", [-3, 0, 2, 5])
def test_amax_over_24_rounds_to_zero_and_amax_over_12_is_smallest(orc, k):
    """amax = 6*2^k, g = 1: s = 2^k exactly; x <= amax/24 -> 0, just above -> amax/12."""
    amax = 6.0 * 2.0 ** k
    lo = amax / FACTS["zero_below_div"]
    above = float(np.nextafter(np.float32(lo), np.float32(1e9)))
    vals = [amax, lo, -lo, above, -above, lo * 0.5] + [0.0] * 10
    x = bf16(vals, (1, 16))
    xv = x.float().numpy()[0]
    codes, scales, g = orc.quantize_nvfp4(x, g=1.0)
    xh = orc.dequant(codes, scales, NV, g)[0]
    assert xh[0] == amax
    assert xh[1] == 0.0 and xh[2] == 0.0 and xh[5] == 0.0    # tie at amax/24 -> 0
    if xv[3] > lo:                                           # bf16 kept it above
        assert xh[3] == amax / FACTS["smallest_nonzero_div"]
        assert xh[4] == -amax / FACTS["smallest_nonzero_div"]
    # invariant: |v| <= 0.25 <=> code in {0x0, 0x8}
    q = unpack(codes)[0]
    v = np.abs(xv) / (orc.e4m3_decode(scales[0, 0]) * g)
    assert np.array_equal((q & 7) == 0, v <= 0.25)


def test_scale_saturates_at_2688_without_global_scale(orc):
    """Block max 3616 (the page's activation): 3616/6 = 603 > 448 -> s = 448,
    3616/448 = 8.07 -> code 6 -> x_hat = 2688, and never NaN."""
    a = FACTS["worked_activation"]
    assert round(a / 6) == FACTS["worked_scale"] and a / 6 > FACTS["e4m3_max"]
    x = bf16([a, -a / 2, 1.0] + [0.5] * 13, (1, 16))
    codes, scales, g = orc.quantize_nvfp4(x, g=1.0)
    assert scales[0, 0] == 0x7E
    xh = orc.dequant(codes, scales, NV, g)[0]
    assert xh[0] == FACTS["scale_overflow_amax"] == 6 * FACTS["e4m3_max"]
    assert np.all(np.isfinite(xh))
    for big in [2688.0, 3000.0, 1e5, 3e38]:
        x2 = bf16([big] + [1.0] * 15, (1, 16))
        c2, s2, _ = orc.quantize_nvfp4(x2, g=1.0)
        assert orc.dequant(c2, s2, NV, 1.0)[0, 0] == 2688.0


def test_dynamic_global_scale_keeps_3616(orc):
    a = FACTS["worked_activation"]
    x = bf16([a] + [1.0] * 15, (1, 16))
    codes, scales, g = orc.quantize_nvfp4(x)
    assert scales[0, 0] == 0x7E
    xh = orc.dequant(codes, scales, NV, g)[0]
    assert abs(xh[0] - a) <= a * 2.0 ** -21


def test_all_zero_tensor(orc):
    x = bf16([0.0] * 64, (2, 32))
    codes, scales, g = orc.quantize_nvfp4(x)
    assert g == 1.0 and not codes.any() and not scales.any()
    c2, s2 = orc.quantize_mxfp4(x)
    assert not c2.any() and np.all(s2 == 0)               # e = -127 -> byte 0


def _roundtrip_blocks(rng, fmt, nblk):
    """Blocks x = s*q built from random codes: quantizing must give them back."""
    pts = golden.e2m1_codepoints()
    bs = 16 if fmt == NV else 32
    q = rng.integers(0, 16, size=(nblk, bs))
    top = rng.integers(0, bs, size=nblk)
    if fmt == NV:
        q[np.arange(nblk), top] = np.where(rng.integers(0, 2, nblk) == 0, 7, 15)   # +-6
        s_codes = rng.integers(0x08, 0x7F, size=nblk)   # normal E4M3 scales
    else:
        q[np.arange(nblk), top] = rng.choice([6, 7, 14, 15], size=nblk)            # +-4 or +-6
        s_codes = rng.integers(100, 150, size=nblk)     # E8M0
    mag = np.array(pts)[q & 7] * np.where(q >= 8, -1.0, 1.0)
    return q, s_codes, mag


def test_nvfp4_roundtrip_identity(orc):
    rng = np.random.default_rng(11)
    q, s, mag = _roundtrip_blocks(rng, NV, 512)
    sv = np.array([orc.e4m3_decode(int(c)) for c in s])
    x = bf16((mag * sv[:, None]).reshape(32, 256))
    assert np.array_equal(x.float().numpy().reshape(512, 16), mag * sv[:, None])  # exact in bf16
    codes, scales, _ = orc.quantize_nvfp4(x, g=1.0)
    got_q = unpack(codes).reshape(512, 16)
    # +0 and -0 both decode to 0; compare values and the scale bytes
    assert np.array_equal(np.array(golden.e2m1_codepoints())[got_q & 7], np.abs(mag))
    assert np.array_equal(scales.reshape(-1), s)


def test_mxfp4_roundtrip_identity(orc):
    rng = np.random.default_rng(12)
    q, s, mag = _roundtrip_blocks(rng, MX, 256)
    sv = 2.0 ** (s.astype(np.float64) - 127)
    x = bf16((mag * sv[:, None]).reshape(32, 256))
    codes, scales = orc.quantize_mxfp4(x)
    got_q = unpack(codes).reshape(256, 32)
    assert np.array_equal(np.array(golden.e2m1_codepoints())[got_q & 7], np.abs(mag))
    assert np.array_equal(scales.reshape(-1), s)


def test_mxfp4_exponent_rule(orc):
    """e = floor(log2 amax) - 2: amax 3 -> e = -1 (byte 126), 3*2 = 6 -> code 7;
    amax 7.5 -> e = 0, 7.5 saturates to 6."""
    x = bf16([3.0, 1.0] + [0.0] * 30, (1, 32))
    c, s = orc.quantize_mxfp4(x)
    assert s[0, 0] == 126 and (c[0, 0] & 15) == 7 and (c[0, 0] >> 4) == 4   # 1*2 = 2
    x = bf16([7.5, -5.0] + [0.0] * 30, (1, 32))
    c, s = orc.quantize_mxfp4(x)
    assert s[0, 0] == 127 and (c[0, 0] & 15) == 7 and (c[0, 0] >> 4) == 8 | 6   # -5 -> -4 (tie to even)


def test_bits_per_value(orc):
    K = 4096
    for fmt, key in [(NV, "nvfp4_bits_per_value"), (MX, "mxfp4_bits_per_value")]:
        x = inputs.random_bf16(1, (4, K))
        codes, scales, _ = orc.quantize(x, fmt)
        bits = 8.0 * (codes.nbytes + scales.nbytes) / x.numel()
        assert bits == FACTS[key]
    assert FACTS["nvfp4_block"] == 16 and FACTS["mxfp4_block"] == 32


def test_codes_match_exact_real_rounding_when_scale_is_power_of_two(orc):
    """If s*g is a power of two the reciprocal is exact, so the code is the
    E2M1 rounding of the exact real x/(s*g)."""
    x = inputs.random_bf16(21, (64, 256))
    codes, scales, g = orc.quantize_nvfp4(x, g=1.0)
    q = unpack(codes)
    sv = orc.e4m3_decode_array(scales)
    pow2 = np.log2(sv) == np.round(np.log2(sv))
    xv = x.float().numpy().astype(np.float64)
    exact = orc.e2m1_encode_array((xv / np.repeat(sv, 16, axis=1)).reshape(-1)).reshape(q.shape)
    mask = np.repeat(pow2, 16, axis=1)
    assert mask.sum() > 100
    assert np.array_equal(q[mask], exact[mask])


# ---------------------------------------------------------------- dequant --

def test_dequant_is_g_times_s_times_q(orc):
    codes = np.array([[0x71, 0xF8]], np.uint8)   # elements: 0.5, 6, -0, -6
    scales = np.array([[0x70]], np.uint8)        # E4M3 0x70 = 2^7 = 128
    out = orc.dequant(np.pad(codes, ((0, 0), (0, 6))), scales, NV, 0.25)[0]
    assert list(out[:4]) == [0.5 * 128 * 0.25, 6 * 128 * 0.25, 0.0, -6 * 128 * 0.25]
    mx_scales = np.array([[130]], np.uint8)      # 2^3
    out = orc.dequant(np.pad(codes, ((0, 0), (0, 14))), mx_scales, MX)[0]
    assert list(out[:4]) == [4.0, 48.0, 0.0, -48.0]


# ------------------------------------------------------------------- GEMM --

def test_gemm_naive_equals_library_matmul(orc):
    rng = np.random.default_rng(3)
    a = rng.standard_normal((7, 64))
    w = rng.standard_normal((9, 64))
    c1 = orc.gemm_naive(a, w)
    c2 = orc.gemm(a, w)
    assert np.allclose(c1, c2, rtol=1e-13, atol=1e-13)
    assert np.allclose(orc.gemm(w, a), c2.T, rtol=1e-13, atol=1e-13)   # swap -> transpose


def test_gemm_closed_form(orc):
    """Operands built from exact code points with exact scales, so C is known.

    A row m is the E2M1 pattern p (block max 6, scale 1) and W row n is the
    constant 6 * 2^(n-2) (scale 2^(n-2), code 6): C[m, n] = 6 * 2^(n-2) * sum(p)."""
    M, N, K = 3, 5, 64
    pts = golden.e2m1_codepoints()
    p = np.array([6, -4, 3, 2, -1.5, 1, 0.5, 0, -6, 4, -3, 2, 1.5, -1, 0, 0.5] * (K // 16))
    a = bf16(np.repeat(p[None, :], M, axis=0))
    w = bf16(np.repeat((6.0 * 2.0 ** (np.arange(N) - 2.0))[:, None], K, axis=1))
    want = np.repeat((6.0 * 2.0 ** (np.arange(N) - 2.0) * p.sum())[None, :], M, axis=0)
    assert set(np.abs(p)) <= set(pts)
    for fmt, kw in [(NV, dict(g_a=1.0, g_w=1.0)), (MX, {})]:
        c, _ = orc.w4a4_reference(a, w, fmt, **kw)
        assert np.array_equal(c, want)


def test_pr1_oracle_properties(orc):
    a, w = inputs.pr1_tiny()
    for fmt in (NV, MX):
        c_ref, q = orc.w4a4_reference(a, w, fmt)
        c_naive = orc.gemm_naive(orc.dequant(q["a_codes"], q["a_scales"], fmt, q["g_a"]),
                                 orc.dequant(q["w_codes"], q["w_scales"], fmt, q["g_w"]))
        assert np.allclose(c_ref, c_naive, rtol=1e-12, atol=1e-9)
        assert np.all(np.isfinite(c_ref))
    # every NVFP4 block that holds a 1000 outlier keeps only values near it
    codes, scales, g = orc.quantize_nvfp4(a)
    xh = orc.dequant(codes, scales, NV, g).reshape(-1, 16)
    blocks = a.float().numpy().reshape(-1, 16)
    has = np.abs(blocks).max(axis=1) == 1000.0
    assert has.sum() > 30
    small = (np.abs(blocks) < 1000.0 / 24) & has[:, None]
    assert np.all(xh[small] == 0.0)


# -------------------------------------------------------- MMA scale order --

def test_mma_scale_offsets(orc):
    L = orc.lib()
    nsf = 180                       # K = 2880, NVFP4: 45 atoms of 4 columns
    assert L.orc_mma_scale_offset(0, 0, nsf) == 0
    assert L.orc_mma_scale_offset(0, 1, nsf) == 1
    assert L.orc_mma_scale_offset(1, 0, nsf) == 16
    assert L.orc_mma_scale_offset(32, 0, nsf) == 4
    assert L.orc_mma_scale_offset(127, 3, nsf) == 31 * 16 + 3 * 4 + 3
    assert L.orc_mma_scale_offset(0, 4, nsf) == 512
    assert L.orc_mma_scale_offset(128, 0, nsf) == 45 * 512
    assert orc.mma_scale_bytes(1, 90) == 23 * 512       # MXFP4 K = 2880


def test_mma_scale_roundtrip_and_zero_padding(orc):
    rng = np.random.default_rng(4)
    for rows, nsf in [(1, 4), (16, 16), (130, 90), (256, 180)]:
        s = rng.integers(1, 255, size=(rows, nsf)).astype(np.uint8)
        m = orc.scales_to_mma(s)
        assert m.size == ((rows + 127) // 128) * ((nsf + 3) // 4) * 512
        assert np.array_equal(orc.scales_from_mma(m, rows, nsf), s)
        assert np.count_nonzero(m) == rows * nsf           # padding bytes are 0
