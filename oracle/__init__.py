"""CPU oracle for W4A4 block-scaled FP4 (NVFP4 / MXFP4).

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference``) may import
this package.  The product library never calls it and shares no code with it.

The arithmetic lives in ``fp4_oracle.c`` (plain C, one correctly rounded
binary32 operation per step, see the readings R1-R8 in its header: R7 is
the online Walsh-Hadamard rotation, R8 the overflow-aware MXFP4 scale
rule).  This
module marshals numpy arrays and adds the GEMM on dequantized values in
binary64, which is the plain definition C = A_hat . W_hat^T.

Sources: "Hardware FP4 inference for speech on Blackwell", section "NVFP4,
and the two ways it fails" (format, scale rule, saturation); "FP4 n'existe
pas : il existe des FP4, et chaque runtime choisit son dialecte", section
"Deux dialectes, deux strategies de scaling" (MXFP4 = OCP MX: 32-blocks,
E8M0 scales) and section "L'ecart de qualite -- et comment il se reduit"
(OAS); "FP4 on a consumer RTX 5090: the Blackwell headline loses to plain
int4", section "Finding 3 -- the real-FP4 path (QuTLASS MXFP4)" (online
Hadamard rotation ahead of the activation quantizer).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

NVFP4 = 0
MXFP4 = 1
BLOCK = {NVFP4: 16, MXFP4: 32}

_lib = None


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the oracle's shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


def _declare(L):
    P = ctypes.c_void_p
    i64 = ctypes.c_long
    L.orc_e2m1_decode.restype = ctypes.c_double
    L.orc_e2m1_decode.argtypes = [ctypes.c_uint]
    L.orc_e2m1_encode.restype = ctypes.c_uint
    L.orc_e2m1_encode.argtypes = [ctypes.c_double]
    L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint]
    L.orc_e4m3_encode_satfinite.restype = ctypes.c_uint
    L.orc_e4m3_encode_satfinite.argtypes = [ctypes.c_float]
    L.orc_e8m0_decode.restype = ctypes.c_double
    L.orc_e8m0_decode.argtypes = [ctypes.c_uint]
    L.orc_amax_bf16.restype = ctypes.c_float
    L.orc_amax_bf16.argtypes = [P, i64]
    L.orc_nvfp4_global_scale.restype = ctypes.c_float
    L.orc_nvfp4_global_scale.argtypes = [ctypes.c_float]
    L.orc_nvfp4_quantize.restype = ctypes.c_int
    L.orc_nvfp4_quantize.argtypes = [P, i64, i64, ctypes.c_int, P, P, P]
    L.orc_mxfp4_quantize.restype = ctypes.c_int
    L.orc_mxfp4_quantize.argtypes = [P, i64, i64, P, P]
    L.orc_dequant.restype = ctypes.c_int
    L.orc_dequant.argtypes = [P, P, i64, i64, ctypes.c_int, ctypes.c_float, P]
    L.orc_gemm_naive.restype = None
    L.orc_gemm_naive.argtypes = [P, P, i64, i64, i64, P]
    L.orc_mma_scale_bytes.restype = i64
    L.orc_mma_scale_bytes.argtypes = [i64, i64]
    L.orc_mma_scale_offset.restype = i64
    L.orc_mma_scale_offset.argtypes = [i64, i64, i64]
    L.orc_scales_to_mma.restype = None
    L.orc_scales_to_mma.argtypes = [P, i64, i64, P]
    L.orc_scales_from_mma.restype = None
    L.orc_scales_from_mma.argtypes = [P, i64, i64, P]
    L.orc_amax_f32.restype = ctypes.c_float
    L.orc_amax_f32.argtypes = [P, i64]
    L.orc_nvfp4_quantize_f32.restype = ctypes.c_int
    L.orc_nvfp4_quantize_f32.argtypes = [P, i64, i64, ctypes.c_int, P, P, P]
    L.orc_mxfp4_quantize_f32.restype = ctypes.c_int
    L.orc_mxfp4_quantize_f32.argtypes = [P, i64, i64, ctypes.c_int, P, P]
    L.orc_hadamard_f32.restype = ctypes.c_int
    L.orc_hadamard_f32.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, P]
    L.orc_mbs_sigma.restype = ctypes.c_float
    L.orc_mbs_sigma.argtypes = [ctypes.c_float]
    L.orc_mxfp4_mbs_quantize.restype = ctypes.c_int
    L.orc_mxfp4_mbs_quantize.argtypes = [P, i64, i64, ctypes.c_int, P, P, P]
    L.orc_e2m1_encode_array.restype = None
    L.orc_e2m1_encode_array.argtypes = [P, i64, P]
    L.orc_e4m3_encode_array.restype = None
    L.orc_e4m3_encode_array.argtypes = [P, i64, P]


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _as_bf16_bits(x) -> np.ndarray:
    """Accept a uint16 array of bf16 bit patterns or a torch bf16 tensor."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch  # local: the oracle itself does not need torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return x


# ----------------------------------------------------------------- codecs --

def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(v)


def e2m1_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode_satfinite(v)


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e8m0_decode(code: int) -> float:
    return lib().orc_e8m0_decode(code)


def e2m1_decode_array(codes: np.ndarray) -> np.ndarray:
    table = np.array([e2m1_decode(c) for c in range(16)], np.float64)
    return table[codes]


def e4m3_decode_array(codes: np.ndarray) -> np.ndarray:
    table = np.array([e4m3_decode(c) for c in range(256)], np.float64)
    return table[codes]


# ------------------------------------------------------------- quantizers --

def amax(x) -> float:
    x = _as_bf16_bits(x)
    return float(lib().orc_amax_bf16(_ptr(x), x.size))


def global_scale(amax_value: float) -> float:
    return float(lib().orc_nvfp4_global_scale(amax_value))


def quantize_nvfp4(x, g: float | None = None):
    """NVFP4-quantize a bf16 [rows, K] tensor.

    g=None: DYNAMIC global scale from the tensor amax; otherwise STATIC g.
    Returns (codes [rows, K/2] u8, scales [rows, K/16] u8 row-major, g).
    """
    x = _as_bf16_bits(x)
    rows, K = x.shape
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 16), np.uint8)
    gbuf = np.array([1.0 if g is None else g], np.float32)
    rc = lib().orc_nvfp4_quantize(_ptr(x), rows, K, int(g is None),
                                  _ptr(gbuf), _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError(f"bad shape for NVFP4: {x.shape}")
    return codes, scales, float(gbuf[0])


def quantize_mxfp4(x):
    """MXFP4-quantize a bf16 [rows, K] tensor.

    Returns (codes [rows, K/2] u8, scales [rows, K/32] u8 row-major).
    """
    x = _as_bf16_bits(x)
    rows, K = x.shape
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    rc = lib().orc_mxfp4_quantize(_ptr(x), rows, K, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError(f"bad shape for MXFP4: {x.shape}")
    return codes, scales


def quantize(x, fmt: int, g: float | None = None):
    """Uniform form: returns (codes, row-major scales, g); g = 1 for MXFP4."""
    if fmt == NVFP4:
        return quantize_nvfp4(x, g)
    c, s = quantize_mxfp4(x)
    return c, s, 1.0


# ------------------------------------- binary32 inputs, rotation, OAS (R7, R8) --

OCP = 0     # MXFP4 scale rule R5: e = floor(log2 amax) - 2
OAS = 1     # MXFP4 scale rule R8: the smallest e with amax <= 6 * 2^e


def widen_bf16(x) -> np.ndarray:
    """bf16 bit patterns -> binary32 values (exact: bf16 is the top half)."""
    x = _as_bf16_bits(x)
    return (x.astype(np.uint32) << 16).view(np.float32)


def rotation_shifts(n: int) -> tuple[int, int]:
    """(activation shift, weight shift) of R7: they add up to log2(n), so the
    product of a rotated activation and a rotated weight equals the plain
    product."""
    lg = int(n).bit_length() - 1
    return (lg + 1) // 2, lg // 2


def hadamard(x, n: int, shift: int) -> np.ndarray:
    """R7: every n-value block of every row rotated by the order-n
    Walsh-Hadamard matrix in binary32 (fast transform), times 2^-shift."""
    x = _as_bf16_bits(x)
    rows, K = x.shape
    out = np.empty((rows, K), np.float32)
    rc = lib().orc_hadamard_f32(_ptr(x), rows, K, int(n), int(shift), _ptr(out))
    if rc != 0:
        raise ValueError(f"bad rotation arguments: shape {x.shape}, n={n}, shift={shift}")
    return out


def amax_f32(x: np.ndarray) -> float:
    x = np.ascontiguousarray(x, np.float32)
    return float(lib().orc_amax_f32(_ptr(x), x.size))


def quantize_f32(x: np.ndarray, fmt: int, g: float | None = None, rule: int = OCP):
    """Quantize binary32 values [rows, K] (R1-R5 on binary32 inputs; MXFP4
    with scale rule `rule`).  Returns (codes, row-major scales, g)."""
    x = np.ascontiguousarray(x, np.float32)
    rows, K = x.shape
    codes = np.empty((rows, K // 2), np.uint8)
    if fmt == NVFP4:
        scales = np.empty((rows, K // 16), np.uint8)
        gbuf = np.array([1.0 if g is None else g], np.float32)
        rc = lib().orc_nvfp4_quantize_f32(_ptr(x), rows, K, int(g is None), _ptr(gbuf),
                                          _ptr(codes), _ptr(scales))
        gv = float(gbuf[0])
    else:
        scales = np.empty((rows, K // 32), np.uint8)
        rc = lib().orc_mxfp4_quantize_f32(_ptr(x), rows, K, int(rule), _ptr(codes),
                                          _ptr(scales))
        gv = 1.0
    if rc != 0:
        raise ValueError(f"bad shape or rule: {x.shape}, rule {rule}")
    return codes, scales, gv


def quantize_ex(x, fmt: int, g: float | None = None, hadamard_n: int = 0,
                operand: str = "act", rule: int = OCP):
    """The quantizer with its options: an online rotation of order
    hadamard_n (0 = none; the operand's R7 shift) and, for MXFP4, the scale
    rule.  Without options it is ``quantize``."""
    if hadamard_n:
        sa, sw = rotation_shifts(hadamard_n)
        xf = hadamard(x, hadamard_n, sa if operand == "act" else sw)
    elif fmt == MXFP4 and rule != OCP:
        xf = widen_bf16(x).reshape(np.shape(x))
    else:
        return quantize(x, fmt, g)
    return quantize_f32(xf, fmt, g, rule)


def mbs_sigma(amax_row: float) -> float:
    """R9: the macro scale of a row whose largest magnitude is amax_row."""
    return float(lib().orc_mbs_sigma(amax_row))


def quantize_mxfp4_mbs(x, rule: int = OCP):
    """R9: MXFP4 with one binary32 macro scale per row.  Returns (codes,
    row-major E8M0 scales, sigma [rows] float32)."""
    x = _as_bf16_bits(x)
    rows, K = x.shape
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    sigma = np.empty(rows, np.float32)
    rc = lib().orc_mxfp4_mbs_quantize(_ptr(x), rows, K, int(rule), _ptr(sigma), _ptr(codes),
                                      _ptr(scales))
    if rc != 0:
        raise ValueError(f"bad shape or rule: {x.shape}, rule {rule}")
    return codes, scales, sigma


def dequant(codes: np.ndarray, scales: np.ndarray, fmt: int, g: float = 1.0):
    """x_hat = g * s * q in binary64 ([rows, K])."""
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows = codes.shape[0]
    K = codes.shape[1] * 2
    out = np.empty((rows, K), np.float64)
    rc = lib().orc_dequant(_ptr(codes), _ptr(scales), rows, K, fmt,
                           float(g), _ptr(out))
    if rc != 0:
        raise ValueError("bad shape")
    return out


# ------------------------------------------------------------------- GEMM --

def gemm_naive(a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """C = A_hat . W_hat^T by the plain triple loop (binary64)."""
    a = np.ascontiguousarray(a_hat, np.float64)
    w = np.ascontiguousarray(w_hat, np.float64)
    M, K = a.shape
    N = w.shape[0]
    c = np.empty((M, N), np.float64)
    lib().orc_gemm_naive(_ptr(a), _ptr(w), M, N, K, _ptr(c))
    return c


def gemm(a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """C = A_hat . W_hat^T in binary64 with the library matmul."""
    return np.asarray(a_hat, np.float64) @ np.asarray(w_hat, np.float64).T


def gemm_grouped(a_hat: np.ndarray, w_hats, offsets) -> np.ndarray:
    """Grouped GEMM by its plain definition: rows [offsets[e], offsets[e+1])
    of A_hat times expert e's W_hat^T (binary64, the library matmul per
    group); rows outside every group stay 0."""
    a = np.asarray(a_hat, np.float64)
    N = np.asarray(w_hats[0]).shape[0]
    c = np.zeros((a.shape[0], N), np.float64)
    for e, w in enumerate(w_hats):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            c[lo:hi] = a[lo:hi] @ np.asarray(w, np.float64).T
    return c


def w4a4_reference(a_bf16, w_bf16, fmt: int, g_a: float | None = None,
                   g_w: float | None = None):
    """Quantize both operands by the definition, then C = A_hat . W_hat^T.

    Returns (C_ref float64 [M, N], dict of the quantized operands)."""
    ca, sa, ga = quantize(a_bf16, fmt, g_a)
    cw, sw, gw = quantize(w_bf16, fmt, g_w)
    a_hat = dequant(ca, sa, fmt, ga)
    w_hat = dequant(cw, sw, fmt, gw)
    return gemm(a_hat, w_hat), dict(a_codes=ca, a_scales=sa, g_a=ga,
                                    w_codes=cw, w_scales=sw, g_w=gw)


# ----------------------------------------------- MMA-consumable scale order --

def mma_scale_bytes(rows: int, nsf: int) -> int:
    return int(lib().orc_mma_scale_bytes(rows, nsf))


def scales_to_mma(rowmajor: np.ndarray) -> np.ndarray:
    rowmajor = np.ascontiguousarray(rowmajor, np.uint8)
    rows, nsf = rowmajor.shape
    out = np.empty(mma_scale_bytes(rows, nsf), np.uint8)
    lib().orc_scales_to_mma(_ptr(rowmajor), rows, nsf, _ptr(out))
    return out


def scales_from_mma(mma: np.ndarray, rows: int, nsf: int) -> np.ndarray:
    mma = np.ascontiguousarray(mma, np.uint8)
    out = np.empty((rows, nsf), np.uint8)
    lib().orc_scales_from_mma(_ptr(mma), rows, nsf, _ptr(out))
    return out


def threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)
