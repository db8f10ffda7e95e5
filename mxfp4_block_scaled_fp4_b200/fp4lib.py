"""ctypes binding of libfp4_b200.so: the C ABI of include/fp4.h, same names.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the library.  There is no fallback: if the shared library is
missing or cannot be loaded, ``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp4_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "fp4.h")

# fp4_status_t
FP4_OK = 0
FP4_ERR_INVALID_ARG = 1
FP4_ERR_UNSUPPORTED_SHAPE = 2
FP4_ERR_MISALIGNED = 3
FP4_ERR_WORKSPACE_TOO_SMALL = 4
FP4_ERR_CUDA = 5
FP4_ERR_DEVICE_TIMEOUT = 6
FP4_ERR_NO_DEVICE = 7
FP4_ERR_NONFINITE = 8
# bit of the device status word that reports a non-finite DYNAMIC amax
FP4_STATUS_NONFINITE_BIT = 0x80
# fp4_format_t
FP4_NVFP4 = 0
FP4_MXFP4 = 1
# fp4_scale_layout_t
FP4_SCALES_MMA = 0
FP4_SCALES_ROWMAJOR = 1
# fp4_global_mode_t
FP4_GLOBAL_DYNAMIC = 0
FP4_GLOBAL_STATIC = 1
# fp4_out_t
FP4_OUT_BF16 = 0
FP4_OUT_F32 = 1
# fp4_mx_rule_t
FP4_MX_RULE_OCP = 0
FP4_MX_RULE_OAS = 1


class QuantOpts(ctypes.Structure):
    """fp4_quant_opts_t: online rotation order (0, 16, 32), MXFP4 rule and
    the device array that receives the macro-block scales (or NULL)."""
    _fields_ = [("hadamard", ctypes.c_int), ("mx_rule", ctypes.c_int),
                ("mbs_scale", ctypes.c_void_p)]


def opts(hadamard: int = 0, mx_rule: int = 0, mbs_scale=None):
    """A fp4_quant_opts_t by reference, or None when all are defaults."""
    if not hadamard and not mx_rule and not mbs_scale:
        return None
    return ctypes.byref(QuantOpts(hadamard, mx_rule, mbs_scale))


class Fp4Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = lib().fp4_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})" if what else msg)


_lib = None

P = ctypes.c_void_p
I = ctypes.c_int
SZ = ctypes.c_size_t
U8P = ctypes.c_void_p
FP = ctypes.c_void_p

SIGNATURES = {
    "fp4_packed_bytes": (SZ, [I, I]),
    "fp4_scale_bytes": (SZ, [I, I, I, I]),
    "fp4_workspace_bytes": (SZ, [I, I, I, I]),
    "fp4_quantize_act": (I, [P, I, I, I, I, I, FP, U8P, U8P, P, SZ, P]),
    "fp4_quantize_weights": (I, [P, I, I, I, U8P, U8P, FP, P, SZ, P]),
    "fp4_quantize_act_ex": (I, [P, I, I, I, I, I, P, FP, U8P, U8P, P, SZ, P]),
    "fp4_quantize_weights_ex": (I, [P, I, I, I, P, U8P, U8P, FP, P, SZ, P]),
    "fp4_gemm_fused_ex": (I, [P, U8P, U8P, FP, I, I, I, I, I, P, FP, P, I, I, P, SZ, I, P]),
    "fp4_gemm": (I, [U8P, U8P, FP, U8P, U8P, FP, I, I, I, I, P, I, I, P, SZ, I, P]),
    "fp4_gemm_fused": (I, [P, U8P, U8P, FP, I, I, I, I, I, FP, P, I, I, P, SZ, I, P]),
    "fp4_gemm_quant": (I, [U8P, U8P, FP, U8P, U8P, FP, I, I, I, I, I, I, P, FP, U8P, U8P, P, I,
                           P, SZ, I, P]),
    "fp4_gemm_mbs": (I, [U8P, U8P, FP, U8P, U8P, FP, I, I, I, P, I, I, P, SZ, I, P]),
    "fp4_gemm_grouped": (I, [U8P, U8P, FP, U8P, U8P, FP, P, I, I, I, I, I, P, I, I, P, SZ, I,
                             P]),
    "fp4_gemm_plan": (I, [I, I, I, I, I, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I)]),
    "fp4_quantize_act_noalloc": (I, [P, I, I, I, I, I, FP, U8P, U8P, P]),
    "fp4_device_status": (I, [ctypes.POINTER(ctypes.c_uint), P]),
    "fp4_watchdog_selftest": (I, [ctypes.c_ulonglong, P]),
    "fp4_status_string": (ctypes.c_char_p, [I]),
}


def header_symbols() -> list[str]:
    """Every function name declared in include/fp4.h."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4_[a-z_]+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python mxfp4_block_scaled_fp4_b200/build.py` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _call(name, *args):
    return getattr(lib(), name)(*args)


def fp4_packed_bytes(rows, K):
    return _call("fp4_packed_bytes", rows, K)


def fp4_scale_bytes(rows, K, fmt, layout):
    return _call("fp4_scale_bytes", rows, K, fmt, layout)


def fp4_workspace_bytes(M, N, K, fmt):
    return _call("fp4_workspace_bytes", M, N, K, fmt)


def fp4_quantize_act(x, rows, K, fmt, layout, gmode, g, codes, scales, ws, ws_bytes, stream):
    return _call("fp4_quantize_act", x, rows, K, fmt, layout, gmode, g, codes, scales, ws,
                 ws_bytes, stream)


def fp4_quantize_weights(w, N, K, fmt, codes, scales, g, ws, ws_bytes, stream):
    return _call("fp4_quantize_weights", w, N, K, fmt, codes, scales, g, ws, ws_bytes, stream)


def fp4_quantize_act_ex(x, rows, K, fmt, layout, gmode, opts, g, codes, scales, ws, ws_bytes,
                        stream):
    return _call("fp4_quantize_act_ex", x, rows, K, fmt, layout, gmode, opts, g, codes, scales,
                 ws, ws_bytes, stream)


def fp4_quantize_weights_ex(w, N, K, fmt, opts, codes, scales, g, ws, ws_bytes, stream):
    return _call("fp4_quantize_weights_ex", w, N, K, fmt, opts, codes, scales, g, ws, ws_bytes,
                 stream)


def fp4_gemm_fused_ex(a, w_codes, w_scales, g_w, M, N, K, fmt, gmode, opts, g_a, C, ldc, out, ws,
                      ws_bytes, max_sms, stream):
    return _call("fp4_gemm_fused_ex", a, w_codes, w_scales, g_w, M, N, K, fmt, gmode, opts, g_a,
                 C, ldc, out, ws, ws_bytes, max_sms, stream)


def fp4_gemm(a_codes, a_scales, g_a, w_codes, w_scales, g_w, M, N, K, fmt, C, ldc, out, ws,
             ws_bytes, max_sms, stream):
    return _call("fp4_gemm", a_codes, a_scales, g_a, w_codes, w_scales, g_w, M, N, K, fmt, C,
                 ldc, out, ws, ws_bytes, max_sms, stream)


def fp4_gemm_fused(a, w_codes, w_scales, g_w, M, N, K, fmt, gmode, g_a, C, ldc, out, ws,
                   ws_bytes, max_sms, stream):
    return _call("fp4_gemm_fused", a, w_codes, w_scales, g_w, M, N, K, fmt, gmode, g_a, C, ldc,
                 out, ws, ws_bytes, max_sms, stream)


def fp4_gemm_quant(a_codes, a_scales, g_a, w_codes, w_scales, g_w, M, N, K, fmt, out_fmt,
                   out_layout, out_opts, g_out, out_codes, out_scales, C, ldc, ws, ws_bytes,
                   max_sms, stream):
    return _call("fp4_gemm_quant", a_codes, a_scales, g_a, w_codes, w_scales, g_w, M, N, K, fmt,
                 out_fmt, out_layout, out_opts, g_out, out_codes, out_scales, C, ldc, ws,
                 ws_bytes, max_sms, stream)


def fp4_gemm_mbs(a_codes, a_scales, sigma_a, w_codes, w_scales, sigma_w, M, N, K, C, ldc, out, ws,
                 ws_bytes, max_sms, stream):
    return _call("fp4_gemm_mbs", a_codes, a_scales, sigma_a, w_codes, w_scales, sigma_w, M, N, K,
                 C, ldc, out, ws, ws_bytes, max_sms, stream)


def fp4_gemm_grouped(a_codes, a_scales, g_a, w_codes, w_scales, g_w, offsets, E, M, N, K, fmt,
                     C, ldc, out, ws, ws_bytes, max_sms, stream):
    return _call("fp4_gemm_grouped", a_codes, a_scales, g_a, w_codes, w_scales, g_w, offsets, E,
                 M, N, K, fmt, C, ldc, out, ws, ws_bytes, max_sms, stream)


def fp4_gemm_plan(M, N, K, fmt, max_sms, tile_m, tile_n, splits):
    return _call("fp4_gemm_plan", M, N, K, fmt, max_sms, tile_m, tile_n, splits)


def fp4_quantize_act_noalloc(x, rows, K, fmt, layout, gmode, g, codes, scales, stream):
    return _call("fp4_quantize_act_noalloc", x, rows, K, fmt, layout, gmode, g, codes, scales,
                 stream)


def fp4_device_status(stream=None):
    code = ctypes.c_uint(0)
    st = _call("fp4_device_status", ctypes.byref(code), stream)
    return st, code.value


def fp4_watchdog_selftest(limit_ns, stream=None):
    return _call("fp4_watchdog_selftest", limit_ns, stream)


def fp4_status_string(status):
    return _call("fp4_status_string", status).decode()
