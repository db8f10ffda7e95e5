"""The C ABI without a GPU: the library loads, exports every function the
header declares, the ctypes binding matches the header's prototypes, and the
host-only functions (sizes, argument checks, status strings) behave as
documented.  No compute call is made here."""
import ctypes

import pytest

from mxfp4_block_scaled_fp4_b200 import fp4lib as L


@pytest.fixture(scope="module")
def lib():
    from mxfp4_block_scaled_fp4_b200 import build
    build.build()
    return L.lib()


def test_exports_every_header_symbol(lib):
    names = L.header_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
        assert n in L.SIGNATURES, n


def test_status_strings(lib):
    for s in range(9):
        assert L.fp4_status_string(s) != "unknown status"
        assert L.fp4_status_string(s)
    assert L.fp4_status_string(0) == "ok"
    assert L.fp4_status_string(99) == "unknown status"


def test_size_queries(lib):
    assert L.fp4_packed_bytes(16, 256) == 16 * 128
    assert L.fp4_scale_bytes(16, 256, L.FP4_NVFP4, L.FP4_SCALES_ROWMAJOR) == 16 * 16
    assert L.fp4_scale_bytes(16, 256, L.FP4_MXFP4, L.FP4_SCALES_ROWMAJOR) == 16 * 8
    # MMA order: rows padded to 128, scale columns to multiples of 4 (512-byte atoms)
    assert L.fp4_scale_bytes(16, 256, L.FP4_NVFP4, L.FP4_SCALES_MMA) == 4 * 512
    assert L.fp4_scale_bytes(130, 2880, L.FP4_NVFP4, L.FP4_SCALES_MMA) == 2 * 45 * 512
    assert L.fp4_scale_bytes(1, 2880, L.FP4_MXFP4, L.FP4_SCALES_MMA) == 23 * 512
    assert L.fp4_scale_bytes(4, 100, L.FP4_NVFP4, L.FP4_SCALES_MMA) == 0     # K % 32
    assert L.fp4_workspace_bytes(8192, 0, 16384, L.FP4_NVFP4) >= 4096


def test_scale_bytes_match_oracle_layout(lib, orc):
    for rows, K in [(1, 256), (16, 2880), (300, 8192)]:
        assert L.fp4_scale_bytes(rows, K, L.FP4_NVFP4, L.FP4_SCALES_MMA) == \
            orc.mma_scale_bytes(rows, K // 16)
        assert L.fp4_scale_bytes(rows, K, L.FP4_MXFP4, L.FP4_SCALES_MMA) == \
            orc.mma_scale_bytes(rows, K // 32)


def test_gemm_plan_argument_checks(lib):
    i = [ctypes.c_int() for _ in range(3)]
    refs = [ctypes.byref(x) for x in i]
    assert L.fp4_gemm_plan(8, 256, 100, 0, 0, *refs) == L.FP4_ERR_UNSUPPORTED_SHAPE   # K % 32
    assert L.fp4_gemm_plan(8, 260, 256, 0, 0, *refs) == L.FP4_ERR_UNSUPPORTED_SHAPE   # N % 8
    assert L.fp4_gemm_plan(8, 256, 256, 7, 0, *refs) == L.FP4_ERR_INVALID_ARG
    assert L.fp4_gemm_plan(8, 256, 256, 0, -1, *refs) == L.FP4_ERR_INVALID_ARG       # max_sms
    assert L.fp4_gemm_plan(8, 256, 256, 0, 0, None, refs[1], refs[2]) == L.FP4_ERR_INVALID_ARG


def test_argument_checks_fail_before_any_launch(lib):
    fake = ctypes.c_void_p(1 << 20)           # never dereferenced: checks fail first
    mis = ctypes.c_void_p((1 << 20) + 8)
    q = L.fp4_quantize_act
    assert q(fake, 4, 100, 0, 0, 0, fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_UNSUPPORTED_SHAPE
    assert q(fake, -1, 256, 0, 0, 0, fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_UNSUPPORTED_SHAPE
    assert q(None, 4, 256, 0, 0, 0, fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_INVALID_ARG
    assert q(fake, 4, 256, 7, 0, 0, fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_INVALID_ARG
    assert q(mis, 4, 256, 0, 0, 0, fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_MISALIGNED
    assert q(fake, 4, 256, 0, 0, 0, fake, fake, fake, fake, 16, None) == \
        L.FP4_ERR_WORKSPACE_TOO_SMALL
    g = L.fp4_gemm
    assert g(fake, fake, fake, fake, fake, fake, 4, 12, 256, 0, fake, 12, 0, None, 0, 0, None) == \
        L.FP4_ERR_UNSUPPORTED_SHAPE                                   # N % 8
    assert g(fake, fake, fake, fake, fake, fake, 4, 16, 256, 0, fake, 8, 0, None, 0, 0, None) == \
        L.FP4_ERR_INVALID_ARG                                         # ldc < N
    assert g(fake, fake, fake, fake, fake, fake, 4, 16, 256, 0, fake, 20, 0, None, 0, 0, None) == \
        L.FP4_ERR_MISALIGNED                                          # ldc*2 % 16
    assert g(fake, fake, None, fake, fake, fake, 4, 16, 256, 0, fake, 16, 0, None, 0, 0, None) == \
        L.FP4_ERR_INVALID_ARG                                         # NVFP4 needs g_a
    assert g(fake, fake, fake, fake, fake, fake, 4, 16, 256, 0, fake, 16, 0, None, 0, -2, None) == \
        L.FP4_ERR_INVALID_ARG                                         # max_sms < 0
    f = L.fp4_gemm_fused
    assert f(fake, fake, fake, fake, 33, 16, 256, 0, 0, fake, fake, 16, 0, fake, 1 << 30, 0, None) == \
        L.FP4_ERR_UNSUPPORTED_SHAPE                                   # M > 32
    assert f(fake, fake, fake, fake, 8, 16, 256, 0, 0, fake, fake, 16, 0, fake, 16, 0, None) == \
        L.FP4_ERR_WORKSPACE_TOO_SMALL
    assert f(fake, fake, fake, fake, 8, 16, 256, 0, 0, fake, fake, 16, 0, fake, 1 << 30, -1, None) == \
        L.FP4_ERR_INVALID_ARG                                         # max_sms < 0


def test_no_gpu_means_no_device_status(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    fake = ctypes.c_void_p(1 << 20)
    st = L.fp4_quantize_act(fake, 4, 256, 0, 0, 0, fake, fake, fake, fake, 1 << 16, None)
    assert st in (L.FP4_ERR_NO_DEVICE,)


def test_quant_options_checked_before_any_launch(lib):
    fake = ctypes.c_void_p(1 << 20)
    qx = L.fp4_quantize_act_ex
    assert qx(fake, 4, 256, 0, 0, 0, L.opts(8, 0), fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_INVALID_ARG                                         # order 8
    assert qx(fake, 4, 256, 0, 0, 0, L.opts(0, 1), fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_INVALID_ARG                                         # OAS with NVFP4
    assert qx(fake, 4, 100, 1, 0, 0, L.opts(32, 1), fake, fake, fake, fake, 1 << 16, None) == \
        L.FP4_ERR_UNSUPPORTED_SHAPE                                   # K % 32
    assert L.fp4_quantize_weights_ex(fake, 4, 256, 1, L.opts(16, 5), fake, fake, fake, fake,
                                     1 << 16, None) == L.FP4_ERR_INVALID_ARG
    fx = L.fp4_gemm_fused_ex
    assert fx(fake, fake, fake, fake, 8, 16, 256, 0, 0, L.opts(64, 0), fake, fake, 16, 0, fake,
              1 << 30, 0, None) == L.FP4_ERR_INVALID_ARG


def _header_prototypes():
    import re
    with open(L.HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for ret, name, params in re.findall(
            r"([A-Za-z_][A-Za-z0-9_ \*]*?)\b(fp4_[a-z_]+)\s*\(([^)]*)\)\s*;", text):
        ps = [p.strip() for p in params.split(",")] if params.strip() not in ("", "void") else []
        out[name] = (ret.strip(), ps)
    return out


def _kind_of_c(t):
    """pointer / 64-bit unsigned (size_t, unsigned long long) / 32-bit int
    or enum, from a C parameter or return declaration."""
    if "*" in t:
        return "ptr"
    if "unsigned long long" in t or "size_t" in t:
        return "u64"
    return "int"


def _kind_of_ctypes(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or isinstance(getattr(t, "_type_", None), type):
        return "ptr"
    if t in (ctypes.c_ulonglong, ctypes.c_size_t) and ctypes.sizeof(t) == 8:
        return "u64"
    assert t is ctypes.c_int, t
    return "int"


def test_binding_matches_header_prototypes():
    """Every binding's argument list has the header's parameter count and,
    parameter by parameter, the same kind (pointer, size_t, 64-bit, int or
    enum); so do the return types."""
    protos = _header_prototypes()
    assert set(protos) == set(L.SIGNATURES)
    for name, (ret, params) in protos.items():
        res, args = L.SIGNATURES[name]
        assert len(args) == len(params), (name, len(args), len(params))
        for i, (c, py) in enumerate(zip(params, args)):
            assert _kind_of_c(c) == _kind_of_ctypes(py), (name, i, c, py)
        assert _kind_of_c(ret) == _kind_of_ctypes(res), (name, ret, res)
