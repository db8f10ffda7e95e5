"""Torch-facing wrappers over the C ABI.

PyTorch is only the plumbing here: it allocates device memory and supplies
the current CUDA stream.  Each function checks its tensors, allocates the
outputs and calls one C entry point; the work runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import ctypes

import torch

from . import fp4lib as L

NVFP4 = L.FP4_NVFP4
MXFP4 = L.FP4_MXFP4
SCALES_MMA = L.FP4_SCALES_MMA
SCALES_ROWMAJOR = L.FP4_SCALES_ROWMAJOR

_ws_cache: dict[int, torch.Tensor] = {}


def workspace(nbytes: int, device: torch.device) -> torch.Tensor:
    """A grow-only per-device scratch buffer (no initialisation needed)."""
    idx = device.index if device.index is not None else torch.cuda.current_device()
    buf = _ws_cache.get(idx)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1 << 16), dtype=torch.uint8, device=device)
        _ws_cache[idx] = buf
    return buf


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _check(status: int, what: str):
    if status != L.FP4_OK:
        raise L.Fp4Error(status, what)


def _check_out(out: torch.Tensor, M: int, N: int, device: torch.device):
    """A caller's output must be exactly [M, N] (rows may be strided: the
    leading dimension is out.stride(0)), unit-stride along N, bf16 or fp32,
    on the operands' device -- the kernels write M x N values through it."""
    if out.dim() != 2 or tuple(out.shape) != (M, N) or (N > 1 and out.stride(1) != 1):
        raise ValueError(f"out must be [{M}, {N}] with unit stride along N, got "
                         f"{tuple(out.shape)} strides {tuple(out.stride())}")
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or fp32")
    if out.device != device:
        raise ValueError(f"out is on {out.device}, the operands on {device}")


def _check_scalar(t: torch.Tensor, name: str, device: torch.device):
    """A global scale the kernels read (or write) at t.data_ptr()."""
    if t.dtype != torch.float32 or t.numel() < 1 or t.device != device:
        raise ValueError(f"{name} must be a float32 tensor of at least one element on {device}")


def _check_quantized(q: "Quantized", name: str, device: torch.device):
    """The buffers of a quantized operand must hold what the kernels read:
    codes uint8 [rows, K/2], at least fp4_scale_bytes scale bytes, a float32
    global scale (and rows macro-block scales), all on one device."""
    if (q.codes.dtype != torch.uint8 or tuple(q.codes.shape) != (q.rows, q.K // 2)
            or not q.codes.is_contiguous()):
        raise ValueError(f"{name}.codes must be contiguous uint8 [{q.rows}, {q.K // 2}]")
    need = L.fp4_scale_bytes(q.rows, q.K, q.fmt, q.layout)
    if q.scales.dtype != torch.uint8 or not q.scales.is_contiguous() or q.scales.numel() < need:
        raise ValueError(f"{name}.scales must be contiguous uint8 of at least {need} bytes")
    _check_scalar(q.g, f"{name}.g", device)
    if q.sigma is not None and (q.sigma.dtype != torch.float32 or q.sigma.numel() < q.rows
                                or not q.sigma.is_contiguous()):
        raise ValueError(f"{name}.sigma must be contiguous float32 of at least {q.rows} values")
    for t in (q.codes, q.scales) + ((q.sigma,) if q.sigma is not None else ()):
        if t.device != device:
            raise ValueError(f"{name} has buffers on {t.device}, expected {device}")


def _cuda_bf16_2d(t: torch.Tensor, name: str):
    if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D bf16 CUDA tensor")


@dataclass
class Quantized:
    """Packed FP4 codes + scales + global scale of a [rows, K] tensor."""
    codes: torch.Tensor      # uint8 [rows, K/2]
    scales: torch.Tensor     # uint8, layout-dependent size
    g: torch.Tensor          # float32 [1] (NVFP4); ones for MXFP4
    fmt: int
    layout: int
    rows: int
    K: int
    hadamard: int = 0        # online rotation order (0, 16, 32)
    mx_rule: int = 0         # MXFP4 scale rule (0 OCP, 1 overflow-aware)
    sigma: torch.Tensor | None = None   # MXFP4 macro-block scales [rows] (or None)


def quantize(x: torch.Tensor, fmt: int = NVFP4, layout: int = SCALES_MMA,
             g: torch.Tensor | None = None, ws: torch.Tensor | None = None,
             hadamard: int = 0, mx_rule: int = 0, mbs: bool = False) -> Quantized:
    """fp4_quantize_act (fp4_quantize_act_ex with a rotation or rule): DYNAMIC
    global scale when g is None, else STATIC g.  ws: scratch of at least
    fp4_workspace_bytes bytes; calls that may run concurrently (other
    streams) need their own, else the shared per-device buffer is used."""
    _cuda_bf16_2d(x, "x")
    rows, K = x.shape
    dev = x.device
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(max(L.fp4_scale_bytes(rows, K, fmt, layout), 1), dtype=torch.uint8,
                         device=dev)
    gmode = L.FP4_GLOBAL_DYNAMIC if g is None else L.FP4_GLOBAL_STATIC
    gt = torch.ones(1, dtype=torch.float32, device=dev) if g is None else g
    _check_scalar(gt, "g", dev)
    ws_bytes = L.fp4_workspace_bytes(rows, 0, K, fmt)
    if ws is None:
        ws = workspace(ws_bytes, dev)
    elif ws.numel() < ws_bytes:
        raise ValueError("workspace too small")
    sigma = torch.empty(max(rows, 1), dtype=torch.float32, device=dev) if mbs else None
    if hadamard or mx_rule or mbs:
        _check(L.fp4_quantize_act_ex(x.data_ptr(), rows, K, fmt, layout, gmode,
                                     L.opts(hadamard, mx_rule,
                                            sigma.data_ptr() if mbs else None),
                                     gt.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                                     ws.data_ptr(), ws.numel(), _stream()),
               "fp4_quantize_act_ex")
    else:
        _check(L.fp4_quantize_act(x.data_ptr(), rows, K, fmt, layout, gmode, gt.data_ptr(),
                                  codes.data_ptr(), scales.data_ptr(), ws.data_ptr(), ws.numel(),
                                  _stream()), "fp4_quantize_act")
    return Quantized(codes, scales, gt, fmt, layout, rows, K, hadamard, mx_rule, sigma)


def quantize_weights(w: torch.Tensor, fmt: int = NVFP4, hadamard: int = 0,
                     mx_rule: int = 0, mbs: bool = False) -> Quantized:
    """fp4_quantize_weights (fp4_quantize_weights_ex with a rotation or
    rule): one-time, MMA scale layout, DYNAMIC g."""
    _cuda_bf16_2d(w, "w")
    N, K = w.shape
    dev = w.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(max(L.fp4_scale_bytes(N, K, fmt, SCALES_MMA), 1), dtype=torch.uint8,
                         device=dev)
    g = torch.ones(1, dtype=torch.float32, device=dev)
    ws = workspace(L.fp4_workspace_bytes(N, 0, K, fmt), dev)
    sigma = torch.empty(max(N, 1), dtype=torch.float32, device=dev) if mbs else None
    if hadamard or mx_rule or mbs:
        _check(L.fp4_quantize_weights_ex(w.data_ptr(), N, K, fmt,
                                         L.opts(hadamard, mx_rule,
                                                sigma.data_ptr() if mbs else None),
                                         codes.data_ptr(), scales.data_ptr(), g.data_ptr(),
                                         ws.data_ptr(), ws.numel(), _stream()),
               "fp4_quantize_weights_ex")
    else:
        _check(L.fp4_quantize_weights(w.data_ptr(), N, K, fmt, codes.data_ptr(),
                                      scales.data_ptr(), g.data_ptr(), ws.data_ptr(), ws.numel(),
                                      _stream()), "fp4_quantize_weights")
    return Quantized(codes, scales, g, fmt, SCALES_MMA, N, K, hadamard, mx_rule, sigma)


def gemm(a: Quantized, w: Quantized, out_dtype=torch.bfloat16,
         out: torch.Tensor | None = None, max_sms: int = 0) -> torch.Tensor:
    """fp4_gemm: C = alpha * A_hat . W_hat^T.  max_sms: the SMs the launch
    shape is chosen for (0 = all; concurrent GEMMs each take a share)."""
    if a.fmt != w.fmt or a.K != w.K or a.layout != SCALES_MMA or w.layout != SCALES_MMA:
        raise ValueError("operands must share format and K and use the MMA scale layout")
    if a.hadamard != w.hadamard:
        raise ValueError("a rotated activation needs weights rotated with the same order")
    if (a.sigma is None) != (w.sigma is None):
        raise ValueError("macro-block scaling needs both operands quantized with it")
    M, N, K = a.rows, w.rows, a.K
    dev = a.codes.device
    _check_quantized(a, "a", dev)
    _check_quantized(w, "w", dev)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    _check_out(out, M, N, dev)
    o = L.FP4_OUT_F32 if out.dtype == torch.float32 else L.FP4_OUT_BF16
    if a.sigma is not None:
        _check(L.fp4_gemm_mbs(a.codes.data_ptr(), a.scales.data_ptr(), a.sigma.data_ptr(),
                              w.codes.data_ptr(), w.scales.data_ptr(), w.sigma.data_ptr(), M, N, K,
                              out.data_ptr(), out.stride(0), o, None, 0, max_sms, _stream()),
               "fp4_gemm_mbs")
        return out
    _check(L.fp4_gemm(a.codes.data_ptr(), a.scales.data_ptr(), a.g.data_ptr(),
                      w.codes.data_ptr(), w.scales.data_ptr(), w.g.data_ptr(), M, N, K, a.fmt,
                      out.data_ptr(), out.stride(0), o, None, 0, max_sms, _stream()), "fp4_gemm")
    return out


def gemm_quant(a: Quantized, w: Quantized, out_fmt: int = NVFP4, out_layout: int = SCALES_MMA,
               g_out: torch.Tensor | None = None, hadamard: int = 0, mx_rule: int = 0,
               with_c: bool = False, max_sms: int = 0):
    """fp4_gemm_quant: C = alpha * A_hat . W_hat^T rounded to bf16 and
    quantized in the GEMM's epilogue as the next layer's activation (NVFP4
    with the STATIC global scale g_out, or MXFP4).  Returns (Quantized of
    the [M, N] activation, bf16 C or None)."""
    if a.fmt != w.fmt or a.K != w.K or a.layout != SCALES_MMA or w.layout != SCALES_MMA:
        raise ValueError("operands must share format and K and use the MMA scale layout")
    if a.hadamard != w.hadamard:
        raise ValueError("a rotated activation needs weights rotated with the same order")
    M, N, K = a.rows, w.rows, a.K
    dev = a.codes.device
    _check_quantized(a, "a", dev)
    _check_quantized(w, "w", dev)
    codes = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(max(L.fp4_scale_bytes(M, N, out_fmt, out_layout), 1), dtype=torch.uint8,
                         device=dev)
    if g_out is None:
        g_out = torch.ones(1, dtype=torch.float32, device=dev)
    _check_scalar(g_out, "g_out", dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if with_c else None
    _check(L.fp4_gemm_quant(a.codes.data_ptr(), a.scales.data_ptr(), a.g.data_ptr(),
                            w.codes.data_ptr(), w.scales.data_ptr(), w.g.data_ptr(), M, N, K,
                            a.fmt, out_fmt, out_layout, L.opts(hadamard, mx_rule),
                            g_out.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                            c.data_ptr() if c is not None else None, N, None, 0, max_sms,
                            _stream()), "fp4_gemm_quant")
    return Quantized(codes, scales, g_out, out_fmt, out_layout, M, N, hadamard, mx_rule), c


@dataclass
class QuantizedExperts:
    """E experts' weights [E, N, K] quantized one by one (MMA scale order),
    stored back to back as fp4_gemm_grouped reads them."""
    codes: torch.Tensor      # uint8 [E, N, K/2]
    scales: torch.Tensor     # uint8 [E, per-expert scale bytes]
    g: torch.Tensor          # float32 [E]
    fmt: int
    E: int
    N: int
    K: int


def quantize_experts(w: torch.Tensor, fmt: int = NVFP4) -> QuantizedExperts:
    """fp4_quantize_weights per expert of a bf16 [E, N, K] tensor (each with
    its own DYNAMIC global scale), into one stacked buffer."""
    if not w.is_cuda or w.dtype != torch.bfloat16 or w.dim() != 3 or not w.is_contiguous():
        raise ValueError("w must be a contiguous 3-D bf16 CUDA tensor [E, N, K]")
    E, N, K = w.shape
    dev = w.device
    sfb = L.fp4_scale_bytes(N, K, fmt, SCALES_MMA)
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((E, sfb), dtype=torch.uint8, device=dev)
    g = torch.ones(E, dtype=torch.float32, device=dev)
    ws = workspace(L.fp4_workspace_bytes(N, 0, K, fmt), dev)
    for e in range(E):
        _check(L.fp4_quantize_weights(w[e].data_ptr(), N, K, fmt, codes[e].data_ptr(),
                                      scales[e].data_ptr(), g[e:].data_ptr(), ws.data_ptr(),
                                      ws.numel(), _stream()), "fp4_quantize_weights")
    return QuantizedExperts(codes, scales, g, fmt, E, N, K)


def gemm_grouped(a: Quantized, w: QuantizedExperts, offsets: torch.Tensor,
                 out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                 max_sms: int = 0) -> torch.Tensor:
    """fp4_gemm_grouped: rows [offsets[e], offsets[e+1]) of the quantized
    activation times expert e's weights.  offsets: int32 CUDA tensor [E+1]."""
    if a.fmt != w.fmt or a.K != w.K or a.layout != SCALES_MMA:
        raise ValueError("operands must share format and K and use the MMA scale layout")
    if (not offsets.is_cuda or offsets.dtype != torch.int32 or offsets.numel() != w.E + 1
            or not offsets.is_contiguous()):
        raise ValueError("offsets must be a contiguous int32 CUDA tensor of E + 1 entries")
    M, N, K = a.rows, w.N, a.K
    dev = a.codes.device
    _check_quantized(a, "a", dev)
    sfb = L.fp4_scale_bytes(N, K, w.fmt, SCALES_MMA)
    if (w.codes.dtype != torch.uint8 or tuple(w.codes.shape) != (w.E, N, K // 2)
            or not w.codes.is_contiguous() or w.scales.dtype != torch.uint8
            or tuple(w.scales.shape) != (w.E, sfb) or not w.scales.is_contiguous()
            or w.g.dtype != torch.float32 or w.g.numel() < w.E
            or any(t.device != dev for t in (w.codes, w.scales, w.g))):
        raise ValueError(f"experts must be uint8 codes [{w.E}, {N}, {K // 2}], uint8 scales "
                         f"[{w.E}, {sfb}] and float32 g [{w.E}], contiguous, on {dev}")
    if offsets.device != dev:
        raise ValueError(f"offsets are on {offsets.device}, the operands on {dev}")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    _check_out(out, M, N, dev)
    o = L.FP4_OUT_F32 if out.dtype == torch.float32 else L.FP4_OUT_BF16
    _check(L.fp4_gemm_grouped(a.codes.data_ptr(), a.scales.data_ptr(), a.g.data_ptr(),
                              w.codes.data_ptr(), w.scales.data_ptr(), w.g.data_ptr(),
                              offsets.data_ptr(), w.E, M, N, K, a.fmt, out.data_ptr(),
                              out.stride(0), o, None, 0, max_sms, _stream()), "fp4_gemm_grouped")
    return out


def gemm_plan(M: int, N: int, K: int, fmt: int = NVFP4, max_sms: int = 0) -> tuple[int, int, int]:
    """fp4_gemm_plan: (tile_m, tile_n, splits) that fp4_gemm launches."""
    tm, tn, sp = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(L.fp4_gemm_plan(M, N, K, fmt, max_sms, ctypes.byref(tm), ctypes.byref(tn),
                           ctypes.byref(sp)), "fp4_gemm_plan")
    return tm.value, tn.value, sp.value


def gemm_fused(x: torch.Tensor, w: Quantized, out_dtype=torch.bfloat16,
               g_a: torch.Tensor | None = None, out: torch.Tensor | None = None,
               g_out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
               max_sms: int = 0, mx_rule: int = 0) -> torch.Tensor:
    """fp4_gemm_fused (fp4_gemm_fused_ex when w is rotated or a rule is
    given): quantize x (M <= 32) on the fly and multiply with w; x is
    rotated with w's order.  ws: as for quantize (concurrent calls need
    their own); max_sms as for gemm."""
    _cuda_bf16_2d(x, "x")
    M, K = x.shape
    N = w.rows
    dev = x.device
    _check_quantized(w, "w", dev)
    if K != w.K:
        raise ValueError(f"x has K = {K}, w has K = {w.K}")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    _check_out(out, M, N, dev)
    o = L.FP4_OUT_F32 if out.dtype == torch.float32 else L.FP4_OUT_BF16
    gmode = L.FP4_GLOBAL_DYNAMIC if g_a is None else L.FP4_GLOBAL_STATIC
    if g_a is None:
        g_a = g_out if g_out is not None else torch.ones(1, dtype=torch.float32, device=dev)
    _check_scalar(g_a, "g_a" if gmode == L.FP4_GLOBAL_STATIC else "g_out", dev)
    need = L.fp4_workspace_bytes(M, N, K, w.fmt)
    if ws is None:
        ws = workspace(need, dev)
    elif ws.numel() < need:
        raise ValueError("workspace too small")
    if w.hadamard or mx_rule:
        _check(L.fp4_gemm_fused_ex(x.data_ptr(), w.codes.data_ptr(), w.scales.data_ptr(),
                                   w.g.data_ptr(), M, N, K, w.fmt, gmode,
                                   L.opts(w.hadamard, mx_rule), g_a.data_ptr(), out.data_ptr(),
                                   out.stride(0), o, ws.data_ptr(), ws.numel(), max_sms,
                                   _stream()), "fp4_gemm_fused_ex")
    else:
        _check(L.fp4_gemm_fused(x.data_ptr(), w.codes.data_ptr(), w.scales.data_ptr(),
                                w.g.data_ptr(), M, N, K, w.fmt, gmode, g_a.data_ptr(),
                                out.data_ptr(), out.stride(0), o, ws.data_ptr(), ws.numel(),
                                max_sms, _stream()), "fp4_gemm_fused")
    return out


def device_status():
    """(status, watchdog word); synchronizes the current stream."""
    return L.fp4_device_status(_stream())
