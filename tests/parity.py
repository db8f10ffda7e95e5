"""Shared parity helpers: GPU results against the oracle.

Tolerances (stated for the GEMM outputs): with C_ref the binary64 product
of the oracle's dequantized operands,
    bf16 output:  |C - C_ref| <= 1e-2 * max(|C_ref|, rms(C_ref))
    fp32 output:  |C - C_ref| <= 1e-4 * max(|C_ref|, rms(C_ref))
elementwise.  Codes, scales and the global scale must match bit for bit.
"""
import numpy as np
import torch

TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def gemm_close(c_gpu: torch.Tensor, c_ref: np.ndarray, dtype, rms=None):
    """Returns (ok, worst ratio err / bound, index of the worst element)."""
    c = c_gpu.detach().float().cpu().numpy().astype(np.float64)
    if rms is None:
        rms = float(np.sqrt(np.mean(c_ref ** 2)))
    bound = TOL[dtype] * np.maximum(np.abs(c_ref), rms)
    bound = np.where(bound == 0, 1e-300, bound)
    ratio = np.abs(c - c_ref) / bound
    worst = np.unravel_index(int(np.argmax(ratio)), ratio.shape) if ratio.size else None
    ok = bool(np.all(np.isfinite(c)) and np.all(ratio <= 1.0))
    return ok, float(ratio.max()) if ratio.size else 0.0, worst


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
