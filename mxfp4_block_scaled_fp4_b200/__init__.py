"""W4A4 block-scaled FP4 (NVFP4 / MXFP4) for NVIDIA B200 (sm_100a).

  fp4lib   ctypes binding of the C ABI (include/fp4.h), same names
  ops      torch-facing wrappers: quantize, quantize_weights, gemm, gemm_fused
  inputs   seeded synthetic workloads (no method arithmetic)
  build    nvcc build of libfp4_b200.so
"""
from .fp4lib import Fp4Error, lib  # noqa: F401
