// codec.cuh -- device-side NVFP4 / MXFP4 element and scale codecs, shared by
// the stand-alone quantizer (quantize.cu) and the fused small-M kernel
// (fused.cu), so both produce identical codes.
//
// "Hardware FP4 inference for speech on Blackwell", section "NVFP4, and the
// two ways it fails": E2M1 code points {0, 0.5, 1, 1.5, 2, 3, 4, 6}, E4M3
// block scale with maximum 448.  MXFP4 E8M0 scale: "FP4 n'existe pas", format
// table.  Every floating-point step is one explicitly rounded binary32
// operation (no contraction).
#pragma once
#include <cstdint>

namespace fp4 {

// Largest bf16 magnitude pattern of two packed bf16 (sign cleared); for
// finite values the 15-bit pattern orders like the magnitude.
__device__ __forceinline__ unsigned bf16x2_mag(unsigned w) { return w & 0x7FFF7FFFu; }

__device__ __forceinline__ unsigned mag_max8(uint4 v) {
  return __vmaxu2(__vmaxu2(bf16x2_mag(v.x), bf16x2_mag(v.y)),
                  __vmaxu2(bf16x2_mag(v.z), bf16x2_mag(v.w)));
}

__device__ __forceinline__ unsigned fold_u16x2(unsigned m) { return max(m & 0xFFFFu, m >> 16); }

__device__ __forceinline__ float bf16_lo(unsigned w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(unsigned w) { return __uint_as_float(w & 0xFFFF0000u); }

// E4M3 (round to nearest even, saturating at 448) of a non-negative float.
__device__ __forceinline__ unsigned to_e4m3(float v) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// Exact value of a non-negative finite E4M3 code.
__device__ __forceinline__ float e4m3_value(unsigned c) {
  const unsigned e = c >> 3, m = c & 7u;
  if (e == 0) return __uint2float_rn(m) * 0.001953125f;          // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));         // (8+m) 2^(e-10)
}

// Eight floats -> eight E2M1 nibbles (value i in nibble i), round to
// nearest even, saturating at 6.
__device__ __forceinline__ unsigned to_e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                              float v5, float v6, float v7) {
  unsigned out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return out;
}

// Sign bits of four bf16x2 words moved to bit 3 of each nibble: the code of
// a negative input carries its sign, also when it rounds to zero.
__device__ __forceinline__ unsigned sign_nibbles(unsigned w0, unsigned w1, unsigned w2,
                                                 unsigned w3) {
  auto s = [](unsigned w) { return ((w >> 12) & 0x8u) | ((w >> 24) & 0x80u); };
  return s(w0) | s(w1) << 8 | s(w2) << 16 | s(w3) << 24;
}

// 8 bf16 (4 words) times r -> 8 packed E2M1 codes.
__device__ __forceinline__ unsigned quant8(unsigned w0, unsigned w1, unsigned w2, unsigned w3,
                                           float r) {
  const unsigned q = to_e2m1x8(__fmul_rn(bf16_lo(w0), r), __fmul_rn(bf16_hi(w0), r),
                               __fmul_rn(bf16_lo(w1), r), __fmul_rn(bf16_hi(w1), r),
                               __fmul_rn(bf16_lo(w2), r), __fmul_rn(bf16_hi(w2), r),
                               __fmul_rn(bf16_lo(w3), r), __fmul_rn(bf16_hi(w3), r));
  return q | sign_nibbles(w0, w1, w2, w3);
}

// floor(log2(b)) of a positive finite float, from its bits.
__device__ __forceinline__ int floor_log2(float b) {
  const unsigned u = __float_as_uint(b);
  const int ex = static_cast<int>((u >> 23) & 0xFFu);
  if (ex != 0) return ex - 127;
  return (31 - __clz(u & 0x7FFFFFu)) - 149;
}

// One 16-value NVFP4 block: magnitude bits of its max -> E4M3 scale byte and
// the reciprocal r = 1 / (s g) (0 when the scale rounds to zero).
__device__ __forceinline__ unsigned nvfp4_scale(unsigned amax_bits, float g, float six_g,
                                                float* r) {
  const unsigned s = to_e4m3(__fdiv_rn(__uint_as_float(amax_bits << 16), six_g));
  const float sv = e4m3_value(s);
  *r = (sv == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(sv, g));
  return s;
}

// One 32-value MXFP4 block: E8M0 scale byte and r = 2^-e.
__device__ __forceinline__ unsigned mxfp4_scale(unsigned amax_bits, float* r) {
  const float b = __uint_as_float(amax_bits << 16);
  int e = (b == 0.0f) ? -127 : floor_log2(b) - 2;
  e = max(-127, min(127, e));
  *r = __uint_as_float(static_cast<unsigned>(127 - e) << 23);
  return static_cast<unsigned>(e + 127);
}

}  // namespace fp4
