// codec.cuh -- device-side NVFP4 / MXFP4 element and scale codecs of the
// quantizer (quantize.cu).
//
// "Hardware FP4 inference for speech on Blackwell", section "NVFP4, and the
// two ways it fails": E2M1 code points {0, 0.5, 1, 1.5, 2, 3, 4, 6}, E4M3
// block scale with maximum 448.  MXFP4 E8M0 scale: "FP4 n'existe pas", format
// table.  Every floating-point step yields the correctly rounded binary32
// result of that step (explicitly rounded operations, no contraction).
#pragma once
#include <cstdint>

namespace fp4 {

// Largest bf16 magnitude pattern of two packed bf16 (sign cleared); for
// finite values the 15-bit pattern orders like the magnitude.
__device__ __forceinline__ unsigned bf16x2_mag(unsigned w) { return w & 0x7FFF7FFFu; }

// Lane-wise maximum of two pairs of 16-bit unsigned values (native on sm_90+).
__device__ __forceinline__ unsigned max_u16x2(unsigned a, unsigned b) {
  unsigned d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ unsigned mag_max8(uint4 v) {
  return max_u16x2(max_u16x2(bf16x2_mag(v.x), bf16x2_mag(v.y)),
                   max_u16x2(bf16x2_mag(v.z), bf16x2_mag(v.w)));
}

__device__ __forceinline__ unsigned fold_u16x2(unsigned m) { return max(m & 0xFFFFu, m >> 16); }

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

// 8 bf16 (4 words, element 2i in the low half of word i) times r -> 8
// packed E2M1 codes (element i in nibble i).  Each product is one binary32
// multiply rounded to nearest (two per mul.rn.f32x2, measured on B200 to be
// bit-identical to two scalar multiplies), then round to nearest even,
// saturating at 6.  The conversion keeps the sign of a negative product that
// rounds to zero (code 0x8), measured on B200 for every such input tried,
// -0.0 included; that is the sign rule of the format.
__device__ __forceinline__ unsigned quant8(unsigned w0, unsigned w1, unsigned w2, unsigned w3,
                                           float r) {
  unsigned out;
  asm("{\n\t"
      ".reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
      ".reg .b64 x0, x1, x2, x3, rr;\n\t"
      ".reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b64 rr, {%5, %5};\n\t"
      "shl.b32 l0, %1, 16;\n\t and.b32 h0, %1, 0xFFFF0000;\n\t mov.b64 x0, {l0, h0};\n\t"
      "shl.b32 l1, %2, 16;\n\t and.b32 h1, %2, 0xFFFF0000;\n\t mov.b64 x1, {l1, h1};\n\t"
      "shl.b32 l2, %3, 16;\n\t and.b32 h2, %3, 0xFFFF0000;\n\t mov.b64 x2, {l2, h2};\n\t"
      "shl.b32 l3, %4, 16;\n\t and.b32 h3, %4, 0xFFFF0000;\n\t mov.b64 x3, {l3, h3};\n\t"
      "mul.rn.f32x2 x0, x0, rr;\n\t mul.rn.f32x2 x1, x1, rr;\n\t"
      "mul.rn.f32x2 x2, x2, rr;\n\t mul.rn.f32x2 x3, x3, rr;\n\t"
      "mov.b64 {l0, h0}, x0;\n\t mov.b64 {l1, h1}, x1;\n\t"
      "mov.b64 {l2, h2}, x2;\n\t mov.b64 {l3, h3}, x3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, h0, l0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, h1, l1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, h2, l2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, h3, l3;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "f"(r));
  return out;
}

// RN(a / b) for a >= 0 by Markstein's method (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", 1990): with
// y = RN(1/b) and q1 = RN(a y), the remainder a - b q1 is exact in one FMA
// and RN(q1 + (a - b q1) y) is the correctly rounded quotient, provided no
// intermediate under- or overflows.  fast_b says b lies in [2^-40, 2^40];
// with q1 also in that range every intermediate is a normal number, outside
// it the division itself runs.  Checked on B200 against the correctly
// rounded division for every positive finite bf16 a and 4000 divisors.
__device__ __forceinline__ float div_rn(float a, float b, float y, bool fast_b) {
  const float q1 = __fmul_rn(a, y);
  if (fast_b && q1 >= 0x1p-40f && q1 <= 0x1p40f) return __fmaf_rn(__fmaf_rn(-q1, b, a), y, q1);
  return __fdiv_rn(a, b);
}

// floor(log2(b)) of a positive finite float, from its bits.
__device__ __forceinline__ int floor_log2(float b) {
  const unsigned u = __float_as_uint(b);
  const int ex = static_cast<int>((u >> 23) & 0xFFu);
  if (ex != 0) return ex - 127;
  return (31 - __clz(u & 0x7FFFFFu)) - 149;
}

// One 16-value NVFP4 block: magnitude bits of its max -> E4M3 scale byte
// s = E4M3(RN(amax / RN(6 g))).  (y6 = RN(1 / RN(6 g)).)
__device__ __forceinline__ unsigned nvfp4_scale_byte(unsigned amax_bits, float six_g, float y6,
                                                     bool fast_b) {
  return to_e4m3(div_rn(__uint_as_float(amax_bits << 16), six_g, y6, fast_b));
}

// The reciprocal the block's values are multiplied by: r = RN(1 / RN(s g)),
// 0 when the scale is zero.  It depends on the scale byte alone, so the
// quantizer tabulates it per CTA.
__device__ __forceinline__ float nvfp4_recip(unsigned s, float g) {
  const float sv = e4m3_value(s);
  return (sv == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(sv, g));
}


// ------------------------------------------------------------------------
// Online rotation (the Hadamard rotation ahead of the activation quantizer of
// "FP4 on a consumer RTX 5090: the Blackwell headline loses to plain int4",
// section "Finding 3 -- the real-FP4 path (QuTLASS MXFP4)").  Block-diagonal
// Walsh-Hadamard of order n in {16, 32} along K, Sylvester order, computed in
// binary32 as the fast transform: for h = 1, 2, 4, ... < n every pair
// (i, i + h) with bit h of i clear becomes (RN(a + b), RN(a - b)); then a
// multiply by 2^-shift (exact).  A thread holds one 16-value unit; with
// n = 32 the last stage pairs the unit with its lane neighbour (lane ^ 1),
// whose unit is the other half of the same 32-value block.

// 16 bf16 (8 words, element 2i in the low half of word i) -> 16 floats.
__device__ __forceinline__ void unpack16(uint4 p, uint4 q, float f[16]) {
  const unsigned w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Two binary32 lanes in one 64-bit register and their packed arithmetic
// (one IEEE rounding per lane, as the scalar operations).
__device__ __forceinline__ unsigned long long f2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long add_f2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long sub_f2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ unsigned long long mul_f2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// RN(a * b + c) per lane; with b = +-1 it is RN(c +- a), one rounding.
__device__ __forceinline__ unsigned long long fma_f2(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// The in-unit stages h = 1, 2, 4, 8 of the transform on 16 values, left as
// 8 packed pairs (P[k] = values 2k, 2k+1).  Stage h = 1 pairs the two lanes
// of a packed register (scalar adds); from h = 2 on a pair of registers
// (i, i + h) moves as one packed add and one packed subtract.
__device__ __forceinline__ void fwht16_packed(float f[16], unsigned long long P[8]) {
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float a = f[i], b = f[i + 1];
    f[i] = __fadd_rn(a, b);
    f[i + 1] = __fsub_rn(a, b);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) P[k] = f2(f[2 * k], f[2 * k + 1]);
#pragma unroll
  for (int hh = 1; hh < 8; hh *= 2) {        // h = 2 hh
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if ((k & hh) == 0) {
        const unsigned long long a = P[k], b = P[k + hh];
        P[k] = add_f2(a, b);
        P[k + hh] = sub_f2(a, b);
      }
    }
  }
}

// The stages h = 1, 2, 4, 8 of the unit, then (n = 16) the scaling; n = 32
// adds the cross-lane stage h = 16 (every lane of the warp must take part)
// before it.  `odd` = this unit is the upper half of its 32-value block.
template <int N>
__device__ __forceinline__ void rotate_unit(float f[16], float scale, bool odd) {
  unsigned long long P[8];
  fwht16_packed(f, P);
  if (N == 32) {
    // lower half: own + other; upper half: other - own (= own * -1 + other)
    const float sg = odd ? -1.0f : 1.0f;
    const unsigned long long S = f2(sg, sg);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      f2_split(P[k], lo, hi);
      const float olo = __shfl_xor_sync(0xFFFFFFFFu, lo, 1);
      const float ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, 1);
      P[k] = fma_f2(P[k], S, f2(olo, ohi));
    }
  }
  const unsigned long long SC = f2(scale, scale);   // a power of two: exact
#pragma unroll
  for (int k = 0; k < 8; ++k) f2_split(mul_f2(P[k], SC), f[2 * k], f[2 * k + 1]);
}

// A whole 32-value block in one thread, held as two 16-value halves: the
// stages of both halves, then h = 16 (lo + hi, lo - hi) and the scaling, all
// as packed pairs; the same roundings as rotate_unit<32> on a lane pair.
__device__ __forceinline__ void rotate_block32(float lo[16], float hi[16], float scale) {
  unsigned long long A[8], B[8];
  fwht16_packed(lo, A);
  fwht16_packed(hi, B);
  const unsigned long long SC = f2(scale, scale);   // a power of two: exact
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    f2_split(mul_f2(add_f2(A[k], B[k]), SC), lo[2 * k], lo[2 * k + 1]);
    f2_split(mul_f2(sub_f2(A[k], B[k]), SC), hi[2 * k], hi[2 * k + 1]);
  }
}

// Largest magnitude of 16 floats as binary32 magnitude bits (Inf and NaN
// order above every finite value).
__device__ __forceinline__ unsigned mag_max16(const float f[16]) {
  // max.NaN.xorsign.abs: the magnitude of the result is the larger of the
  // two magnitudes (a NaN wins); the sign bit is dropped at the end
  float m = f[0];
#pragma unroll
  for (int i = 1; i < 16; ++i) asm("max.NaN.xorsign.abs.f32 %0, %0, %1;" : "+f"(m) : "f"(f[i]));
  return __float_as_uint(m) & 0x7FFFFFFFu;
}

// 8 floats times r -> 8 packed E2M1 codes (element i in nibble i); the
// rounding and sign rules of quant8.
__device__ __forceinline__ unsigned quant8_f32(const float* f, float r) {
  unsigned out;
  asm("{\n\t"
      ".reg .b64 x0, x1, x2, x3, rr;\n\t"
      ".reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
      ".reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b64 rr, {%9, %9};\n\t"
      "mov.b64 x0, {%1, %2};\n\t mov.b64 x1, {%3, %4};\n\t"
      "mov.b64 x2, {%5, %6};\n\t mov.b64 x3, {%7, %8};\n\t"
      "mul.rn.f32x2 x0, x0, rr;\n\t mul.rn.f32x2 x1, x1, rr;\n\t"
      "mul.rn.f32x2 x2, x2, rr;\n\t mul.rn.f32x2 x3, x3, rr;\n\t"
      "mov.b64 {l0, h0}, x0;\n\t mov.b64 {l1, h1}, x1;\n\t"
      "mov.b64 {l2, h2}, x2;\n\t mov.b64 {l3, h3}, x3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, h0, l0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, h1, l1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, h2, l2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, h3, l3;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7]),
        "f"(r));
  return out;
}

// One 16-value NVFP4 block of binary32 values: s = E4M3(RN(b / RN(6 g)))
// with b the block's largest magnitude (binary32 bits).
__device__ __forceinline__ unsigned nvfp4_scale_byte_f32(unsigned b_bits, float six_g, float y6,
                                                         bool fast_b) {
  return to_e4m3(div_rn(__uint_as_float(b_bits), six_g, y6, fast_b));
}

// One 32-value MXFP4 block of binary32 values with block maximum b (bits):
// rule 0 = OCP, e = floor(log2 b) - 2; rule 1 = overflow-aware (OAS), the
// smallest e with b <= 6 * 2^e, i.e. one more than OCP's when the
// significand of b exceeds 1.5 ("FP4 n'existe pas", section "L'ecart de
// qualite -- et comment il se reduit").  Clamped to [-127, 127]; E8M0 byte
// e + 127, r = 2^-e.
__device__ __forceinline__ unsigned mxfp4_scale_f32(unsigned b_bits, int rule, float* r) {
  const float b = __uint_as_float(b_bits);
  int e = -127;
  if (b != 0.0f) {
    e = floor_log2(b) - 2;
    if (rule) {
      const unsigned ex = (b_bits >> 23) & 0xFFu, man = b_bits & 0x7FFFFFu;
      bool above;   // significand of b > 1.5
      if (ex != 0) {
        above = man > 0x400000u;
      } else {
        const int msb = 31 - __clz(man);
        above = msb >= 1 && (man & ((1u << msb) - 1u)) > (1u << (msb - 1));
      }
      e += above ? 1 : 0;
    }
  }
  e = max(-127, min(127, e));
  *r = __uint_as_float(static_cast<unsigned>(127 - e) << 23);
  return static_cast<unsigned>(e + 127);
}

// MXFP4 macro-block scaling (the second-level scale of "FP4 n'existe pas",
// section "L'ecart de qualite -- et comment il se reduit", read as one
// binary32 scale per row): sigma = the significand of RN(A / 6) for the
// row's largest magnitude A (in [1, 2); 1 when A == 0), exact from the bits.
__device__ __forceinline__ float mbs_sigma(float A) {
  if (A == 0.0f) return 1.0f;
  const unsigned b = __float_as_uint(__fdiv_rn(A, 6.0f));
  unsigned man = b & 0x7FFFFFu;
  if (((b >> 23) & 0xFFu) == 0) {   // subnormal: normalise the significand
    const int msb = 31 - __clz(man);
    man = (man << (23 - msb)) & 0x7FFFFFu;
  }
  return __uint_as_float(0x3F800000u | man);
}

}  // namespace fp4
