// out_quant.cuh -- the GEMM epilogue that emits the next layer's FP4
// activation instead of (or beside) a bf16 C: every output row's bf16 values
// (C rounded to bf16 exactly as fp4_gemm writes it) go through the
// activation quantizer's arithmetic (codec.cuh) with a STATIC global scale
// (NVFP4) or the MXFP4 rule, optionally after the online rotation, and leave
// as packed codes [M, N/2] plus scales in the MMA or row-major order of a
// [M, N] activation.  "FP4 n'existe pas : il existe des FP4, et chaque
// runtime choisit son dialecte", section "TensorRT-LLM 1.3 : NVFP4 natif,
// verrouille NVIDIA": quantization, scaling, matmul and de-scaling in one
// launch, with no HBM round trip between the steps.
#pragma once
#include <cstdint>

#include "codec.cuh"

namespace fp4 {

struct QuantOut {
  uint8_t* codes;       // [M, N/2]
  uint8_t* scales;      // MMA order (rows padded to 128, columns to 4) or [M, N/B]
  const float* g;       // NVFP4: the STATIC global scale of the output
  int fmt, layout;      // 0 NVFP4 / 1 MXFP4; 0 MMA / 1 row-major
  int rule;             // MXFP4 scale rule
  int rot;              // 0, 16 or 32
  float rot_scale;
  int nsf, ncb;         // scale columns of a row (N / B) and their 4-column groups
};

// Per-thread constants of the NVFP4 scale step from the STATIC g, and the
// reciprocals r = RN(1 / RN(s g)) of every scale byte s <= 0x7F in shared
// memory (r_tab, 128 floats, filled by the 128 epilogue threads: it
// depends on the scale byte alone, so no block computes a reciprocal).
struct QuantOutG {
  float g, six_g, y6;
  bool fast_b;
  const float* r_tab;
};
// Every epilogue thread calls this once (tid = 0..127); the caller
// synchronizes the 128 threads before the first quant_out_row.
__device__ __forceinline__ QuantOutG quant_out_g(const QuantOut& q, float* r_tab, int tid) {
  QuantOutG c;
  c.g = q.fmt == 0 ? *q.g : 1.0f;
  c.six_g = __fmul_rn(6.0f, c.g);
  c.y6 = __frcp_rn(c.six_g);
  c.fast_b = c.six_g >= 0x1p-40f && c.six_g <= 0x1p40f;
  if (q.fmt == 0) r_tab[tid] = nvfp4_recip(static_cast<unsigned>(tid), c.g);
  c.r_tab = r_tab;
  return c;
}

__device__ __forceinline__ long long out_scale_offset(const QuantOut& q, long long r, int c) {
  if (q.layout == 1) return r * q.nsf + c;
  const long long atom = (r >> 7) * q.ncb + (c >> 2);
  const int rr = static_cast<int>(r & 127);
  return atom * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3);
}

// The epilogue's multiplier of accumulator column n: alpha, or with MXFP4
// macro-block scaling (MBS) RN(sigma_a[row] * sigma_w[n]) -- `a` is then
// sigma_a[row]; columns past N get 0 (never stored).
template <bool MBS>
__device__ __forceinline__ float col_scale(float a, const float* sigma_w, int n, int N) {
  if (!MBS) return a;
  return __fmul_rn(a, n < N ? __ldg(sigma_w + n) : 0.0f);
}

// One row's BN output columns [n0, n0 + BN) as packed bf16 (word i = columns
// 2i, 2i+1): quantize and store them.  row_real: row < M (codes and scales);
// a row of the last 128-row block past M (MMA order) gets zero scales.
// Scale columns past N up to the 4-column group boundary (MMA order) are
// written as zero by the tile that covers them.  N % 32 == 0.
// srow != 0: the row's BN / 2 code bytes go to shared memory at srow (16-byte
// chunk j at srow + ((j ^ swz) << 4), the 128-byte swizzle of a TMA store
// box) instead of global memory; the caller stores the box.  ROT: the
// rotation order fixed at compile time (0: none, 16, 32), or -1 for q.rot at
// run time (a kernel that instantiates one rotation keeps no registers for
// the others).
template <int BN, int FMT, int ROT = -1>
__device__ __forceinline__ void quant_out_row(const QuantOut& q, const QuantOutG& gc,
                                              const uint32_t* packed, long long row, bool row_real,
                                              bool row_pad, int n0, int N, uint32_t srow = 0u,
                                              int swz = 0) {
  constexpr int B16 = BN / 16;
  if (!row_real && !row_pad) return;
  uint8_t sb[B16];
#pragma unroll
  for (int u = 0; u < B16; u += 2) {
    // two 16-value units: an MXFP4 block or two NVFP4 blocks
    const int col = n0 + 16 * u;
    uint2 c0 = make_uint2(0u, 0u), c1 = make_uint2(0u, 0u);
    unsigned s0 = 0u, s1 = 0u;
    if (row_real && col < N) {
      const uint32_t* w = packed + 8 * u;
      const int rot = ROT >= 0 ? ROT : q.rot;
      if (rot == 0) {
        unsigned m0 = fold_u16x2(max_u16x2(mag_max8(make_uint4(w[0], w[1], w[2], w[3])),
                                           mag_max8(make_uint4(w[4], w[5], w[6], w[7]))));
        unsigned m1 = fold_u16x2(max_u16x2(mag_max8(make_uint4(w[8], w[9], w[10], w[11])),
                                           mag_max8(make_uint4(w[12], w[13], w[14], w[15]))));
        if (FMT == 0) {
          s0 = nvfp4_scale_byte(m0, gc.six_g, gc.y6, gc.fast_b);
          s1 = nvfp4_scale_byte(m1, gc.six_g, gc.y6, gc.fast_b);
          const float r0 = gc.r_tab[s0 & 127u], r1 = gc.r_tab[s1 & 127u];
          if (r0 != 0.0f) c0 = make_uint2(quant8(w[0], w[1], w[2], w[3], r0), quant8(w[4], w[5], w[6], w[7], r0));
          if (r1 != 0.0f) c1 = make_uint2(quant8(w[8], w[9], w[10], w[11], r1), quant8(w[12], w[13], w[14], w[15], r1));
        } else {
          float r;
          s0 = mxfp4_scale_f32(max(m0, m1) << 16, q.rule, &r);
          c0 = make_uint2(quant8(w[0], w[1], w[2], w[3], r), quant8(w[4], w[5], w[6], w[7], r));
          c1 = make_uint2(quant8(w[8], w[9], w[10], w[11], r), quant8(w[12], w[13], w[14], w[15], r));
        }
      } else {
        float lo[16], hi[16];
        unpack16(make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]), lo);
        unpack16(make_uint4(w[8], w[9], w[10], w[11]), make_uint4(w[12], w[13], w[14], w[15]), hi);
        if (rot == 32) {
          rotate_block32(lo, hi, q.rot_scale);
        } else {
          rotate_unit<16>(lo, q.rot_scale, false);
          rotate_unit<16>(hi, q.rot_scale, false);
        }
        const unsigned m0 = mag_max16(lo), m1 = mag_max16(hi);
        if (FMT == 0) {
          s0 = nvfp4_scale_byte_f32(m0, gc.six_g, gc.y6, gc.fast_b);
          s1 = nvfp4_scale_byte_f32(m1, gc.six_g, gc.y6, gc.fast_b);
          const float r0 = gc.r_tab[s0 & 127u], r1 = gc.r_tab[s1 & 127u];
          if (r0 != 0.0f) c0 = make_uint2(quant8_f32(lo, r0), quant8_f32(lo + 8, r0));
          if (r1 != 0.0f) c1 = make_uint2(quant8_f32(hi, r1), quant8_f32(hi + 8, r1));
        } else {
          float r;
          s0 = mxfp4_scale_f32(max(m0, m1), q.rule, &r);
          c0 = make_uint2(quant8_f32(lo, r), quant8_f32(lo + 8, r));
          c1 = make_uint2(quant8_f32(hi, r), quant8_f32(hi + 8, r));
        }
      }
      if (srow == 0u)
        *reinterpret_cast<uint4*>(q.codes + row * (N / 2) + col / 2) = make_uint4(c0.x, c0.y, c1.x, c1.y);
    }
    if (srow != 0u)
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(srow + (((u >> 1) ^ swz) << 4)),
                   "r"(c0.x), "r"(c0.y), "r"(c1.x), "r"(c1.y) : "memory");
    sb[u] = static_cast<uint8_t>(s0);
    sb[u + 1] = static_cast<uint8_t>(s1);
  }
  // scale bytes: scale column c of this tile = n0 / B + j; the last tile
  // also writes the padding columns up to the 4-column group (MMA order),
  // which a 64-wide MXFP4 tile does not reach by itself
  constexpr int per = FMT == 0 ? B16 : B16 / 2;
  const int c0 = FMT == 0 ? n0 / 16 : n0 / 32;
  const int c_end = q.layout == 0 ? 4 * q.ncb : q.nsf;   // padding columns up to the group
  if (!row_real && q.layout != 0) return;
  // four consecutive scale columns from a multiple of 4 are one aligned word
  // in the MMA order (and in a row-major order whose rows are whole words):
  // one 4-byte store instead of four byte stores
  if (per % 4 == 0 && (q.layout == 0 || q.nsf % 4 == 0)) {
#pragma unroll
    for (int j = 0; j < per; j += 4) {
      const int c = c0 + j;
      if (c >= c_end) break;
      uint32_t v = 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (row_real && c + k < q.nsf) v |= static_cast<uint32_t>(FMT == 0 ? sb[j + k] : sb[2 * (j + k)]) << (8 * k);
      *reinterpret_cast<uint32_t*>(q.scales + out_scale_offset(q, row, c)) = v;
    }
    if (n0 + BN >= N)
      for (int c = c0 + per; c < c_end; c += 4)
        *reinterpret_cast<uint32_t*>(q.scales + out_scale_offset(q, row, c)) = 0u;
    return;
  }
#pragma unroll
  for (int j = 0; j < per; ++j) {
    const int c = c0 + j;
    if (c >= c_end) break;
    const uint8_t v = (row_real && c < q.nsf) ? (FMT == 0 ? sb[j] : sb[2 * j]) : uint8_t{0};
    q.scales[out_scale_offset(q, row, c)] = v;
  }
  if (n0 + BN >= N)
    for (int c = c0 + per; c < c_end; ++c) q.scales[out_scale_offset(q, row, c)] = 0;
}

}  // namespace fp4
