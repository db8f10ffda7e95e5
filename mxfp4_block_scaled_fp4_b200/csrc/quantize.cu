// quantize.cu -- per-tensor amax and the fused block quantizer (NVFP4 and
// MXFP4) for sm_100a.
//
// Format and scale rule: "Hardware FP4 inference for speech on Blackwell",
// section "NVFP4, and the two ways it fails" (E2M1 code points, 16-value
// blocks, s = E4M3(max|x|/6), E4M3 max 448, per-tensor FP32 scale with
// saturation, 2688 = 6 * 448).  MXFP4: "FP4 n'existe pas : il existe des
// FP4, et chaque runtime choisit son dialecte", section "Deux dialectes,
// deux strategies de scaling" (32-value blocks, E8M0 power-of-two scale).
//
// Work split: a "unit" is 16 consecutive bf16 values of a row (32 bytes in,
// 8 bytes of packed codes out).  One thread owns one unit per iteration: an
// NVFP4 block is one unit, an MXFP4 block is a pair of adjacent lanes that
// combine their maxima with one shuffle.  Consecutive lanes own consecutive
// units, so the loads (2 x 16 B per lane) and the 8-byte code stores of a
// warp are contiguous.  All floating-point steps use explicitly rounded
// intrinsics (no contraction), one IEEE binary32 rounding per step.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Largest bf16 magnitude (as 15-bit pattern) of a packed bf16x2 word; for
// finite values the bit pattern orders like the magnitude.
__device__ __forceinline__ unsigned mag2(unsigned w) { return w & 0x7FFF7FFFu; }

__device__ __forceinline__ unsigned max_u16x2(unsigned a, unsigned b) { return __vmaxu2(a, b); }

__device__ __forceinline__ unsigned fold_u16x2(unsigned m) { return max(m & 0xFFFFu, m >> 16); }

__device__ __forceinline__ float bf16_lo(unsigned w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(unsigned w) { return __uint_as_float(w & 0xFFFF0000u); }

// E4M3 (satfinite, round to nearest even) of a non-negative float.
__device__ __forceinline__ unsigned to_e4m3(float v) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// Exact value of a non-negative E4M3 code (never NaN here: the encoder
// saturates at 0x7E).
__device__ __forceinline__ float e4m3_value(unsigned c) {
  const unsigned e = c >> 3, m = c & 7u;
  if (e == 0) return __uint2float_rn(m) * 0.001953125f;          // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));         // (8+m) 2^(e-10)
}

// Eight values -> eight E2M1 nibbles (value i in nibble i), round to
// nearest even with saturation to 6.
__device__ __forceinline__ unsigned to_e2m1x8(float v0, float v1, float v2, float v3,
                                              float v4, float v5, float v6, float v7) {
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
// a negative input always carries its sign, also when it rounds to zero.
__device__ __forceinline__ unsigned sign_nibbles(unsigned w0, unsigned w1, unsigned w2,
                                                 unsigned w3) {
  auto s = [](unsigned w) { return ((w >> 12) & 0x8u) | ((w >> 24) & 0x80u); };
  return s(w0) | s(w1) << 8 | s(w2) << 16 | s(w3) << 24;
}

// 8 bf16 (4 words) times r -> 8 packed codes.
__device__ __forceinline__ unsigned quant8(unsigned w0, unsigned w1, unsigned w2, unsigned w3,
                                           float r) {
  unsigned q = to_e2m1x8(__fmul_rn(bf16_lo(w0), r), __fmul_rn(bf16_hi(w0), r),
                         __fmul_rn(bf16_lo(w1), r), __fmul_rn(bf16_hi(w1), r),
                         __fmul_rn(bf16_lo(w2), r), __fmul_rn(bf16_hi(w2), r),
                         __fmul_rn(bf16_lo(w3), r), __fmul_rn(bf16_hi(w3), r));
  return q | sign_nibbles(w0, w1, w2, w3);
}

// floor(log2(b)) of a positive finite float from its bits.
__device__ __forceinline__ int floor_log2(float b) {
  const unsigned u = __float_as_uint(b);
  const int ex = static_cast<int>((u >> 23) & 0xFFu);
  if (ex != 0) return ex - 127;
  return (31 - __clz(u & 0x7FFFFFu)) - 149;
}

// Byte offset of scale (row r, column c) in the MMA-consumable order.
__device__ __forceinline__ long long mma_scale_offset(long long r, int c, int ncb) {
  const long long atom = (r >> 7) * ncb + (c >> 2);
  const int rr = static_cast<int>(r & 127);
  return atom * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3);
}

// Global scale from the partial maxima of the amax pass (DYNAMIC), or the
// caller's value (STATIC).  g = amax / 2688, 1 for an all-zero tensor.
__device__ float global_scale(int dynamic, const float* g, const unsigned* partial,
                              int n_partial) {
  if (!dynamic) return *g;
  __shared__ unsigned red[kThreads / 32];
  unsigned m = 0;
  for (int i = threadIdx.x; i < n_partial; i += blockDim.x) m = max(m, partial[i]);
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) m = max(m, red[i]);
  const float amax = __uint_as_float(m << 16);
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// ------------------------------------------------------------- amax pass

__global__ void __launch_bounds__(kThreads) amax_kernel(const uint4* __restrict__ x,
                                                        long long n_vec,
                                                        unsigned* __restrict__ partial) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  unsigned m0 = 0, m1 = 0;
  for (; i + 3 * stride < n_vec; i += 4 * stride) {
    const uint4 a = ld_stream(x + i), b = ld_stream(x + i + stride);
    const uint4 c = ld_stream(x + i + 2 * stride), d = ld_stream(x + i + 3 * stride);
    m0 = max_u16x2(m0, max_u16x2(max_u16x2(mag2(a.x), mag2(a.y)), max_u16x2(mag2(a.z), mag2(a.w))));
    m1 = max_u16x2(m1, max_u16x2(max_u16x2(mag2(b.x), mag2(b.y)), max_u16x2(mag2(b.z), mag2(b.w))));
    m0 = max_u16x2(m0, max_u16x2(max_u16x2(mag2(c.x), mag2(c.y)), max_u16x2(mag2(c.z), mag2(c.w))));
    m1 = max_u16x2(m1, max_u16x2(max_u16x2(mag2(d.x), mag2(d.y)), max_u16x2(mag2(d.z), mag2(d.w))));
  }
  for (; i < n_vec; i += stride) {
    const uint4 a = ld_stream(x + i);
    m0 = max_u16x2(m0, max_u16x2(max_u16x2(mag2(a.x), mag2(a.y)), max_u16x2(mag2(a.z), mag2(a.w))));
  }
  unsigned m = fold_u16x2(max_u16x2(m0, m1));
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ unsigned red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned r = 0;
    for (int w = 0; w < kThreads / 32; ++w) r = max(r, red[w]);
    partial[blockIdx.x] = r;
  }
}

// -------------------------------------------------------- quantize pass

template <int FMT, int LAYOUT>
__global__ void __launch_bounds__(kThreads) quantize_kernel(QuantArgs a, long long units,
                                                            int upr, int nsf, int ncb,
                                                            long long pad_a, long long pad_b) {
  const float g = (FMT == 0) ? global_scale(a.dynamic, a.g, a.partial, a.n_partial) : 1.0f;
  if (FMT == 0 && a.dynamic && blockIdx.x == 0 && threadIdx.x == 0) *a.g = g;
  const float six_g = __fmul_rn(6.0f, g);

  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  uint2* __restrict__ codes = reinterpret_cast<uint2*>(a.codes);
  uint8_t* __restrict__ scales = a.scales;
  const int lane = threadIdx.x & 31;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  // every lane of a warp runs the same number of iterations (MXFP4 pairs
  // exchange their maxima with a full-warp shuffle)
  for (long long base = static_cast<long long>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
       base < units; base += stride) {
    const long long u = base + lane;
    const bool active = u < units;
    uint4 p = make_uint4(0, 0, 0, 0), q = make_uint4(0, 0, 0, 0);
    if (active) {
      p = ld_stream(x + u * 16);
      q = ld_stream(x + u * 16 + 8);
    }
    unsigned m = fold_u16x2(max_u16x2(max_u16x2(max_u16x2(mag2(p.x), mag2(p.y)),
                                                max_u16x2(mag2(p.z), mag2(p.w))),
                                      max_u16x2(max_u16x2(mag2(q.x), mag2(q.y)),
                                                max_u16x2(mag2(q.z), mag2(q.w)))));
    unsigned sbyte;
    uint2 packed;
    if (FMT == 0) {
      const float b = __uint_as_float(m << 16);
      sbyte = to_e4m3(__fdiv_rn(b, six_g));
      const float sv = e4m3_value(sbyte);
      if (sv == 0.0f) {
        packed = make_uint2(0, 0);
      } else {
        const float r = __frcp_rn(__fmul_rn(sv, g));
        packed = make_uint2(quant8(p.x, p.y, p.z, p.w, r), quant8(q.x, q.y, q.z, q.w, r));
      }
    } else {
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      const float b = __uint_as_float(m << 16);
      int e = (b == 0.0f) ? -127 : floor_log2(b) - 2;
      e = max(-127, min(127, e));
      sbyte = static_cast<unsigned>(e + 127);
      const float r = __uint_as_float(static_cast<unsigned>(127 - e) << 23);   // 2^-e
      packed = make_uint2(quant8(p.x, p.y, p.z, p.w, r), quant8(q.x, q.y, q.z, q.w, r));
    }
    if (active) {
      codes[u] = packed;
      const long long row = u / upr;
      const int j = static_cast<int>(u - row * upr);
      if (FMT == 0 || (j & 1) == 0) {
        const int c = (FMT == 0) ? j : (j >> 1);
        const long long off = (LAYOUT == 1) ? row * nsf + c : mma_scale_offset(row, c, ncb);
        scales[off] = static_cast<uint8_t>(sbyte);
      }
    }
  }
  if (LAYOUT == 0) {
    // zero the padding of the MMA order: columns [nsf, 4 ncb) of real rows,
    // then every column of rows [rows, rows padded to 128)
    const long long total = pad_a + pad_b;
    const int padc = 4 * ncb - nsf;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += stride) {
      long long r;
      int c;
      if (i < pad_a) {
        r = i / padc;
        c = nsf + static_cast<int>(i - r * padc);
      } else {
        const long long k = i - pad_a;
        r = a.rows + k / (4 * ncb);
        c = static_cast<int>(k % (4 * ncb));
      }
      scales[mma_scale_offset(r, c, ncb)] = 0;
    }
  }
}

}  // namespace

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t launch_amax(const void* x, long long n, unsigned* partial, int* n_used,
                        cudaStream_t s) {
  const long long n_vec = n / 8;
  long long want = (n_vec + kThreads * 4 - 1) / (kThreads * 4);
  int blocks = static_cast<int>(std::min<long long>(want, static_cast<long long>(sm_count()) * 4));
  blocks = std::max(1, std::min(blocks, kAmaxSlots));
  amax_kernel<<<blocks, kThreads, 0, s>>>(static_cast<const uint4*>(x), n_vec, partial);
  *n_used = blocks;
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t s) {
  const int upr = a.K / 16;
  const long long units = a.rows * upr;
  const int nsf = nsf_of(a.K, a.fmt);
  const int ncb = ncb_of(nsf);
  long long pad_a = 0, pad_b = 0;
  if (a.layout == 0) {
    pad_a = a.rows * (4 * ncb - nsf);
    pad_b = (rows_pad128(a.rows) - a.rows) * 4 * ncb;
  }
  const long long work = std::max(units, pad_a + pad_b);
  long long want = (work + kThreads - 1) / kThreads;
  const int blocks = static_cast<int>(
      std::max<long long>(1, std::min<long long>(want, static_cast<long long>(sm_count()) * 8)));
  if (a.fmt == 0) {
    if (a.layout == 0)
      quantize_kernel<0, 0><<<blocks, kThreads, 0, s>>>(a, units, upr, nsf, ncb, pad_a, pad_b);
    else
      quantize_kernel<0, 1><<<blocks, kThreads, 0, s>>>(a, units, upr, nsf, ncb, pad_a, pad_b);
  } else {
    if (a.layout == 0)
      quantize_kernel<1, 0><<<blocks, kThreads, 0, s>>>(a, units, upr, nsf, ncb, pad_a, pad_b);
    else
      quantize_kernel<1, 1><<<blocks, kThreads, 0, s>>>(a, units, upr, nsf, ncb, pad_a, pad_b);
  }
  return cudaGetLastError();
}

}  // namespace fp4
