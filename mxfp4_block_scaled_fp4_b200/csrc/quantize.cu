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
#include <atomic>

#include "internal.h"
#include "codec.cuh"
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

// 32 contiguous bytes of a lane: one 256-bit load when `wide` (the tensor is
// 32-byte aligned), else two 16-byte loads.  A warp's 16-byte loads at a
// lane stride above 16 bytes each touch part of every sector, and the next
// load refetches them from L2 (no L1 allocation); the 256-bit load reads a
// lane's sectors once.  Measured on B200 it pays where a lane reads 64
// contiguous bytes (the 32-rotation's blocks: 8192 x 16384 MXFP4 + Hadamard-32
// 67.6 -> 63.5 us) and not at 32 (the 16-value units: 2-6% slower), so only
// the block pass uses it.
__device__ __forceinline__ void ld_stream32(const void* p, bool wide, uint4& a, uint4& b) {
  if (wide) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z),
                   "=r"(b.w)
                 : "l"(p));
  } else {
    a = ld_stream(p);
    b = ld_stream(static_cast<const uint4*>(p) + 1);
  }
}

// Byte offset of scale (row r, column c) in the MMA-consumable order.
__device__ __forceinline__ long long mma_scale_offset(long long r, int c, int ncb) {
  const long long atom = (r >> 7) * ncb + (c >> 2);
  const int rr = static_cast<int>(r & 127);
  return atom * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3);
}

// Global scale from the partial maxima of the amax pass (DYNAMIC), or the
// caller's value (STATIC).  g = amax / 2688, 1 for an all-zero tensor.
// self_amax: the maximum over the whole tensor x (n_vec 16-byte vectors)
// instead of the partial maxima (small tensors; 4 loads in flight a thread).
// With a rotation (ROT = 16 or 32) the maximum is over the rotated values
// and the partial maxima are binary32 magnitude bits; without, bf16 bits.
// A non-finite input is reported in `status` and the maximum clamped to the
// largest finite value (amax_checked), so g stays finite.
template <int ROT>
__device__ float global_scale(int dynamic, const float* g, const unsigned* partial,
                              int n_partial, int self_amax, const uint4* x, long long n_vec,
                              unsigned* status, float rot_scale) {
  if (!dynamic) return *g;
  __shared__ unsigned red[kThreads / 32];
  unsigned m = 0;
  if (self_amax) {
    if (ROT == 0) {
      for (long long i = threadIdx.x; i < n_vec; i += 4 * blockDim.x) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const long long k = i + j * blockDim.x;
          v[j] = (k < n_vec) ? ld_stream(x + k) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) m = max_u16x2(m, mag_max8(v[j]));
      }
      m = fold_u16x2(m);
    } else {
      // units of 16 values; whole warps iterate together (lane pairs)
      const long long n_units = n_vec / 2;
      for (long long base = 0; base < n_units; base += blockDim.x) {
        const long long u = base + threadIdx.x;
        const uint4 p = (u < n_units) ? ld_stream(x + 2 * u) : make_uint4(0, 0, 0, 0);
        const uint4 q = (u < n_units) ? ld_stream(x + 2 * u + 1) : make_uint4(0, 0, 0, 0);
        float f[16];
        unpack16(p, q, f);
        rotate_unit<ROT>(f, rot_scale, (threadIdx.x & 1) != 0);
        m = max(m, mag_max16(f));
      }
    }
  } else {
    for (int i = threadIdx.x; i < n_partial; i += blockDim.x) m = max(m, partial[i]);
  }
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) m = max(m, red[i]);
  float amax;
  if (ROT == 0) {
    // one CTA reports a non-finite input; every CTA clamps alike
    if (m > kBf16MaxFinite) m = (blockIdx.x == 0 && threadIdx.x == 0) ? amax_checked(m, status)
                                                                        : kBf16MaxFinite;
    amax = __uint_as_float(m << 16);
  } else {
    if (m > kF32MaxFinite) m = (blockIdx.x == 0 && threadIdx.x == 0) ? amax_checked_f32(m, status)
                                                                       : kF32MaxFinite;
    amax = __uint_as_float(m);
  }
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// ------------------------------------------------------------- amax pass

// Each warp reads a slab of 4 x 32 consecutive 16-byte vectors per
// iteration, all four loads in flight before any compute.
__global__ void __launch_bounds__(kThreads, 4) amax_kernel(const uint4* __restrict__ x,
                                                           long long n_vec,
                                                           unsigned* __restrict__ partial) {
  // In a programmatic-dependent-launch chain the next kernel may launch now
  // (this pass writes nothing but its own partial maxima, which only the
  // quantize pass reads, after its griddepcontrol.wait); the input is read
  // only after the previous kernel finished.  Without such a launch both are
  // no-ops.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long n_slabs = (n_vec + 127) / 128;
  const long long gwarp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  unsigned m = 0;
  for (long long t = gwarp; t < n_slabs; t += nwarps) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long i = t * 128 + j * 32 + lane;
      v[j] = (i < n_vec) ? ld_stream(x + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) m = max_u16x2(m, mag_max8(v[j]));
  }
  m = fold_u16x2(m);
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

// The amax pass over rotated values: warps take slabs of 4 x 32 units of 16
// values (every lane issues its 8 loads first), rotate each unit and keep
// the largest magnitude (binary32 bits).  The 32-rotation gives each lane a
// whole 32-value block instead (2 x 32 blocks per slab, rotate_block32).
template <int ROT>
__global__ void __launch_bounds__(kThreads, 4) amax_rot_kernel(const uint4* __restrict__ x,
                                                               long long n_units, float scale,
                                                               unsigned* __restrict__ partial) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long n_slabs = (n_units + 127) / 128;
  const long long gwarp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  unsigned m = 0;
  for (long long t = gwarp; t < n_slabs; t += nwarps) {
    if (ROT == 32) {
      const long long n_blocks = n_units >> 1;
      uint4 v[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const long long b = t * 64 + j * 32 + lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) v[j][k] = (b < n_blocks) ? ld_stream(x + 4 * b + k) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float lo[16], hi[16];
        unpack16(v[j][0], v[j][1], lo);
        unpack16(v[j][2], v[j][3], hi);
        rotate_block32(lo, hi, scale);
        m = max(m, max(mag_max16(lo), mag_max16(hi)));
      }
    } else {
      uint4 v[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const long long u = t * 128 + j * 32 + lane;
        if (u < n_units) {
          v[j][0] = ld_stream(x + 2 * u);
          v[j][1] = ld_stream(x + 2 * u + 1);
        } else {
          v[j][0] = v[j][1] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float f[16];
        unpack16(v[j][0], v[j][1], f);
        rotate_unit<ROT>(f, scale, (lane & 1) != 0);
        m = max(m, mag_max16(f));
      }
    }
  }
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

// The macro-block scaling row pass: one warp per row (grid-stride over the
// rows), eight 16-byte loads in flight per lane; sigma of the row's largest
// magnitude.  A non-finite input is reported and clamped as in the DYNAMIC
// global scale.
__global__ void __launch_bounds__(kThreads, 4) mbs_rows_kernel(const uint16_t* __restrict__ x,
                                                               long long rows, int K,
                                                               float* __restrict__ sigma,
                                                               unsigned* status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const long long gwarp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const int n_vec = K / 8;
  for (long long r = gwarp; r < rows; r += nwarps) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * K);
    unsigned m = 0;
    for (int v = lane; v < n_vec; v += 256) {
      uint4 t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = (v + 32 * j < n_vec) ? ld_stream(xr + v + 32 * j) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 8; ++j) m = max_u16x2(m, mag_max8(t[j]));
    }
    m = fold_u16x2(m);
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) {
      if (m > kBf16MaxFinite) m = amax_checked(m, status);
      sigma[r] = mbs_sigma(__uint_as_float(m << 16));
    }
  }
}

// -------------------------------------------------------- quantize pass

// n / d for 32-bit n by multiply-high (Granlund & Montgomery, "Division by
// invariant integers using multiplication", 1994): l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, q = (mulhi(n, m) + n) >> l; d = 1 is
// m = 0, l = 0.
struct FastDiv {
  unsigned m;
  unsigned l;
};
__device__ __forceinline__ unsigned fast_div(unsigned n, FastDiv f) {
  return static_cast<unsigned>((static_cast<unsigned long long>(__umulhi(n, f.m)) + n) >> f.l);
}

// Units [u_begin, u_end) in slabs of 4 x 32 consecutive units: warp w of
// nwarps takes slabs w, w + nwarps, ... (from the end when `reverse`), and
// every lane issues its 8 loads (4 units x 32 bytes) before computing.
template <int FMT, int LAYOUT, int ROT>
__device__ __forceinline__ void quantize_units(const QuantArgs& a, long long u_begin,
                                               long long u_end, long long w, long long nwarps,
                                               bool reverse, int upr, FastDiv upr_div, int nsf,
                                               int ncb, float six_g, float y6, bool fast_b,
                                               const float* r_tab) {
  const bool big = u_end > 0xFFFFFFFFll;   // unit indices beyond 32 bits: plain division
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  uint2* __restrict__ codes = reinterpret_cast<uint2*>(a.codes);
  uint8_t* __restrict__ scales = a.scales;
  const int lane = threadIdx.x & 31;
  const long long n_slabs = (u_end - u_begin + 127) / 128;
  for (long long t = w; t < n_slabs; t += nwarps) {
    const long long slab = reverse ? n_slabs - 1 - t : t;
    uint4 xs[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long u = u_begin + slab * 128 + j * 32 + lane;
      if (u < u_end) {
        xs[j][0] = ld_stream(x + u * 16);
        xs[j][1] = ld_stream(x + u * 16 + 8);
      } else {
        xs[j][0] = xs[j][1] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long u = u_begin + slab * 128 + j * 32 + lane;
      const uint4 p = xs[j][0], q = xs[j][1];
      unsigned sbyte;
      uint2 packed;
      float r;
      if (ROT == 1) {
        // macro-block scaling (MXFP4): x' = RN(x * RN(1 / sigma_row)), then
        // the block exponent from the largest |x'| of the lane pair
        const long long urow = (u < u_end) ? u : u_begin;
        const long long row =
            big ? urow / upr : static_cast<long long>(fast_div(static_cast<unsigned>(urow), upr_div));
        const float rho = __frcp_rn(a.mbs_sigma[row]);
        float f[16];
        unpack16(p, q, f);
        const unsigned long long R = f2(rho, rho);
#pragma unroll
        for (int k = 0; k < 8; ++k) f2_split(mul_f2(f2(f[2 * k], f[2 * k + 1]), R), f[2 * k], f[2 * k + 1]);
        unsigned m = mag_max16(f);
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        sbyte = mxfp4_scale_f32(m, a.rule, &r);
        packed = make_uint2(quant8_f32(f, r), quant8_f32(f + 8, r));
      } else if (ROT == 0) {
        unsigned m = fold_u16x2(max_u16x2(mag_max8(p), mag_max8(q)));
        if (FMT == 0) {
          sbyte = nvfp4_scale_byte(m, six_g, y6, fast_b);
          r = r_tab[sbyte & 127u];
          packed = (r == 0.0f) ? make_uint2(0, 0)
                               : make_uint2(quant8(p.x, p.y, p.z, p.w, r), quant8(q.x, q.y, q.z, q.w, r));
        } else {
          m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));   // 32-value block = lane pair
          sbyte = mxfp4_scale_f32(m << 16, a.rule, &r);
          packed = make_uint2(quant8(p.x, p.y, p.z, p.w, r), quant8(q.x, q.y, q.z, q.w, r));
        }
      } else if (ROT >= 16) {
        // the unit's rotated values (a 32-value rotation pairs lanes 2i, 2i+1:
        // their units are the two halves of one 32-value block)
        float f[16];
        unpack16(p, q, f);
        rotate_unit<ROT>(f, a.rot_scale, (lane & 1) != 0);
        unsigned m = mag_max16(f);
        if (FMT == 0) {
          sbyte = nvfp4_scale_byte_f32(m, six_g, y6, fast_b);
          r = r_tab[sbyte & 127u];
          packed = (r == 0.0f) ? make_uint2(0, 0) : make_uint2(quant8_f32(f, r), quant8_f32(f + 8, r));
        } else {
          m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
          sbyte = mxfp4_scale_f32(m, a.rule, &r);
          packed = make_uint2(quant8_f32(f, r), quant8_f32(f + 8, r));
        }
      }
      if (u < u_end) {
        codes[u] = packed;
        const long long row =
            big ? u / upr : static_cast<long long>(fast_div(static_cast<unsigned>(u), upr_div));
        const int jj = static_cast<int>(u - row * upr);
        if (FMT == 0 || (jj & 1) == 0) {
          const int c = (FMT == 0) ? jj : (jj >> 1);
          const long long off = (LAYOUT == 1) ? row * nsf + c : mma_scale_offset(row, c, ncb);
          scales[off] = static_cast<uint8_t>(sbyte);
        }
      }
    }
  }
}

// The 32-rotation's quantize pass with a whole 32-value block per lane
// (units 2b, 2b + 1 of block b): the rotation runs in the thread
// (rotate_block32, no lane exchange), then the block's scale(s) and codes.
// Blocks [u_begin / 2, u_end / 2) in slabs of 2 x 32 blocks per warp step
// (128 units, as quantize_units), 4 loads per lane and block.
template <int FMT, int LAYOUT>
__device__ __forceinline__ void quantize_blocks32(const QuantArgs& a, long long u_begin,
                                                  long long u_end, long long w, long long nwarps,
                                                  bool reverse, int upr, FastDiv upr_div, int nsf,
                                                  int ncb, float six_g, float y6, bool fast_b,
                                                  const float* r_tab) {
  const bool big = u_end > 0xFFFFFFFFll;
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  uint4* __restrict__ codes = reinterpret_cast<uint4*>(a.codes);
  uint8_t* __restrict__ scales = a.scales;
  const int lane = threadIdx.x & 31;
  const long long b_begin = u_begin >> 1, b_end = u_end >> 1;
  const long long n_slabs = (b_end - b_begin + 63) / 64;
  for (long long t = w; t < n_slabs; t += nwarps) {
    const long long slab = reverse ? n_slabs - 1 - t : t;
    uint4 xs[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const long long b = b_begin + slab * 64 + j * 32 + lane;
      if (b < b_end) {
        ld_stream32(x + b * 32, a.wide != 0, xs[j][0], xs[j][1]);
        ld_stream32(x + b * 32 + 16, a.wide != 0, xs[j][2], xs[j][3]);
      } else {
        xs[j][0] = xs[j][1] = xs[j][2] = xs[j][3] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const long long b = b_begin + slab * 64 + j * 32 + lane;
      float lo[16], hi[16];
      unpack16(xs[j][0], xs[j][1], lo);
      unpack16(xs[j][2], xs[j][3], hi);
      rotate_block32(lo, hi, a.rot_scale);
      const unsigned m0 = mag_max16(lo), m1 = mag_max16(hi);
      unsigned s0, s1 = 0u;
      uint4 packed;
      if (FMT == 0) {
        s0 = nvfp4_scale_byte_f32(m0, six_g, y6, fast_b);
        s1 = nvfp4_scale_byte_f32(m1, six_g, y6, fast_b);
        const float r0 = r_tab[s0 & 127u], r1 = r_tab[s1 & 127u];
        packed.x = r0 == 0.0f ? 0u : quant8_f32(lo, r0);
        packed.y = r0 == 0.0f ? 0u : quant8_f32(lo + 8, r0);
        packed.z = r1 == 0.0f ? 0u : quant8_f32(hi, r1);
        packed.w = r1 == 0.0f ? 0u : quant8_f32(hi + 8, r1);
      } else {
        float r;
        s0 = mxfp4_scale_f32(max(m0, m1), a.rule, &r);
        packed = make_uint4(quant8_f32(lo, r), quant8_f32(lo + 8, r), quant8_f32(hi, r),
                            quant8_f32(hi + 8, r));
      }
      if (b < b_end) {
        codes[b] = packed;   // units 2b, 2b + 1
        const long long u = 2 * b;
        const long long row =
            big ? u / upr : static_cast<long long>(fast_div(static_cast<unsigned>(u), upr_div));
        const int jj = static_cast<int>(u - row * upr);   // even: a block never spans rows
        if (FMT == 0) {
          // scale columns jj, jj + 1: adjacent bytes, an aligned 16-bit word
          // (in the MMA order jj % 4 is 0 or 2; row-major rows hold an even
          // number of scales)
          const long long off = (LAYOUT == 1) ? row * nsf + jj : mma_scale_offset(row, jj, ncb);
          *reinterpret_cast<uint16_t*>(scales + off) = static_cast<uint16_t>(s0 | (s1 << 8));
        } else {
          const int c = jj >> 1;
          const long long off = (LAYOUT == 1) ? row * nsf + c : mma_scale_offset(row, c, ncb);
          scales[off] = static_cast<uint8_t>(s0);
        }
      }
    }
  }
}

// MMA order: zero the padding, columns [nsf, 4 ncb) of real rows, then every
// column of rows [rows, rows padded to 128); items i = first, first + stride...
__device__ __forceinline__ void zero_mma_padding(const QuantArgs& a, long long pad_a,
                                                 long long pad_b, int nsf, int ncb,
                                                 long long first, long long stride) {
  const long long total = pad_a + pad_b;
  const int padc = 4 * ncb - nsf;
  for (long long i = first; i < total; i += stride) {
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
    a.scales[mma_scale_offset(r, c, ncb)] = 0;
  }
}

// The full-chip quantize pass.  With a DYNAMIC global scale the slabs are
// walked from the end, so the first ones are still in L2 from the amax pass.
template <int FMT, int LAYOUT, int ROT>
__global__ void __launch_bounds__(kThreads, 4) quantize_kernel(QuantArgs a, long long units,
                                                               int upr, FastDiv upr_div, int nsf,
                                                               int ncb, long long pad_a,
                                                               long long pad_b) {
  if (a.release_early) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float g = (FMT == 0) ? global_scale<ROT>(a.dynamic, a.g, a.partial, a.n_partial,
                                                 a.self_amax, static_cast<const uint4*>(a.x),
                                                 units * 2, a.status, a.rot_scale)
                             : 1.0f;
  if (FMT == 0 && a.dynamic && blockIdx.x == 0 && threadIdx.x == 0) *a.g = g;
  const float six_g = __fmul_rn(6.0f, g);
  const float y6 = __frcp_rn(six_g);
  const bool fast_b = six_g >= 0x1p-40f && six_g <= 0x1p40f;
  // r = RN(1 / RN(s g)) for every scale byte this pass can produce (s <= 0x7F)
  __shared__ float r_tab[128];
  if (FMT == 0) {
    for (int i = threadIdx.x; i < 128; i += blockDim.x) r_tab[i] = nvfp4_recip(i, g);
    __syncthreads();
  }
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long gwarp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (ROT == 32)
    quantize_blocks32<FMT, LAYOUT>(a, 0, units, gwarp, stride >> 5, a.dynamic != 0, upr, upr_div,
                                   nsf, ncb, six_g, y6, fast_b, r_tab);
  else
    quantize_units<FMT, LAYOUT, ROT>(a, 0, units, gwarp, stride >> 5, a.dynamic != 0, upr,
                                     upr_div, nsf, ncb, six_g, y6, fast_b, r_tab);
  if (LAYOUT == 0)
    zero_mma_padding(a, pad_a, pad_b, nsf, ncb,
                     static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x, stride);
}

}  // namespace

int sm_count() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {
// Launch with the programmatic-stream-serialization attribute when pdl is set.
template <typename... Args>
cudaError_t launch_k(void (*k)(Args...), int blocks, bool pdl, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? at : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, args...);
}
}  // namespace

cudaError_t launch_amax_rot(const void* x, long long rows, int K, int rot, float scale,
                            unsigned* partial, int* n_used, cudaStream_t s, bool pdl) {
  const long long n_units = rows * (K / 16);
  long long want = (n_units + kThreads * 4 - 1) / (kThreads * 4);
  int blocks = static_cast<int>(std::min<long long>(want, static_cast<long long>(sm_count()) * 4));
  blocks = std::max(1, std::min(blocks, kAmaxSlots));
  *n_used = blocks;
  auto kern = (rot == 32) ? amax_rot_kernel<32> : amax_rot_kernel<16>;
  const cudaError_t e = launch_k(kern, blocks, pdl, s, static_cast<const uint4*>(x), n_units,
                                 scale, partial);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_amax(const void* x, long long n, unsigned* partial, int* n_used,
                        cudaStream_t s, bool pdl) {
  const long long n_vec = n / 8;
  long long want = (n_vec + kThreads * 4 - 1) / (kThreads * 4);
  int blocks = static_cast<int>(std::min<long long>(want, static_cast<long long>(sm_count()) * 4));
  blocks = std::max(1, std::min(blocks, kAmaxSlots));
  *n_used = blocks;
  const cudaError_t e = launch_k(amax_kernel, blocks, pdl, s, static_cast<const uint4*>(x), n_vec,
                                 partial);
  return e != cudaSuccess ? e : cudaGetLastError();
}

namespace {

struct QuantGeom {
  int upr, nsf, ncb;
  long long units, pad_a, pad_b;
  FastDiv fd;
};

QuantGeom quant_geom(const QuantArgs& a) {
  QuantGeom q;
  q.upr = a.K / 16;
  q.units = a.rows * q.upr;
  q.nsf = nsf_of(a.K, a.fmt);
  q.ncb = ncb_of(q.nsf);
  q.pad_a = q.pad_b = 0;
  if (a.layout == 0) {
    q.pad_a = a.rows * (4 * q.ncb - q.nsf);
    q.pad_b = a.zero_pad_rows ? (rows_pad128(a.rows) - a.rows) * 4 * q.ncb : 0;
  }
  q.fd = FastDiv{0u, 0u};
  if (q.upr > 1) {
    unsigned l = 0;
    while ((1ull << l) < static_cast<unsigned long long>(q.upr)) ++l;
    q.fd.l = l;
    q.fd.m = static_cast<unsigned>(((1ull << 32) * ((1ull << l) - static_cast<unsigned long long>(q.upr))) /
                                       static_cast<unsigned long long>(q.upr) + 1);
  }
  return q;
}

}  // namespace

cudaError_t launch_quantize(const QuantArgs& a_in, cudaStream_t s, bool pdl) {
  QuantArgs a = a_in;
  if (!a.status && !(a.status = watchdog_ptr())) return cudaErrorInvalidSymbol;
  // rows are 64-byte multiples (K % 32 == 0): the base decides the alignment
  a.wide = (reinterpret_cast<uintptr_t>(a.x) % 32) == 0 ? 1 : 0;
  const QuantGeom q = quant_geom(a);
  const long long want = std::max((q.units + kThreads * 4 - 1) / (kThreads * 4),
                                  (q.pad_a + q.pad_b + kThreads - 1) / kThreads);
  const int blocks = static_cast<int>(
      std::max<long long>(1, std::min<long long>(want, static_cast<long long>(sm_count()) * 4)));
  using Kern = void (*)(QuantArgs, long long, int, FastDiv, int, int, long long, long long);
  if (a.mbs_sigma) {   // MXFP4 with macro-block scaling
    const Kern k = a.layout == 0 ? quantize_kernel<1, 0, 1> : quantize_kernel<1, 1, 1>;
    const cudaError_t e =
        launch_k(k, blocks, pdl, s, a, q.units, q.upr, q.fd, q.nsf, q.ncb, q.pad_a, q.pad_b);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  static const Kern table[3][2][2] = {
      {{quantize_kernel<0, 0, 0>, quantize_kernel<0, 1, 0>},
       {quantize_kernel<1, 0, 0>, quantize_kernel<1, 1, 0>}},
      {{quantize_kernel<0, 0, 16>, quantize_kernel<0, 1, 16>},
       {quantize_kernel<1, 0, 16>, quantize_kernel<1, 1, 16>}},
      {{quantize_kernel<0, 0, 32>, quantize_kernel<0, 1, 32>},
       {quantize_kernel<1, 0, 32>, quantize_kernel<1, 1, 32>}}};
  const int ri = a.rot == 32 ? 2 : (a.rot == 16 ? 1 : 0);
  const Kern kern = table[ri][a.fmt != 0][a.layout != 0];
  const cudaError_t e =
      launch_k(kern, blocks, pdl, s, a, q.units, q.upr, q.fd, q.nsf, q.ncb, q.pad_a, q.pad_b);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_quantize_act(QuantArgs a, unsigned* partial, cudaStream_t s) {
  if (a.mbs_sigma) {
    // the row pass, then the quantize pass (each a programmatic dependent)
    if (!a.status && !(a.status = watchdog_ptr())) return cudaErrorInvalidSymbol;
    const long long warps_per_block = kThreads / 32;
    const int blocks = static_cast<int>(std::max<long long>(
        1, std::min<long long>((a.rows + warps_per_block - 1) / warps_per_block,
                               static_cast<long long>(sm_count()) * 4)));
    cudaError_t e = launch_k(mbs_rows_kernel, blocks, true, s, static_cast<const uint16_t*>(a.x),
                             a.rows, a.K, a.mbs_sigma, a.status);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_quantize(a, s, true);
  }
  if (a.dynamic && a.rows * a.K * 2 <= kSelfAmaxBytes) {
    a.self_amax = 1;
    return launch_quantize(a, s, true);
  }
  if (a.dynamic) {
    int used = 0;
    const cudaError_t e =
        a.rot ? launch_amax_rot(a.x, a.rows, a.K, a.rot, a.rot_scale, partial, &used, s, true)
              : launch_amax(a.x, a.rows * a.K, partial, &used, s, true);
    if (e != cudaSuccess) return e;
    a.partial = partial;
    a.n_partial = used;
  }
  return launch_quantize(a, s, true);
}

}  // namespace fp4
