// fused.cu -- small-M (decode) W4A4 path: the bf16 activation is quantized
// inside the GEMM kernel, never written to global memory in FP4 form.
//
// "FP4 n'existe pas", runtime survey: quantization, scaling, matmul and
// de-scaling fused in one launch; the small-M regime cuBLAS refuses:
// "Hardware FP4 inference for speech on Blackwell", section "Do the FP4
// tensor cores even engage?".  Same arithmetic as fp4_quantize_act followed
// by fp4_gemm (bit-identical codes and scales), up to FP32 summation order.
//
// Two launches per call:
//  prologue  (tiny) zeroes the split-K arrival counters and, for a DYNAMIC
//            global scale, writes one partial amax per CTA.  It lets the
//            main kernel launch right away (programmatic dependent launch),
//            so weight streaming starts while the amax is still running.
//  main      swap-AB: the weights are the 128-row "A" operand of
//            tcgen05.mma kind::mxf4nvf4 and the <= 32 activation rows are the
//            16- or 32-wide "B" operand.  Grid = N/128 weight tiles x S
//            split-K slices.  Per CTA:
//     warp 0     TMA: weight tiles (16 KiB per 256 K) + their scale atoms
//                through a 4-stage ring;
//     warp 1     MMA issuer;
//     warps 2-5  (a) after griddepcontrol.wait: global scale, then quantize
//                    the CTA's K slice of the activation into shared memory
//                    (128-byte swizzled K-major rows, the MMA's B layout) and
//                    its scales into tensor memory (tcgen05.st);
//                (b) stage each ring stage's weight scales into tensor
//                    memory; (c) epilogue: accumulator -> C (S = 1) or ->
//                    split-K partials; the last CTA of a tile sums the S
//                    partials in slice order (deterministic) and writes C.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int FBM = 128;                 // weight rows per tile
constexpr int FBK = 256;                 // K per ring stage
constexpr int FBK_BYTES = FBK / 2;
constexpr int FSTAGES = 4;
constexpr int FW_STAGE = FBM * FBK_BYTES;   // 16 KiB
constexpr int FSF_STAGE = 4 * 512;          // up to 4 scale atoms
constexpr int kMaxStepsPerSplit = 16;       // K slice <= 4096 per CTA
constexpr int kFusedThreads = 192;          // TMA, MMA, 4 worker warps
constexpr int kTargetCtas = 148;            // one CTA per B200 SM
constexpr int kPrologueThreads = 256;
constexpr int kMaxPrologueCtas = 148;
// Tensor-memory columns.  Every scale-factor address an MMA gets is a
// multiple of 4 columns (16 bytes), the alignment the passing GEMM uses: a
// fault was seen on B200 when activation scales sat at columns 4i + k.
constexpr uint32_t F_TMEM_COLS = 512;
constexpr uint32_t F_ACC_COL = 0;           // <= 32 fp32 columns
constexpr uint32_t F_SFA_COL = 32;          // weight scales: 16 columns per ring stage
constexpr uint32_t F_SFB_COL = 128;         // activation scales: 4 columns per scale word

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

struct Plan {
  int n_tiles, k_steps, splits, steps_max, nmma_n;
  size_t ws_partial_off, ws_counter_off, ws_sum_off, ws_bytes;
  int smem_bytes;
};

Plan make_plan(int M, int N, int K, int fmt) {
  Plan p{};
  p.n_tiles = (N + FBM - 1) / FBM;
  p.k_steps = (K + FBK - 1) / FBK;
  int s = (kTargetCtas + p.n_tiles - 1) / p.n_tiles;
  s = std::max(s, (p.k_steps + kMaxStepsPerSplit - 1) / kMaxStepsPerSplit);
  p.splits = std::max(1, std::min(s, p.k_steps));
  p.steps_max = (p.k_steps + p.splits - 1) / p.splits;
  p.nmma_n = M <= 16 ? 16 : 32;
  p.ws_partial_off = 0;
  p.ws_counter_off = align256(static_cast<size_t>(kMaxPrologueCtas) * sizeof(unsigned));
  p.ws_sum_off = p.ws_counter_off + align256(static_cast<size_t>(p.n_tiles) * sizeof(unsigned));
  const size_t sums = p.splits > 1 ? static_cast<size_t>(p.n_tiles) * p.splits * M * FBM * 4 : 0;
  p.ws_bytes = p.ws_sum_off + align256(sums);
  const int act_bytes = p.steps_max * p.nmma_n * FBK_BYTES;
  const int sf_scratch = p.nmma_n * p.steps_max * 16;
  p.smem_bytes = 1024 + FSTAGES * (FW_STAGE + FSF_STAGE) + act_bytes + sf_scratch + 256;
  (void)fmt;
  return p;
}

struct FParams {
  const uint16_t* a;
  const uint8_t* w_scales;
  const float* g_w;
  float* g_a;
  const unsigned* amax_partial;
  unsigned* counters;
  float* sums;
  void* C;
  long long ldc;
  int M, N, K;
  int dynamic, out_f32;
  int n_tiles, k_steps, splits, steps_max, nmma_n, ncb, n_partial;
  unsigned* watchdog;
};

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void workers_sync() {   // named barrier of the 4 worker warps
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ unsigned mag_max8(uint4 v) {
  unsigned m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                        __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return m;
}

// ---- element codecs (same rounding steps as the stand-alone quantizer)
__device__ __forceinline__ unsigned f_to_e4m3(float v) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}
__device__ __forceinline__ float f_e4m3_value(unsigned c) {
  const unsigned e = c >> 3, m = c & 7u;
  if (e == 0) return __uint2float_rn(m) * 0.001953125f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}
__device__ __forceinline__ unsigned f_e2m1x8(float v0, float v1, float v2, float v3, float v4,
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
__device__ __forceinline__ unsigned f_quant8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                             float r) {
  auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
  auto hi = [](uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); };
  auto sg = [](uint32_t w) { return ((w >> 12) & 0x8u) | ((w >> 24) & 0x80u); };
  const unsigned q = f_e2m1x8(__fmul_rn(lo(w0), r), __fmul_rn(hi(w0), r), __fmul_rn(lo(w1), r),
                              __fmul_rn(hi(w1), r), __fmul_rn(lo(w2), r), __fmul_rn(hi(w2), r),
                              __fmul_rn(lo(w3), r), __fmul_rn(hi(w3), r));
  return q | sg(w0) | sg(w1) << 8 | sg(w2) << 16 | sg(w3) << 24;
}
__device__ __forceinline__ int f_floor_log2(float b) {
  const unsigned u = __float_as_uint(b);
  const int ex = static_cast<int>((u >> 23) & 0xFFu);
  if (ex != 0) return ex - 127;
  return (31 - __clz(u & 0x7FFFFFu)) - 149;
}

// ------------------------------------------------------------ prologue

__global__ void __launch_bounds__(kPrologueThreads)
    fused_prologue_kernel(const uint4* __restrict__ a, long long n_vec, int dynamic,
                          unsigned* __restrict__ partial, unsigned* __restrict__ counters,
                          int n_counters) {
  grid_dep_launch();   // the main kernel may start streaming weights now
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_counters; i += gridDim.x * blockDim.x)
    counters[i] = 0;
  if (!dynamic) return;
  unsigned m = 0;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    m = __vmaxu2(m, mag_max8(ld_nc16(a + i)));
  m = max(m & 0xFFFFu, m >> 16);
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ unsigned red[kPrologueThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned r = 0;
    for (int w = 0; w < kPrologueThreads / 32; ++w) r = max(r, red[w]);
    partial[blockIdx.x] = r;
  }
}

// ---------------------------------------------------------------- main

template <int FMT>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_kernel(const __grid_constant__ CUtensorMap tm_w, const FParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;
  uint8_t* sSF = sW + FSTAGES * FW_STAGE;
  uint8_t* sAct = sSF + FSTAGES * FSF_STAGE;                 // 1024-aligned
  const int act_chunk = p.nmma_n * FBK_BYTES;                 // bytes per 256 K
  uint8_t* sScr = sAct + p.steps_max * act_chunk;             // activation scale bytes
  const int scr_row = p.steps_max * 16;                       // scale bytes per row
  uint64_t* bars = reinterpret_cast<uint64_t*>(sScr + p.nmma_n * scr_row);
  uint64_t* full = bars;
  uint64_t* empty = full + FSTAGES;
  uint64_t* sf_loaded = empty + FSTAGES;
  uint64_t* sf_full = sf_loaded + FSTAGES;
  uint64_t* act_ready = sf_full + FSTAGES;
  uint64_t* acc_full = act_ready + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / p.splits, split = blockIdx.x % p.splits;
  const int s_lo = static_cast<int>(static_cast<long long>(split) * p.k_steps / p.splits);
  const int s_hi = static_cast<int>(static_cast<long long>(split + 1) * p.k_steps / p.splits);
  const int n_steps = s_hi - s_lo;
  constexpr int kAtoms = (FMT == 0) ? 4 : 2;   // weight scale atoms per 256 K

  if (threadIdx.x == 0) {
    for (int s = 0; s < FSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_loaded[s], 1);
      mbar_init(&sf_full[s], 4);
    }
    mbar_init(act_ready, 4);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, F_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    uint32_t armed = 0, armed_parity = 0;
    for (int i = 0; i < n_steps; ++i) {
      const int stage = i % FSTAGES;
      const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
      if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER)) goto p_drain;
      {
        const int ks = s_lo + i;
        const int cb0 = ks * kAtoms;
        const int atoms = min(kAtoms, p.ncb - cb0);
        mbar_expect_tx(&sf_loaded[stage], static_cast<uint32_t>(atoms) * 512u);
        bulk_load(sSF + stage * FSF_STAGE,
                  p.w_scales + (static_cast<long long>(tile) * p.ncb + cb0) * 512,
                  static_cast<uint32_t>(atoms) * 512u, &sf_loaded[stage]);
        mbar_expect_tx(&full[stage], FW_STAGE);
        tma_load_2d(sW + stage * FW_STAGE, &tm_w, ks * FBK_BYTES, tile * FBM, &full[stage]);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
      }
    }
    goto p_done;
  p_drain:
    for (int s = 0; s < FSTAGES; ++s)
      if (armed & (1u << s)) {
        mbar_wait_drain(&sf_loaded[s], (armed_parity >> s) & 1u, p.watchdog);
        mbar_wait_drain(&full[s], (armed_parity >> s) & 1u, p.watchdog);
      }
  p_done:;
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    if (!mbar_wait(act_ready, 0, abort_flag, p.watchdog, WD_MMA_FULL)) goto m_drain;
    tc_fence_after();
    for (int i = 0; i < n_steps; ++i) {
      const int stage = i % FSTAGES;
      const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
      if (!mbar_wait(&full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL)) goto m_drain;
      if (!mbar_wait(&sf_full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL)) goto m_drain;
      tc_fence_after();
      {
        const int kglob = (s_lo + i) * FBK;
        const int n_mma = min(4, (p.K - kglob + 63) / 64);
        const uint32_t w_s = smem_u32(sW + stage * FW_STAGE);
        const uint32_t x_s = smem_u32(sAct + i * act_chunk);
        const uint32_t sfa = tmem + F_SFA_COL + stage * 16;
        for (int k = 0; k < n_mma; ++k) {
          const uint64_t ad = smem_desc(w_s + k * 32, 16, 1024, kLayoutSwizzle128B);
          const uint64_t bd = smem_desc(x_s + k * 32, 16, 1024, kLayoutSwizzle128B);
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          if (FMT == 0) {
            tc_mma_nvf4(tmem + F_ACC_COL, ad, bd, idesc_fp4(FBM, p.nmma_n, false, 0, 0),
                        sfa + 4 * k, tmem + F_SFB_COL + 4 * (4 * i + k), acc);
          } else {
            const uint32_t id = 2u * (k & 1);
            tc_mma_mxf4(tmem + F_ACC_COL, ad, bd, idesc_fp4(FBM, p.nmma_n, true, id, id),
                        sfa + 4 * (k >> 1), tmem + F_SFB_COL + 4 * (2 * i + (k >> 1)), acc);
          }
        }
      }
      tc_commit(&empty[stage]);
    }
    tc_commit(acc_full);
    goto m_done;
  m_drain:
    tc_commit(drain);
    mbar_wait_drain(drain, 0, p.watchdog);
  m_done:;
  } else if (warp >= 2) {
    // ------------------------------------------------------------ workers
    const int quarter = warp & 3;
    const int wt = threadIdx.x - 64;                 // 0..127
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    grid_dep_wait();                                 // prologue finished and visible
    // (a) global scale
    float g = 1.0f;
    if (FMT == 0) {
      if (p.dynamic) {
        __shared__ unsigned red[4];
        unsigned m = 0;
        for (int i = wt; i < p.n_partial; i += 128) m = max(m, p.amax_partial[i]);
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) red[quarter] = m;
        workers_sync();
        m = max(max(red[0], red[1]), max(red[2], red[3]));
        const float amax = __uint_as_float(m << 16);
        g = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
        if (blockIdx.x == 0 && wt == 0) *p.g_a = g;
      } else {
        g = *p.g_a;
      }
    }
    const float six_g = __fmul_rn(6.0f, g);
    // (a) quantize rows [0, nmma_n) x K slice into the MMA's B layout
    const int units_per_row = n_steps * 16;
    const int total = p.nmma_n * units_per_row;      // a multiple of 256
    for (int u = wt; u < total; u += 128) {
      const int m = u / units_per_row;
      const int ku = u - m * units_per_row;
      const int kg = s_lo * FBK + ku * 16;
      const bool live = m < p.M && kg < p.K;
      uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
      if (live) {
        const uint16_t* src = p.a + static_cast<long long>(m) * p.K + kg;
        x0 = ld_nc16(src);
        x1 = ld_nc16(src + 8);
      }
      unsigned mm = __vmaxu2(mag_max8(x0), mag_max8(x1));
      mm = max(mm & 0xFFFFu, mm >> 16);
      unsigned sbyte;
      uint2 q;
      if (FMT == 0) {
        sbyte = f_to_e4m3(__fdiv_rn(__uint_as_float(mm << 16), six_g));
        const float sv = f_e4m3_value(sbyte);
        if (sv == 0.0f) {
          q = make_uint2(0, 0);
        } else {
          const float r = __frcp_rn(__fmul_rn(sv, g));
          q = make_uint2(f_quant8(x0.x, x0.y, x0.z, x0.w, r), f_quant8(x1.x, x1.y, x1.z, x1.w, r));
        }
      } else {
        mm = max(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, 1));   // 32-value block = lane pair
        const float b = __uint_as_float(mm << 16);
        int e = (b == 0.0f) ? -127 : f_floor_log2(b) - 2;
        e = max(-127, min(127, e));
        sbyte = static_cast<unsigned>(e + 127);
        const float r = __uint_as_float(static_cast<unsigned>(127 - e) << 23);
        q = make_uint2(f_quant8(x0.x, x0.y, x0.z, x0.w, r), f_quant8(x1.x, x1.y, x1.z, x1.w, r));
        if (!live) sbyte = 0;
      }
      // codes: chunk ku/16, byte (ku%16)*8 of the row, 128-byte swizzle
      const int chunk = ku >> 4, kb = (ku & 15) * 8;
      const int off = chunk * act_chunk + (m >> 3) * 1024 + (m & 7) * 128 +
                      ((((kb >> 4) ^ (m & 7)) << 4) | (kb & 15));
      *reinterpret_cast<uint2*>(sAct + off) = q;
      if (FMT == 0)
        sScr[m * scr_row + ku] = static_cast<uint8_t>(sbyte);
      else if ((ku & 1) == 0)
        sScr[m * scr_row + (ku >> 1)] = static_cast<uint8_t>(sbyte);
    }
    fence_proxy_async_smem();    // generic-proxy writes -> visible to the tensor core
    workers_sync();
    {
      // activation scales -> tensor memory: lane i (every quarter) holds row i;
      // word c = scale bytes [4c, 4c+4) of the row (one MMA for NVFP4, two for
      // MXFP4) goes to column F_SFB_COL + 4c; the other 3 columns hold 0
      const int words = (FMT == 0) ? n_steps * 4 : n_steps * 2;
      const uint32_t* row = reinterpret_cast<const uint32_t*>(sScr + lane * scr_row);
      const bool has_row = lane < p.nmma_n;
      for (int c0 = 0; c0 < words; c0 += 4) {
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          v[j] = ((j & 3) == 0 && has_row && c0 + (j >> 2) < words) ? row[c0 + (j >> 2)] : 0u;
        tmem_st_x16(tmem + lane_off + F_SFB_COL + 4 * c0, v);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(act_ready);
    // (b) weight scales of each ring stage -> tensor memory (every quarter
    // gets the 32-row x 16-byte block of each atom).  A failed wait only
    // leaves the loop: the accumulator wait below then fails fast too, and
    // all four warps decide together whether to run the epilogue.
    for (int i = 0; i < n_steps; ++i) {
      const int stage = i % FSTAGES;
      const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait(&sf_loaded[stage], phase, abort_flag, p.watchdog, WD_STAGING)))
        break;
      {
        const uint32_t src = smem_u32(sSF + stage * FSF_STAGE) + lane * 16;
        uint32_t v[4 * kAtoms];
#pragma unroll
        for (int a = 0; a < kAtoms; ++a) {
          const uint4 x = lds128(src + a * 512);
          v[4 * a] = x.x; v[4 * a + 1] = x.y; v[4 * a + 2] = x.z; v[4 * a + 3] = x.w;
        }
        const uint32_t dst = tmem + lane_off + F_SFA_COL + stage * 16;
        if (kAtoms == 4) tmem_st_x16(dst, v); else tmem_st_x8(dst, v);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[stage]);
    }
    // (c) epilogue
    {
      const bool ok =
          __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, abort_flag, p.watchdog, WD_EPILOGUE));
      workers_sync();               // every worker warp reaches this barrier
      if (!ok || *abort_flag) goto w_done;
    }
    tc_fence_after();
    {
      uint32_t r[32];
      const uint32_t taddr = tmem + lane_off + F_ACC_COL;
      if (p.nmma_n == 16) {
        uint32_t* rr = r;
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(rr[0]), "=r"(rr[1]), "=r"(rr[2]), "=r"(rr[3]), "=r"(rr[4]), "=r"(rr[5]),
              "=r"(rr[6]), "=r"(rr[7]), "=r"(rr[8]), "=r"(rr[9]), "=r"(rr[10]), "=r"(rr[11]),
              "=r"(rr[12]), "=r"(rr[13]), "=r"(rr[14]), "=r"(rr[15])
            : "r"(taddr));
      } else {
        FP4_TMEM_LD_32x32b_X32(taddr, r);
      }
      tmem_ld_wait();
      const int nloc = quarter * 32 + lane;          // weight row within the tile
      const int n = tile * FBM + nloc;
      const float alpha = (FMT == 0) ? __fmul_rn(g, *p.g_w) : 1.0f;
      if (p.splits == 1) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < 32; ++m) {
            if (m >= p.M) break;
            const float c = __fmul_rn(alpha, __uint_as_float(r[m]));
            if (p.out_f32)
              static_cast<float*>(p.C)[m * p.ldc + n] = c;
            else
              static_cast<__nv_bfloat16*>(p.C)[m * p.ldc + n] = __float2bfloat16_rn(c);
          }
        }
      } else {
        float* mine = p.sums + (static_cast<long long>(tile) * p.splits + split) * p.M * FBM;
#pragma unroll
        for (int m = 0; m < 32; ++m) {
          if (m >= p.M) break;
          mine[m * FBM + nloc] = __uint_as_float(r[m]);
        }
        __threadfence();
        workers_sync();
        if (wt == 0) {
          const unsigned prev = atomicAdd(&p.counters[tile], 1u);
          *last_flag = (prev == static_cast<unsigned>(p.splits - 1)) ? 1 : 0;
        }
        workers_sync();
        if (*last_flag) {
          __threadfence();
          if (n < p.N) {
            const float* base = p.sums + static_cast<long long>(tile) * p.splits * p.M * FBM;
            for (int m = 0; m < p.M; ++m) {
              float acc = 0.0f;
              for (int s = 0; s < p.splits; ++s)
                acc = __fadd_rn(acc, __ldcg(base + (static_cast<long long>(s) * p.M + m) * FBM + nloc));
              const float c = __fmul_rn(alpha, acc);
              if (p.out_f32)
                static_cast<float*>(p.C)[m * p.ldc + n] = c;
              else
                static_cast<__nv_bfloat16*>(p.C)[m * p.ldc + n] = __float2bfloat16_rn(c);
            }
          }
          if (wt == 0) p.counters[tile] = 0;
        }
      }
    }
  w_done:;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, F_TMEM_COLS);
  }
}

// ------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_w_map(CUtensorMap* m, const uint8_t* base, int N, int K) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(FBK_BYTES), static_cast<cuuint32_t>(FBM)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t fused_workspace_bytes(int M, int N, int K, int fmt) {
  return make_plan(M, N, K, fmt).ws_bytes;
}

cudaError_t launch_gemm_fused(const FusedArgs& f, cudaStream_t s) {
  const Plan pl = make_plan(f.M, f.N, f.K, f.fmt);
  uint8_t* ws = static_cast<uint8_t*>(f.ws);
  FParams p{};
  p.a = static_cast<const uint16_t*>(f.a);
  p.w_scales = f.w_scales;
  p.g_w = f.g_w;
  p.g_a = f.g_a;
  p.amax_partial = reinterpret_cast<unsigned*>(ws + pl.ws_partial_off);
  p.counters = reinterpret_cast<unsigned*>(ws + pl.ws_counter_off);
  p.sums = reinterpret_cast<float*>(ws + pl.ws_sum_off);
  p.C = f.C;
  p.ldc = f.ldc;
  p.M = f.M;
  p.N = f.N;
  p.K = f.K;
  p.dynamic = f.dynamic;
  p.out_f32 = f.out_f32;
  p.n_tiles = pl.n_tiles;
  p.k_steps = pl.k_steps;
  p.splits = pl.splits;
  p.steps_max = pl.steps_max;
  p.nmma_n = pl.nmma_n;
  p.ncb = ncb_of(nsf_of(f.K, f.fmt));
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;

  const long long n_vec = static_cast<long long>(f.M) * f.K / 8;
  int pro_blocks = static_cast<int>(std::min<long long>(
      kMaxPrologueCtas, std::max<long long>(1, (n_vec + kPrologueThreads * 4 - 1) /
                                                   (kPrologueThreads * 4))));
  pro_blocks = std::max(pro_blocks, (pl.n_tiles + kPrologueThreads - 1) / kPrologueThreads);
  pro_blocks = std::min(pro_blocks, kMaxPrologueCtas);
  p.n_partial = pro_blocks;
  fused_prologue_kernel<<<pro_blocks, kPrologueThreads, 0, s>>>(
      static_cast<const uint4*>(f.a), n_vec, f.dynamic, const_cast<unsigned*>(p.amax_partial),
      p.counters, pl.n_tiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  CUtensorMap mw;
  if (!make_w_map(&mw, f.w_codes, f.N, f.K)) return cudaErrorInvalidValue;
  auto kern = (f.fmt == 0) ? fused_kernel<0> : fused_kernel<1>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem_bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.n_tiles * pl.splits));
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(pl.smem_bytes);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4
