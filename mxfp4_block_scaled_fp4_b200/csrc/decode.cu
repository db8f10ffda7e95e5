// decode.cu -- one-kernel small-M path of fp4_gemm_fused, for activations
// of at most 128K values (M <= 32 rows).
//
// The W4A4 call of the "fp4-cuda-kernel" forum post at decode sizes: the
// activation is quantized on the fly and multiplied with the weights that
// were quantized at load.  "Hardware FP4 inference for speech on
// Blackwell", sections "Do the FP4 tensor cores even engage?" and the CUDA
// graph discussion: at this size the cost of a call is its fixed overhead,
// not its arithmetic.  A call of the three-kernel chain in fused.cu (amax,
// quantize, GEMM) measured 6.6-9.5 us on B200 for weights that stream in
// 0.5-0.7 us, each kernel boundary costing 1-2 us; this path is one kernel.
//
// Same arithmetic as fp4_quantize_act followed by fp4_gemm (bit-identical
// codes and scales, the codecs of codec.cuh), up to FP32 summation order.
//
// Per CTA (a 128-row weight tile x one K slice of at most 8 steps of 256):
//   warp 0     TMA: the weight tile (16 KiB per step, 128-byte swizzle) and
//              its scale atoms through a 4-stage ring, from the kernel's
//              first instruction (weights never depend on the preceding
//              kernel of the stream);
//   warp 1     tensor memory; one thread issues the MMAs (swap-AB: weights
//              are the 128-row A operand, the activation rows the 16- or
//              32-wide B operand) once the activation slice is ready;
//   warps 2-5  after griddepcontrol.wait: the activation's global amax
//              (every CTA reads the whole activation from L2: at most
//              256 KiB), then this CTA's K slice of the activation quantized
//              straight into the MMA's B layout in shared memory (codes with
//              the 128-byte swizzle, scales per row); then per step the
//              weight and activation scales into tensor memory; then the
//              epilogue.
// With S > 1 slices per tile the S CTAs of a tile form a cluster and reduce
// their FP32 partials in slice order through distributed shared memory
// (deterministic), as in fused.cu.  Every wait is bounded (watchdog).
#include <algorithm>
#include <cuda_bf16.h>

#include "codec.cuh"
#include "internal.h"
#include "launch_shape.h"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int DBM = 128;                     // weight rows per tile
constexpr int DBK = 256;                     // K per step
constexpr int DBK_BYTES = DBK / 2;
constexpr int DSTAGES = 4;
constexpr int DW_STAGE = DBM * DBK_BYTES;    // 16 KiB weight codes
constexpr int DSF_STAGE = 4 * 512;           // weight scale atoms of a step
constexpr int kMaxSteps = 8;                 // K steps per CTA
constexpr int kMaxRows = 32;                 // activation rows (MMA N, padded)
constexpr int DX_STEP = kMaxRows * DBK_BYTES;   // 4 KiB activation codes per step
constexpr int DXS_STEP = kMaxRows * 16;         // activation scales per step, 16 B per row
constexpr int kMaxSplits = 8;                // portable cluster size
constexpr int kThreads = 192;
// Every CTA reads the whole activation (amax) and quantizes M x its K slice:
// beyond these sizes the three-kernel chain, which quantizes once, is faster
// (measured on B200).
constexpr long long kMaxActValues = 32768;   // 64 KiB of bf16 read by every CTA
constexpr int kMaxSliceValues = 16384;       // values quantized by one CTA
constexpr int SMEM_BYTES =
    1024 + DSTAGES * (DW_STAGE + DSF_STAGE) + kMaxSteps * (DX_STEP + DXS_STEP) + 512 + 256;
constexpr uint32_t D_TMEM_COLS = 256;
constexpr uint32_t D_ACC_COL = 0;            // <= 32 fp32 columns
constexpr uint32_t D_SFA_COL = 32;           // weight scales: 16 columns per stage
constexpr uint32_t D_SFB_COL = 96;           // activation scales: 16 columns per stage

static_assert(SMEM_BYTES <= 113 * 1024, "two CTAs must fit an SM");
static_assert(D_SFB_COL + DSTAGES * 16 <= D_TMEM_COLS, "scale stages exceed tensor memory");

struct DPlan {
  bool ok;
  int n_tiles, k_steps, splits, nmma_n;
};

// The largest split count S <= 8 whose grid fits one wave of two CTAs per
// SM; the path applies when every slice then has at most kMaxSteps steps.
DPlan make_dplan(int M, int N, int K, int sms) {
  DPlan p{};
  p.n_tiles = (N + DBM - 1) / DBM;
  p.k_steps = (K + DBK - 1) / DBK;
  p.nmma_n = M <= 16 ? 16 : 32;
  static_assert(kMaxSplits == 8, "decode_splits assumes portable clusters of 8");
  const int s = decode_splits(M, p.n_tiles, p.k_steps, sms, kMaxSteps);
  p.splits = s;
  const int slice_steps = (p.k_steps + s - 1) / s;
  p.ok = M >= 1 && M <= kMaxRows && static_cast<long long>(M) * K <= kMaxActValues &&
         slice_steps <= kMaxSteps && M * slice_steps * DBK <= kMaxSliceValues;
  return p;
}

struct DParams {
  const uint16_t* x;         // bf16 [M, K]
  const uint8_t* w_scales;   // MMA order
  const float* g_w;
  float* g_a;                // DYNAMIC: written (by CTA 0); STATIC: read
  void* C;
  long long ldc;
  int M, N, K;
  int dynamic, out_f32;
  int n_tiles, k_steps, splits, nmma_n, ncb;
  unsigned* watchdog;
  float rot_scale;           // rotation (ROT = 16 or 32): 2^-shift
  int rule;                  // MXFP4 scale rule: 0 OCP, 1 overflow-aware
};

__device__ __forceinline__ void workers_sync() {   // named barrier of the 4 worker warps
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_x16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ float ld_peer_f32(uint32_t local_saddr, uint32_t rank) {
  float v;
  // no memory clobber: the loads of one row may be in flight together (the
  // cluster barrier before them orders them after the peers' stores)
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(map_to_rank(local_saddr, rank)));
  return v;
}

__device__ __forceinline__ void store_out(const DParams& p, int m, int n, float c) {
  if (p.out_f32)
    static_cast<float*>(p.C)[m * p.ldc + n] = c;
  else
    static_cast<__nv_bfloat16*>(p.C)[m * p.ldc + n] = __float2bfloat16_rn(c);
}

template <int FMT, int ROT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_w, const DParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;                                  // DSTAGES x 16 KiB weight codes
  uint8_t* sX = sW + DSTAGES * DW_STAGE;               // kMaxSteps x 4 KiB activation codes
  uint8_t* sWS = sX + kMaxSteps * DX_STEP;             // DSTAGES x weight scale atoms
  uint8_t* sXS = sWS + DSTAGES * DSF_STAGE;            // kMaxSteps x activation scales
  float* r_tab = reinterpret_cast<float*>(sXS + kMaxSteps * DXS_STEP);   // 128 reciprocals
  uint64_t* full = reinterpret_cast<uint64_t*>(r_tab + 128);
  uint64_t* empty = full + DSTAGES;
  uint64_t* sf_full = empty + DSTAGES;
  uint64_t* act_ready = sf_full + DSTAGES;
  uint64_t* acc_full = act_ready + 1;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  unsigned* red = reinterpret_cast<unsigned*>(tmem_slot + 2);   // 4 words

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / p.splits, split = blockIdx.x % p.splits;
  const int s_lo = static_cast<int>(static_cast<long long>(split) * p.k_steps / p.splits);
  const int s_hi = static_cast<int>(static_cast<long long>(split + 1) * p.k_steps / p.splits);
  const int n_steps = s_hi - s_lo;
  constexpr int kAtoms = (FMT == 0) ? 4 : 2;   // scale atoms (and scale words) per step

  if (threadIdx.x == 0) {
    for (int s = 0; s < DSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 4);
    }
    mbar_init(act_ready, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_w);
  }
  __syncthreads();
  // every CTA of this grid is resident: the next kernel of the stream may
  // launch now (it reads nothing this one writes before its own wait)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  uint32_t tmem = 0;
  if (warp >= 1) {
    if (warp == 1) {
      tmem_alloc(tmem_slot, D_TMEM_COLS);
      tmem_relinquish();
    }
    tc_fence_before();
    asm volatile("bar.sync 2, 160;" ::: "memory");   // warps 1-5
    tc_fence_after();
    tmem = *tmem_slot;
  }
  bool epilogue_ok = false;
  float g = 1.0f;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ weight producer
      uint32_t armed = 0, armed_parity = 0;
      for (int i = 0; i < n_steps; ++i) {
        const int stage = i % DSTAGES;
        const uint32_t phase = static_cast<uint32_t>(i / DSTAGES) & 1u;
        if (i == DSTAGES) {
          // the ring is full and frees only once the MMAs run (after the
          // activation's amax and quantization): the slice's remaining
          // weight tiles and scale atoms stream into L2 meanwhile
          for (int j = DSTAGES; j < n_steps; ++j) {
            const int ksj = s_lo + j, cbj = ksj * kAtoms;
            tma_prefetch_l2_2d(&tm_w, ksj * DBK_BYTES, tile * DBM);
            bulk_prefetch_l2(p.w_scales + (static_cast<long long>(tile) * p.ncb + cbj) * 512,
                             static_cast<uint32_t>(min(kAtoms, p.ncb - cbj)) * 512u);
          }
        }
        if (i >= DSTAGES &&
            !mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER))
          break;
        const int ks = s_lo + i;
        const int cb0 = ks * kAtoms;
        const uint32_t sf_bytes = static_cast<uint32_t>(min(kAtoms, p.ncb - cb0)) * 512u;
        mbar_expect_tx(&full[stage], DW_STAGE + sf_bytes);
        bulk_load(sWS + stage * DSF_STAGE,
                  p.w_scales + (static_cast<long long>(tile) * p.ncb + cb0) * 512, sf_bytes,
                  &full[stage]);
        tma_load_2d(sW + stage * DW_STAGE, &tm_w, ks * DBK_BYTES, tile * DBM, &full[stage]);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
      }
      if (*abort_flag) {
        for (int s = 0; s < DSTAGES; ++s)
          if (armed & (1u << s)) mbar_wait_drain(&full[s], (armed_parity >> s) & 1u, p.watchdog);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      bool ok = mbar_wait(act_ready, 0, abort_flag, p.watchdog, WD_MMA_FULL);
      for (int i = 0; i < n_steps && ok; ++i) {
        const int stage = i % DSTAGES;
        const uint32_t phase = static_cast<uint32_t>(i / DSTAGES) & 1u;
        // one wait per step: the staging warps arrive on sf_full only after
        // the step's weight tile has landed (a test of an mbarrier is a
        // ~250-cycle round trip even when its phase has completed)
        ok = mbar_wait(&sf_full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL);
        if (!ok) break;
        tc_fence_after();
        const int kglob = (s_lo + i) * DBK;
        const int n_mma = min(4, (p.K - kglob + 63) / 64);
        const uint32_t w_s = smem_u32(sW + stage * DW_STAGE);
        const uint32_t x_s = smem_u32(sX + i * DX_STEP);
        const uint32_t sfa = tmem + D_SFA_COL + stage * 16;
        const uint32_t sfb = tmem + D_SFB_COL + stage * 16;
        for (int k = 0; k < n_mma; ++k) {
          const uint64_t ad = smem_desc(w_s + k * 32, 16, 1024, kLayoutSwizzle128B);
          const uint64_t bd = smem_desc(x_s + k * 32, 16, 1024, kLayoutSwizzle128B);
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          if (FMT == 0) {
            tc_mma_nvf4(tmem + D_ACC_COL, ad, bd, idesc_fp4(DBM, p.nmma_n, false, 0, 0),
                        sfa + 4 * k, sfb + 4 * k, acc);
          } else {
            const uint32_t id = 2u * (k & 1);
            tc_mma_mxf4(tmem + D_ACC_COL, ad, bd, idesc_fp4(DBM, p.nmma_n, true, id, id),
                        sfa + 4 * (k >> 1), sfb + 4 * (k >> 1), acc);
          }
        }
        tc_commit(&empty[stage]);
      }
      if (ok) {
        tc_commit(acc_full);
      } else {
        tc_commit(drain);
        mbar_wait_drain(drain, 0, p.watchdog);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ workers
    const int wt = threadIdx.x - 64;   // 0..127
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    // (a) activation buffers start at zero: rows >= M and K past the end
    //     meet the MMA as zero codes with zero scales
    {
      const uint32_t xb = smem_u32(sX), xsb = smem_u32(sXS);
      for (int i = wt; i < n_steps * (DX_STEP / 16); i += 128) sts128(xb + i * 16, 0u, 0u, 0u, 0u);
      for (int i = wt; i < n_steps * (DXS_STEP / 16); i += 128) sts128(xsb + i * 16, 0u, 0u, 0u, 0u);
    }
    // the activation (and a STATIC g) come from the preceding kernels
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // this CTA's K slice: 16-value units, upr per row (even)
    const int k0 = s_lo * DBK;
    const int upr = (min(p.K, s_hi * DBK) - k0) / 16;
    const int units = p.M * upr;
    // the first 128 units' loads go out now, so that their round trip
    // overlaps the amax pass's
    uint4 pre0 = make_uint4(0u, 0u, 0u, 0u), pre1 = pre0;
    if (wt < units) {
      const int m = wt / upr, i = wt - (wt / upr) * upr;
      const uint16_t* src = p.x + static_cast<long long>(m) * p.K + k0 + 16 * i;
      pre0 = ld_x16(src);
      pre1 = ld_x16(src + 8);
    }
    // (b) the global scale: g = RN(amax / 2688), 1 for an all-zero tensor
    //     (DYNAMIC; every CTA computes it, CTA 0 reports it), or the caller's
    if (FMT == 0) {
      if (p.dynamic) {
        unsigned m = 0;
        if (ROT == 0) {
          const long long n_vec = static_cast<long long>(p.M) * p.K / 8;
          // eight 16-byte loads in flight per thread
          for (long long v = wt; v < n_vec; v += 1024) {
            uint4 t[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              t[j] = (v + 128 * j < n_vec) ? ld_x16(p.x + (v + 128 * j) * 8) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int j = 0; j < 8; ++j) m = max_u16x2(m, mag_max8(t[j]));
          }
          m = fold_u16x2(m);
        } else {
          // rotated values: 16-value units, four (eight loads) in flight per
          // thread; whole warps iterate together (a 32-rotation pairs lanes)
          const long long n_units = static_cast<long long>(p.M) * p.K / 16;
          for (long long base = 0; base < n_units; base += 512) {
            uint4 t[4][2];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const long long u = base + wt + 128 * j;
              const bool in = u < n_units;
              t[j][0] = in ? ld_x16(p.x + u * 16) : make_uint4(0u, 0u, 0u, 0u);
              t[j][1] = in ? ld_x16(p.x + u * 16 + 8) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float f[16];
              unpack16(t[j][0], t[j][1], f);
              rotate_unit<ROT>(f, p.rot_scale, (lane & 1) != 0);
              m = max(m, mag_max16(f));
            }
          }
        }
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) red[warp - 2] = m;
        workers_sync();
        m = max(max(red[0], red[1]), max(red[2], red[3]));
        // CTA 0 reports a non-finite input; every CTA clamps alike
        float amax;
        if (ROT == 0) {
          if (m > kBf16MaxFinite)
            m = (blockIdx.x == 0 && wt == 0) ? amax_checked(m, p.watchdog) : kBf16MaxFinite;
          amax = __uint_as_float(m << 16);
        } else {
          if (m > kF32MaxFinite)
            m = (blockIdx.x == 0 && wt == 0) ? amax_checked_f32(m, p.watchdog) : kF32MaxFinite;
          amax = __uint_as_float(m);
        }
        g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
        if (blockIdx.x == 0 && wt == 0) *p.g_a = g;
      } else {
        g = *p.g_a;
      }
      r_tab[wt] = nvfp4_recip(static_cast<unsigned>(wt), g);
    }
    workers_sync();
    // (c) this CTA's K slice of the activation, quantized into the MMA's B
    //     layout: per step, row m's 128 code bytes with the 128-byte swizzle
    //     (16-byte chunk j at j ^ (m % 8)), and its 16 scale bytes (scale
    //     index i of the step at byte i: word w = the scales MMA w reads)
    {
      const float six_g = __fmul_rn(6.0f, g);
      const float y6 = __frcp_rn(six_g);
      const bool fast_b = six_g >= 0x1p-40f && six_g <= 0x1p40f;
      uint4 nx0 = pre0, nx1 = pre1;
      for (int base = 0; base < units; base += 128) {
        const int u = base + wt;
        const bool valid = u < units;
        const int m = valid ? u / upr : 0;
        const int i = valid ? u - m * upr : 0;
        const uint4 a0 = nx0, a1 = nx1;
        // the next batch's loads go out before this batch is converted
        nx0 = nx1 = make_uint4(0u, 0u, 0u, 0u);
        if (u + 128 < units) {
          const int mn = (u + 128) / upr, in = u + 128 - mn * upr;
          const uint16_t* src = p.x + static_cast<long long>(mn) * p.K + k0 + 16 * in;
          nx0 = ld_x16(src);
          nx1 = ld_x16(src + 8);
        }
        unsigned sbyte;
        float r;
        uint2 packed;
        if (ROT == 0) {
          unsigned mx = fold_u16x2(max_u16x2(mag_max8(a0), mag_max8(a1)));
          if (FMT == 0) {
            sbyte = 0u;
            packed = make_uint2(0u, 0u);
            if (valid) {
              sbyte = nvfp4_scale_byte(mx, six_g, y6, fast_b);
              r = r_tab[sbyte & 127u];
              if (r != 0.0f)
                packed = make_uint2(quant8(a0.x, a0.y, a0.z, a0.w, r), quant8(a1.x, a1.y, a1.z, a1.w, r));
            }
          } else {
            // a 32-value block is a pair of adjacent units = adjacent lanes
            mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
            sbyte = mxfp4_scale_f32(mx << 16, p.rule, &r);
            packed = make_uint2(quant8(a0.x, a0.y, a0.z, a0.w, r), quant8(a1.x, a1.y, a1.z, a1.w, r));
          }
        } else {
          // rotated unit (lanes 2i, 2i+1 hold the halves of a 32-value block;
          // every lane takes part, invalid ones with zeros)
          float f[16];
          unpack16(a0, a1, f);
          rotate_unit<ROT>(f, p.rot_scale, (lane & 1) != 0);
          unsigned mx = mag_max16(f);
          if (FMT == 0) {
            sbyte = nvfp4_scale_byte_f32(mx, six_g, y6, fast_b);
            r = r_tab[sbyte & 127u];
            packed = (r == 0.0f) ? make_uint2(0u, 0u) : make_uint2(quant8_f32(f, r), quant8_f32(f + 8, r));
          } else {
            mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
            sbyte = mxfp4_scale_f32(mx, p.rule, &r);
            packed = make_uint2(quant8_f32(f, r), quant8_f32(f + 8, r));
          }
        }
        if (valid) {
          const int step = i >> 4, iu = i & 15;
          const uint32_t caddr = smem_u32(sX) + step * DX_STEP + m * DBK_BYTES +
                                 ((((iu >> 1) ^ (m & 7)) << 4) | ((iu & 1) << 3));
          asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(caddr), "r"(packed.x),
                       "r"(packed.y) : "memory");
          if (FMT == 0 || (iu & 1) == 0) {
            const int idx = (FMT == 0) ? iu : (iu >> 1);
            sXS[step * DXS_STEP + m * 16 + idx] = static_cast<uint8_t>(sbyte);
          }
        }
      }
    }
    // the MMA (async proxy) reads what these generic stores wrote
    fence_proxy_async_smem();
    workers_sync();
    if (wt == 0) mbar_arrive(act_ready);
    // (d) per step, the weight scale atoms and the activation scales into
    //     tensor memory; every 32-lane quarter gets the whole image (atom a
    //     at columns 4a..4a+3; an activation row's word a at column 4a)
    for (int i = 0; i < n_steps; ++i) {
      const int stage = i % DSTAGES;
      const uint32_t phase = static_cast<uint32_t>(i / DSTAGES) & 1u;
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait(&full[stage], phase, abort_flag, p.watchdog, WD_STAGING)))
        continue;
      const uint32_t ws = smem_u32(sWS + stage * DSF_STAGE) + lane * 16;
      const uint4 xw = lds128(smem_u32(sXS + i * DXS_STEP) + lane * 16);   // zero past M
      const uint32_t xwords[4] = {xw.x, xw.y, xw.z, xw.w};
      uint32_t va[16], vb[16];
#pragma unroll
      for (int a = 0; a < kAtoms; ++a) {
        const uint4 w = lds128(ws + a * 512);
        va[4 * a] = w.x; va[4 * a + 1] = w.y; va[4 * a + 2] = w.z; va[4 * a + 3] = w.w;
        vb[4 * a] = xwords[a]; vb[4 * a + 1] = 0u; vb[4 * a + 2] = 0u; vb[4 * a + 3] = 0u;
      }
      if (kAtoms == 4) {
        tmem_st_x16(tmem + lane_off + D_SFA_COL + stage * 16, va);
        tmem_st_x16(tmem + lane_off + D_SFB_COL + stage * 16, vb);
      } else {
        tmem_st_x8(tmem + lane_off + D_SFA_COL + stage * 16, va);
        tmem_st_x8(tmem + lane_off + D_SFB_COL + stage * 16, vb);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[stage]);
    }
    // (e) accumulator -> C (one slice) or -> this CTA's partial in shared
    //     memory (several slices: the cluster reduces them below)
    {
      const bool done =
          __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, abort_flag, p.watchdog, WD_EPILOGUE));
      workers_sync();
      epilogue_ok = done && !*abort_flag;
    }
    const float alpha = (FMT == 0) ? __fmul_rn(g, *p.g_w) : 1.0f;
    g = alpha;   // kept for the cluster reduction below
    if (epilogue_ok) {
      tc_fence_after();
      uint32_t r[32];
      const uint32_t taddr = tmem + lane_off + D_ACC_COL;
      if (p.nmma_n == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
              "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
              "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
      } else {
        FP4_TMEM_LD_32x32b_X32(taddr, r);
      }
      tmem_ld_wait();
      const int nloc = quarter * 32 + lane;   // weight row within the tile
      const int n = tile * DBM + nloc;
      if (p.splits == 1) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < 32; ++m)
            if (m < p.M) store_out(p, m, n, __fmul_rn(alpha, __uint_as_float(r[m])));
        }
      } else {
        float* part = reinterpret_cast<float*>(sW);   // the ring is idle now
#pragma unroll
        for (int m = 0; m < 32; ++m)
          if (m < p.M) part[m * DBM + nloc] = __uint_as_float(r[m]);
      }
    }
  }

  if (p.splits > 1) {
    // every CTA of the tile's cluster has written its partial sums
    cluster_sync_all();
    if (warp >= 2 && epilogue_ok) {
      const int t = threadIdx.x - 64;
      const int n = tile * DBM + t;
      const uint32_t base = smem_u32(sW) + t * 4;
      // CTA `split` reduces rows m = split, split + S, ... in slice order;
      // all S remote loads of a row are issued before the first add
      for (int m = split; m < p.M; m += p.splits) {
        float v[kMaxSplits];
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s)
          v[s] = (s < p.splits) ? ld_peer_f32(base + m * DBM * 4, static_cast<uint32_t>(s)) : 0.0f;
        float acc = 0.0f;
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s)
          if (s < p.splits) acc = __fadd_rn(acc, v[s]);
        if (n < p.N) store_out(p, m, n, __fmul_rn(g, acc));
      }
    }
    // peers read this CTA's shared memory until here
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, D_TMEM_COLS);
  }
}

}  // namespace

bool decode_supported(int M, int N, int K, int max_sms) {
  return make_dplan(M, N, K, gemm_sms(max_sms)).ok;
}

cudaError_t launch_decode(const FusedArgs& f, cudaStream_t s) {
  const DPlan pl = make_dplan(f.M, f.N, f.K, gemm_sms(f.max_sms));
  if (!pl.ok) return cudaErrorInvalidValue;
  DParams p{};
  p.x = static_cast<const uint16_t*>(f.a);
  p.w_scales = f.w_scales;
  p.g_w = f.g_w;
  p.g_a = f.g_a;
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
  p.nmma_n = pl.nmma_n;
  p.ncb = ncb_of(nsf_of(f.K, f.fmt));
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;
  p.rot_scale = f.rot_scale;
  p.rule = f.rule;
  CUtensorMap mw;
  if (!make_code_map(&mw, f.w_codes, f.N, f.K, DBM)) return cudaErrorInvalidValue;
  using Kern = void (*)(const CUtensorMap, const DParams);
  static const Kern table[3][2] = {{decode_kernel<0, 0>, decode_kernel<1, 0>},
                                   {decode_kernel<0, 16>, decode_kernel<1, 16>},
                                   {decode_kernel<0, 32>, decode_kernel<1, 32>}};
  const Kern kern = table[f.rot == 32 ? 2 : (f.rot == 16 ? 1 : 0)][f.fmt != 0];
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.n_tiles * pl.splits));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(SMEM_BYTES);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pl.splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(pl.splits);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  // a programmatic dependent of the preceding kernel: the weights stream
  // while it finishes (the activation is read after griddepcontrol.wait)
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, mw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4
