// gemm.cu -- block-scaled FP4 GEMM on the sm_100a tcgen05 tensor cores.
//
//   C[M, N] = alpha * sum_k s_a[m, k/B] q_a[m, k] * s_w[n, k/B] q_w[n, k]
//
// The W4A4 GEMM of the "fp4-cuda-kernel" forum post (pre-quantized weights,
// on-the-fly activations); NVFP4 blocks (B = 16, E4M3 scales, alpha = g_a
// g_w) from "Hardware FP4 inference for speech on Blackwell", section
// "NVFP4, and the two ways it fails"; MXFP4 blocks (B = 32, E8M0 scales,
// alpha = 1) from the format table of "FP4 n'existe pas".
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      one thread drives TMA: packed A / W tiles (128 B of K per
//               row, 128-byte swizzle) and the matching scale atoms (plain
//               bulk copies: in the MMA scale order a tile's scales for one
//               K step are contiguous) into a 4-stage shared-memory ring;
//   warp 1      one thread issues tcgen05.mma kind::mxf4nvf4 (128 x 256 x 64
//               per instruction) into an FP32 accumulator in tensor memory
//               and releases ring stages with tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld the accumulator (one 32-lane quarter
//               per warp), multiply by alpha, round to bf16 / keep fp32,
//               store C;
//   warps 6-9   scale staging: each warp reads a stage's scale atoms from
//               shared memory and writes them with tcgen05.st into its own
//               32-lane quarter of the stage's scale region in tensor memory
//               (every quarter gets the whole 32-row x 16-byte block of an
//               atom, the image the MMA reads), then signals the MMA thread.
//               Moving scales with warp stores instead of tcgen05.cp keeps
//               the copies out of the MMA pipe: measured on B200, even one
//               tcgen05.cp per K step stalled the MMAs of every step.
// Every mbarrier wait is bounded; a wait that runs out sets the watchdog
// word, the CTA stops issuing, waits (bounded) for its copies and MMAs in
// flight, frees its tensor memory and returns.
#include <algorithm>
#include <cstdio>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;                 // FP4 elements of K per ring stage
constexpr int BK_BYTES = BK / 2;        // 128: one 128-byte swizzle row
constexpr int MMA_K = 64;               // FP4 elements per tcgen05.mma
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK_BYTES;  // 16 KiB
constexpr int B_STAGE = BN * BK_BYTES;  // 32 KiB
constexpr int SFA_STAGE = 4 * 512;      // up to 4 scale atoms (128 rows x 4 scales)
constexpr int SFB_STAGE = 2 * 4 * 512;  // two 128-row blocks x 4 atoms
constexpr int RING_BYTES = STAGES * (A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE);
constexpr int SMEM_BYTES = RING_BYTES + 1024 + 256;   // ring + alignment + barriers
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;         // 256 fp32 columns
constexpr uint32_t SF_COL = 256;        // per stage: 16 columns A scales + 32 B scales
constexpr uint32_t SF_STAGE_COLS = 48;
constexpr int kGemmThreads = 320;       // 10 warps: TMA, MMA, 4 epilogue, 4 scale staging
constexpr int GROUP_M = 16;             // tile raster: 16 M-tiles share their W tiles in L2

struct Params {
  const uint8_t* a_scales;
  const uint8_t* w_scales;
  const float* g_a;
  const float* g_w;
  void* C;
  long long ldc;
  int M, N, K;
  int m_tiles, n_tiles, k_steps;
  int ncb;                // scale atoms per 128-row block
  int w_rowblocks;        // ceil(N / 128)
  unsigned* watchdog;
};

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mt, int& nt) {
  const int per_group = GROUP_M * p.n_tiles;
  const int group = t / per_group;
  const int first_m = group * GROUP_M;
  const int gsize = min(GROUP_M, p.m_tiles - first_m);
  const int within = t - group * per_group;
  mt = first_m + within % gsize;
  nt = within / gsize;
}

template <int FMT, int OUT_F32>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE;
  uint8_t* sSFA = sB + STAGES * B_STAGE;
  uint8_t* sSFB = sSFA + STAGES * SFA_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * SFB_STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_loaded = empty + STAGES;
  uint64_t* sf_full = sf_loaded + STAGES;
  uint64_t* acc_full = sf_full + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_loaded[s], 1);
      mbar_init(&sf_full[s], 4);   // one arrival per scale-staging warp
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);   // one arrival per epilogue warp
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_tiles_total = p.m_tiles * p.n_tiles;
  constexpr int kAtomsPerStage = (FMT == 0) ? 4 : 2;   // scale atoms per 256 K

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    for (int t = blockIdx.x; t < n_tiles_total; t += gridDim.x) {
      int mt, nt;
      tile_coords(t, p, mt, nt);
      for (int kb = 0; kb < p.k_steps; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER)) goto producer_drain;
        {
          const int cb0 = kb * kAtomsPerStage;
          const int atoms = min(kAtomsPerStage, p.ncb - cb0);
          const uint32_t sf_bytes = static_cast<uint32_t>(atoms) * 512u;
          const int rb0 = nt * 2;
          const int wblocks = min(2, p.w_rowblocks - rb0);
          // scales first, on their own barrier, so that staging them into
          // tensor memory overlaps the (larger) code tiles' flight
          mbar_expect_tx(&sf_loaded[stage], sf_bytes * (1 + wblocks));
          bulk_load(sSFA + stage * SFA_STAGE,
                    p.a_scales + (static_cast<long long>(mt) * p.ncb + cb0) * 512, sf_bytes,
                    &sf_loaded[stage]);
          for (int i = 0; i < wblocks; ++i)
            bulk_load(sSFB + stage * SFB_STAGE + i * 2048,
                      p.w_scales + (static_cast<long long>(rb0 + i) * p.ncb + cb0) * 512, sf_bytes,
                      &sf_loaded[stage]);
          mbar_expect_tx(&full[stage], A_STAGE + B_STAGE);
          tma_load_2d(sA + stage * A_STAGE, &tm_a, kb * BK_BYTES, mt * BM, &full[stage]);
          tma_load_2d(sB + stage * B_STAGE, &tm_w, kb * BK_BYTES, nt * BN, &full[stage]);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    goto producer_done;
  producer_drain:
    // let every copy this thread started land before the CTA goes away
    for (int s = 0; s < STAGES; ++s)
      if (armed & (1u << s)) {
        mbar_wait_drain(&sf_loaded[s], (armed_parity >> s) & 1u, p.watchdog);
        mbar_wait_drain(&full[s], (armed_parity >> s) & 1u, p.watchdog);
      }
  producer_done:;
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    for (int t = blockIdx.x; t < n_tiles_total; t += gridDim.x, ++it) {
      if (it > 0 && !mbar_wait(acc_empty, static_cast<uint32_t>(it - 1) & 1u, abort_flag, p.watchdog, WD_MMA_ACC))
        goto mma_drain;
      tc_fence_after();
      for (int kb = 0; kb < p.k_steps; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL)) goto mma_drain;
        if (!mbar_wait(&sf_full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL)) goto mma_drain;
        tc_fence_after();
        {
          const int n_mma = min(BK / MMA_K, (p.K - kb * BK + MMA_K - 1) / MMA_K);
          const uint32_t sfa_t = tmem + SF_COL + stage * SF_STAGE_COLS;
          const uint32_t sfb_t = sfa_t + 16;
          const uint32_t a_s = smem_u32(sA + stage * A_STAGE);
          const uint32_t b_s = smem_u32(sB + stage * B_STAGE);
          for (int k = 0; k < n_mma; ++k) {
            const uint64_t ad = smem_desc(a_s + k * (MMA_K / 2), 16, 1024, kLayoutSwizzle128B);
            const uint64_t bd = smem_desc(b_s + k * (MMA_K / 2), 16, 1024, kLayoutSwizzle128B);
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
            if (FMT == 0) {
              tc_mma_nvf4(tmem + ACC_COL, ad, bd, idesc_fp4(BM, BN, false, 0, 0), sfa_t + 4 * k,
                          sfb_t + 8 * k, acc);
            } else {
              const uint32_t id = 2u * (k & 1);
              tc_mma_mxf4(tmem + ACC_COL, ad, bd, idesc_fp4(BM, BN, true, id, id),
                          sfa_t + 4 * (k >> 1), sfb_t + 8 * (k >> 1), acc);
            }
          }
        }
        tc_commit(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      tc_commit(acc_full);
    }
    goto mma_done;
  mma_drain:
    tc_commit(drain);
    mbar_wait_drain(drain, 0, p.watchdog);
  mma_done:;
  } else if (warp >= 6) {
    // ----------------------------------------------------- scale staging
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < n_tiles_total; t += gridDim.x) {
      for (int kb = 0; kb < p.k_steps; ++kb) {
        // warp-uniform outcome: tcgen05.st below needs all 32 lanes
        if (!__all_sync(0xFFFFFFFFu,
                        mbar_wait(&sf_loaded[stage], phase, abort_flag, p.watchdog, WD_STAGING)))
          goto staging_done;
        {
          const uint32_t sfa_s = smem_u32(sSFA + stage * SFA_STAGE) + lane * 16;
          const uint32_t sfb_s = smem_u32(sSFB + stage * SFB_STAGE) + lane * 16;
          const uint32_t sfa_t = tmem + lane_off + SF_COL + stage * SF_STAGE_COLS;
          const uint32_t sfb_t = sfa_t + 16;
          // atom a, row `lane`: 16 bytes = 4 columns; A at columns 4a..4a+3,
          // W row block rb at columns 8a + 4rb .. 8a + 4rb + 3
          uint32_t va[4 * kAtomsPerStage], vb[8 * kAtomsPerStage];
#pragma unroll
          for (int a = 0; a < kAtomsPerStage; ++a) {
            const uint4 x = lds128(sfa_s + a * 512);
            va[4 * a + 0] = x.x; va[4 * a + 1] = x.y; va[4 * a + 2] = x.z; va[4 * a + 3] = x.w;
#pragma unroll
            for (int rb = 0; rb < 2; ++rb) {
              const uint4 y = lds128(sfb_s + rb * 2048 + a * 512);
              vb[8 * a + 4 * rb + 0] = y.x; vb[8 * a + 4 * rb + 1] = y.y;
              vb[8 * a + 4 * rb + 2] = y.z; vb[8 * a + 4 * rb + 3] = y.w;
            }
          }
          if (kAtomsPerStage == 4) {
            tmem_st_x16(sfa_t, va);
            tmem_st_x32(sfb_t, vb);
          } else {
            tmem_st_x8(sfa_t, va);
            tmem_st_x16(sfb_t, vb);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  staging_done:;
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;        // tensor-memory lanes this warp may read
    float alpha = 1.0f;
    if (FMT == 0) alpha = __fmul_rn(*p.g_a, *p.g_w);
    int it = 0;
    for (int t = blockIdx.x; t < n_tiles_total; t += gridDim.x, ++it) {
      int mt, nt;
      tile_coords(t, p, mt, nt);
      // warp-uniform outcome: tcgen05.ld below needs all 32 lanes
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag,
                                             p.watchdog, WD_EPILOGUE)))
        break;
      tc_fence_after();
      const int row = mt * BM + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + ACC_COL;
      if (!OUT_F32) {
        // bf16: the whole 256-column row fits in 128 registers once packed,
        // so the accumulator is released before any global store is issued
        uint32_t packed[BN / 2];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          FP4_TMEM_LD_32x32b_X32(tbase + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float lo = __fmul_rn(alpha, __uint_as_float(r[2 * j]));
            const float hi = __fmul_rn(alpha, __uint_as_float(r[2 * j + 1]));
            __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
            packed[16 * c + j] = *reinterpret_cast<uint32_t*>(&h);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        if (row_ok) {
          uint16_t* out = static_cast<uint16_t*>(p.C) + static_cast<long long>(row) * p.ldc;
#pragma unroll
          for (int v = 0; v < BN / 8; ++v) {
            const int n = nt * BN + 8 * v;
            if (n < p.N)
              *reinterpret_cast<uint4*>(out + n) = make_uint4(packed[4 * v], packed[4 * v + 1],
                                                              packed[4 * v + 2], packed[4 * v + 3]);
          }
        }
      } else {
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          FP4_TMEM_LD_32x32b_X32(tbase + c * 32, r);
          tmem_ld_wait();
          if (c == BN / 32 - 1) {
            // accumulator fully read: let the next tile's MMAs start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          const int n0 = nt * BN + c * 32;
          if (!row_ok || n0 >= p.N) continue;
          float* out = static_cast<float*>(p.C) + static_cast<long long>(row) * p.ldc + n0;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            if (n0 + 4 * v < p.N) {
              float4 o;
              o.x = __fmul_rn(alpha, __uint_as_float(r[4 * v + 0]));
              o.y = __fmul_rn(alpha, __uint_as_float(r[4 * v + 1]));
              o.z = __fmul_rn(alpha, __uint_as_float(r[4 * v + 2]));
              o.w = __fmul_rn(alpha, __uint_as_float(r[4 * v + 3]));
              *reinterpret_cast<float4*>(out + 4 * v) = o;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

bool make_code_map(CUtensorMap* m, const uint8_t* base, long long rows, int K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK_BYTES), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_bf16_out_map(CUtensorMap* m, void* C, long long rows, int cols, int ldc, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldc) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

template <int FMT, int OUT_F32>
cudaError_t launch_typed(const CUtensorMap& ma, const CUtensorMap& mw, const Params& p, int grid,
                         cudaStream_t s) {
  auto kern = gemm_kernel<FMT, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<grid, kGemmThreads, SMEM_BYTES, s>>>(ma, mw, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s) {
  if (a.M > BM) return launch_gemm_pair(a, s);
  CUtensorMap ma, mw;
  if (!make_code_map(&ma, a.a_codes, a.M, a.K, BM)) return cudaErrorInvalidValue;
  if (!make_code_map(&mw, a.w_codes, a.N, a.K, BN)) return cudaErrorInvalidValue;
  Params p;
  p.a_scales = a.a_scales;
  p.w_scales = a.w_scales;
  p.g_a = a.g_a;
  p.g_w = a.g_w;
  p.C = a.C;
  p.ldc = a.ldc;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.m_tiles = (a.M + BM - 1) / BM;
  p.n_tiles = (a.N + BN - 1) / BN;
  p.k_steps = (a.K + BK - 1) / BK;
  p.ncb = ncb_of(nsf_of(a.K, a.fmt));
  p.w_rowblocks = (a.N + 127) / 128;
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = std::max(1, std::min(tiles, sm_count()));
  if (a.fmt == 0)
    return a.out_f32 ? launch_typed<0, 1>(ma, mw, p, grid, s) : launch_typed<0, 0>(ma, mw, p, grid, s);
  return a.out_f32 ? launch_typed<1, 1>(ma, mw, p, grid, s) : launch_typed<1, 0>(ma, mw, p, grid, s);
}

}  // namespace fp4
