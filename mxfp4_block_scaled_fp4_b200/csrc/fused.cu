// fused.cu -- small-M (decode) W4A4 path behind fp4_gemm_fused.
//
// "FP4 n'existe pas", runtime survey: quantization, scaling, matmul and
// de-scaling chained without a host round trip; the small-M regime cuBLAS
// refuses: "Hardware FP4 inference for speech on Blackwell", section "Do the
// FP4 tensor cores even engage?".  Same arithmetic as fp4_quantize_act
// followed by fp4_gemm (bit-identical codes and scales), up to FP32
// summation order.
//
// One call is a chain of programmatic dependent launches on one stream:
//   amax      (DYNAMIC global scale only) per-CTA partial maxima;
//   quantize  the activation once, into the workspace: packed codes
//             [M, K/2] and scales in the MMA order (the stand-alone
//             quantizer kernels);
//   main      swap-AB tcgen05 GEMM: the weights are the 128-row "A" operand
//             of tcgen05.mma kind::mxf4nvf4, the <= 32 activation rows the
//             16- or 32-wide "B" operand.  Grid = N/128 weight tiles x S
//             split-K slices, S chosen so the grid fits one wave.
// Every kernel releases its dependent at once and waits for its predecessor
// (griddepcontrol.wait) before reading what that one wrote, so the main
// kernel streams its first weight stages while the activation is still
// being quantized.
//
// Quantizing inside every weight-tile CTA instead (an earlier version) made
// the activation's quantization N/128 times redundant; measured on B200 it
// cost more than the weight stream for M >= 8.
//
// Main kernel, per CTA:
//   warp 0     TMA: per 256-K stage the weight tile (16 KiB, 128-byte
//              swizzle), its scale atoms, the activation tile (rows >= M
//              read as zeros) and its scale atoms, through a 4-stage ring;
//   warp 1     MMA issuer (4 MMAs of K = 64 per stage);
//   warps 2-5  move each stage's weight and activation scales into tensor
//              memory (tcgen05.st; every scale address is 4-column aligned),
//              then the epilogue.
//   With S > 1 slices the S CTAs of a weight tile form a thread-block
//   cluster: each leaves its FP32 partial in shared memory and CTA s sums
//   rows m = s, s + S, ... over the S partials in slice order through
//   distributed shared memory (deterministic, no global round trip).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "launch_shape.h"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int FBM = 128;                 // weight rows per tile
constexpr int FBK = 256;                 // K per ring stage
constexpr int FBK_BYTES = FBK / 2;
constexpr int FSTAGES = 4;
constexpr int FW_STAGE = FBM * FBK_BYTES;   // 16 KiB weight codes
constexpr int FSF_STAGE = 4 * 512;          // up to 4 scale atoms (weights or activation)
constexpr int FX_STAGE = 32 * FBK_BYTES;    // activation codes, up to 32 rows
constexpr int kMaxSplits = 8;               // portable cluster size
constexpr int kFusedThreads = 192;          // TMA, MMA, 4 worker warps
constexpr int SMEM_BYTES =
    1024 + FSTAGES * (FW_STAGE + 2 * FSF_STAGE + FX_STAGE) + 256;   // two CTAs fit an SM
// Tensor-memory columns; every scale-factor address an MMA gets is a
// multiple of 4 columns (16 bytes): a misaligned-address fault was seen on
// B200 when scales sat at columns 4i + k.
constexpr uint32_t F_TMEM_COLS = 256;
constexpr uint32_t F_ACC_COL = 0;           // <= 32 fp32 columns
constexpr uint32_t F_SFA_COL = 32;          // weight scales: 16 columns per stage
constexpr uint32_t F_SFB_COL = 96;          // activation scales: 16 columns per stage

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

struct Plan {
  int n_tiles, k_steps, splits, nmma_n;
  size_t off_partial, off_codes, off_scales, ws_bytes;
};

// Split count: the largest S <= 8 (one cluster) whose grid fits one wave of
// two CTAs per SM.
Plan make_plan(int M, int N, int K, int fmt, int sms) {
  Plan p{};
  p.n_tiles = (N + FBM - 1) / FBM;
  p.k_steps = (K + FBK - 1) / FBK;
  p.nmma_n = M <= 16 ? 16 : 32;
  static_assert(kMaxSplits == 8, "chain_splits assumes portable clusters of 8");
  const int s = chain_splits(M, p.n_tiles, p.k_steps, sms);
  p.splits = s;
  const int nsf = nsf_of(K, fmt);
  p.off_partial = 0;
  p.off_codes = align256(static_cast<size_t>(kAmaxSlots) * sizeof(unsigned));
  p.off_scales = p.off_codes + align256(static_cast<size_t>(M) * (K / 2));
  p.ws_bytes = p.off_scales + align256(static_cast<size_t>(ncb_of(nsf)) * 512);
  return p;
}

struct FParams {
  const uint8_t* w_scales;
  const uint8_t* x_scales;   // activation scales, MMA order (one 128-row block)
  const float* g_w;
  const float* g_a;
  void* C;
  long long ldc;
  int M, N, K;
  int out_f32;
  int n_tiles, k_steps, splits, nmma_n, ncb;
  unsigned* watchdog;
};

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void workers_sync() {   // named barrier of the 4 worker warps
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
__device__ __forceinline__ float ld_peer_f32(uint32_t local_saddr, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_saddr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote));
  return v;
}

__device__ __forceinline__ void store_out(const FParams& p, int m, int n, float c) {
  if (p.out_f32)
    static_cast<float*>(p.C)[m * p.ldc + n] = c;
  else
    static_cast<__nv_bfloat16*>(p.C)[m * p.ldc + n] = __float2bfloat16_rn(c);
}

template <int FMT>
__global__ void __launch_bounds__(kFusedThreads, 1)
    small_m_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                   const FParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sW = smem;                                    // FSTAGES x 16 KiB
  uint8_t* sX = sW + FSTAGES * FW_STAGE;                 // FSTAGES x 4 KiB (1024-aligned)
  uint8_t* sWS = sX + FSTAGES * FX_STAGE;                // weight scale atoms
  uint8_t* sXS = sWS + FSTAGES * FSF_STAGE;              // activation scale atoms
  uint64_t* full = reinterpret_cast<uint64_t*>(sXS + FSTAGES * FSF_STAGE);
  uint64_t* empty = full + FSTAGES;
  uint64_t* sf_full = empty + FSTAGES;
  uint64_t* acc_full = sf_full + FSTAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / p.splits, split = blockIdx.x % p.splits;
  const int s_lo = static_cast<int>(static_cast<long long>(split) * p.k_steps / p.splits);
  const int s_hi = static_cast<int>(static_cast<long long>(split + 1) * p.k_steps / p.splits);
  const int n_steps = s_hi - s_lo;
  constexpr int kAtoms = (FMT == 0) ? 4 : 2;   // scale atoms per 256 K
  const uint32_t x_bytes = static_cast<uint32_t>(p.nmma_n * FBK_BYTES);

  if (threadIdx.x == 0) {
    for (int s = 0; s < FSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 4);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_w);
    prefetch_tensormap(&tm_x);
  }
  __syncthreads();
  // every CTA of this grid is resident: the next kernel in the stream may
  // launch now and start streaming its own weights
  grid_dep_launch();
  // warp 1 allocates tensor memory while warp 0 already streams weights;
  // warps 1-5 meet on named barrier 2 before using it
  uint32_t tmem = 0;
  if (warp >= 1) {
    if (warp == 1) {
      tmem_alloc(tmem_slot, F_TMEM_COLS);
      tmem_relinquish();
    }
    tc_fence_before();
    asm volatile("bar.sync 2, 160;" ::: "memory");
    tc_fence_after();
    tmem = *tmem_slot;
  }
  bool epilogue_ok = false;   // workers: the accumulator was read
  float alpha = 1.0f;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      // Weights do not depend on the preceding kernels; the activation does.
      // Issue the weights of the first stages, wait for the quantizer, then
      // stream weights and activation together.
      uint32_t armed = 0, armed_parity = 0;
      const int first = min(FSTAGES, n_steps);
      for (int i = 0; i < n_steps; ++i) {
        const int stage = i % FSTAGES;
        const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
        const int ks = s_lo + i;
        const int cb0 = ks * kAtoms;
        const int atoms = min(kAtoms, p.ncb - cb0);
        const uint32_t sf_bytes = static_cast<uint32_t>(atoms) * 512u;
        if (i >= first &&
            !mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER))
          break;
        // weight half of the stage
        mbar_expect_tx(&full[stage], FW_STAGE + x_bytes + 2u * sf_bytes);
        bulk_load(sWS + stage * FSF_STAGE,
                  p.w_scales + (static_cast<long long>(tile) * p.ncb + cb0) * 512, sf_bytes,
                  &full[stage]);
        tma_load_2d(sW + stage * FW_STAGE, &tm_w, ks * FBK_BYTES, tile * FBM, &full[stage]);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (i == first - 1) {
          // the ring is full and frees only as the MMAs consume it: the
          // slice's remaining weight tiles and scale atoms stream into L2
          // while the preceding kernels finish and the ring drains
          for (int j = first; j < n_steps; ++j) {
            const int ksj = s_lo + j, cbj = ksj * kAtoms;
            tma_prefetch_l2_2d(&tm_w, ksj * FBK_BYTES, tile * FBM);
            bulk_prefetch_l2(p.w_scales + (static_cast<long long>(tile) * p.ncb + cbj) * 512,
                             static_cast<uint32_t>(min(kAtoms, p.ncb - cbj)) * 512u);
          }
          // the quantized activation is produced by the preceding kernel
          grid_dep_wait();
          for (int j = 0; j < first; ++j) {
            const int ksj = s_lo + j, sj = j % FSTAGES;
            const int cbj = ksj * kAtoms;
            const uint32_t bj = static_cast<uint32_t>(min(kAtoms, p.ncb - cbj)) * 512u;
            bulk_load(sXS + sj * FSF_STAGE, p.x_scales + static_cast<long long>(cbj) * 512, bj,
                      &full[sj]);
            tma_load_2d(sX + sj * FX_STAGE, &tm_x, ksj * FBK_BYTES, 0, &full[sj]);
          }
        } else if (i >= first) {
          bulk_load(sXS + stage * FSF_STAGE, p.x_scales + static_cast<long long>(cb0) * 512,
                    sf_bytes, &full[stage]);
          tma_load_2d(sX + stage * FX_STAGE, &tm_x, ks * FBK_BYTES, 0, &full[stage]);
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < FSTAGES; ++s)
          if (armed & (1u << s)) mbar_wait_drain(&full[s], (armed_parity >> s) & 1u, p.watchdog);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      bool ok = true;
      for (int i = 0; i < n_steps && ok; ++i) {
        const int stage = i % FSTAGES;
        const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
        // one wait per step: the staging warps arrive on sf_full only after
        // the step's weight tile has landed (a test of an mbarrier is a
        // ~250-cycle round trip even when its phase has completed)
        ok = mbar_wait(&sf_full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL);
        if (!ok) break;
        tc_fence_after();
        const int kglob = (s_lo + i) * FBK;
        const int n_mma = min(4, (p.K - kglob + 63) / 64);
        const uint32_t w_s = smem_u32(sW + stage * FW_STAGE);
        const uint32_t x_s = smem_u32(sX + stage * FX_STAGE);
        const uint32_t sfa = tmem + F_SFA_COL + stage * 16;
        const uint32_t sfb = tmem + F_SFB_COL + stage * 16;
        for (int k = 0; k < n_mma; ++k) {
          const uint64_t ad = smem_desc(w_s + k * 32, 16, 1024, kLayoutSwizzle128B);
          const uint64_t bd = smem_desc(x_s + k * 32, 16, 1024, kLayoutSwizzle128B);
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          if (FMT == 0) {
            tc_mma_nvf4(tmem + F_ACC_COL, ad, bd, idesc_fp4(FBM, p.nmma_n, false, 0, 0),
                        sfa + 4 * k, sfb + 4 * k, acc);
          } else {
            const uint32_t id = 2u * (k & 1);
            tc_mma_mxf4(tmem + F_ACC_COL, ad, bd, idesc_fp4(FBM, p.nmma_n, true, id, id),
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
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    // Scales of each stage -> tensor memory.  Every quarter gets the 32-row
    // x 16-byte block of each atom (atom a at columns 4a..4a+3), the image
    // the MMA reads; the activation uses only its atoms' first 32 rows.
    for (int i = 0; i < n_steps; ++i) {
      const int stage = i % FSTAGES;
      const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait(&full[stage], phase, abort_flag, p.watchdog, WD_STAGING)))
        continue;
      const uint32_t ws = smem_u32(sWS + stage * FSF_STAGE) + lane * 16;
      const uint32_t xs = smem_u32(sXS + stage * FSF_STAGE) + lane * 16;
      uint32_t va[16], vb[16];
#pragma unroll
      for (int a = 0; a < kAtoms; ++a) {
        const uint4 x = lds128(ws + a * 512);
        va[4 * a] = x.x; va[4 * a + 1] = x.y; va[4 * a + 2] = x.z; va[4 * a + 3] = x.w;
        const uint4 y = lds128(xs + a * 512);
        vb[4 * a] = y.x; vb[4 * a + 1] = y.y; vb[4 * a + 2] = y.z; vb[4 * a + 3] = y.w;
      }
      if (kAtoms == 4) {
        tmem_st_x16(tmem + lane_off + F_SFA_COL + stage * 16, va);
        tmem_st_x16(tmem + lane_off + F_SFB_COL + stage * 16, vb);
      } else {
        tmem_st_x8(tmem + lane_off + F_SFA_COL + stage * 16, va);
        tmem_st_x8(tmem + lane_off + F_SFB_COL + stage * 16, vb);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[stage]);
    }
    // accumulator -> C directly (one slice) or -> this CTA's partial in
    // shared memory (several slices: the cluster reduces them below)
    {
      const bool done =
          __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, abort_flag, p.watchdog, WD_EPILOGUE));
      workers_sync();               // every worker warp reaches this barrier
      epilogue_ok = done && !*abort_flag;
    }
    // g_a comes from the quantizer (already finished: the producer waited
    // for it before loading the activation this accumulator was built from)
    grid_dep_wait();
    if (FMT == 0) alpha = __fmul_rn(*p.g_a, *p.g_w);
    if (epilogue_ok) {
      tc_fence_after();
      uint32_t r[32];
      const uint32_t taddr = tmem + lane_off + F_ACC_COL;
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
      const int nloc = quarter * 32 + lane;          // weight row within the tile
      const int n = tile * FBM + nloc;
      if (p.splits == 1) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < 32; ++m)
            if (m < p.M) store_out(p, m, n, __fmul_rn(alpha, __uint_as_float(r[m])));
        }
      } else {
        float* part = reinterpret_cast<float*>(sW);  // the ring is idle now
#pragma unroll
        for (int m = 0; m < 32; ++m)
          if (m < p.M) part[m * FBM + nloc] = __uint_as_float(r[m]);
      }
    }
  }

  if (p.splits > 1) {
    // every CTA of the tile's cluster has written its partial sums
    cluster_sync_all();
    if (warp >= 2 && epilogue_ok) {
      const int t = threadIdx.x - 64;
      const int n = tile * FBM + t;
      const uint32_t base = smem_u32(sW) + t * 4;
      // CTA `split` reduces rows m = split, split + S, ... in slice order
      // all S remote loads of a row are issued before the first add
      for (int m = split; m < p.M; m += p.splits) {
        float v[kMaxSplits];
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s)
          v[s] = (s < p.splits) ? ld_peer_f32(base + m * FBM * 4, static_cast<uint32_t>(s)) : 0.0f;
        float acc = 0.0f;
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s)
          if (s < p.splits) acc = __fadd_rn(acc, v[s]);
        if (n < p.N) store_out(p, m, n, __fmul_rn(alpha, acc));
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
    tmem_dealloc(tmem, F_TMEM_COLS);
  }
}

// ------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Packed codes [rows, K/2] as a 2-D uint8 tensor, boxes of 128 bytes x
// box_rows rows, 128-byte swizzle; out-of-range rows and columns read as 0.
bool make_map(CUtensorMap* m, const uint8_t* base, int rows, int K, int box_rows) {
  // the driver's encoder, looked up once (thread-safe static initialization)
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(FBK_BYTES), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fused_supported(int M, int N, int K) { return M >= 1 && M <= 32 && N >= 1 && K >= 1; }

size_t fused_workspace_bytes(int M, int N, int K, int fmt) {
  return make_plan(M, N, K, fmt, 1).ws_bytes;   // (independent of the split)
}

cudaError_t launch_gemm_fused(const FusedArgs& f, cudaStream_t s) {
  if (decode_supported(f.M, f.N, f.K, f.max_sms)) return launch_decode(f, s);
  const Plan pl = make_plan(f.M, f.N, f.K, f.fmt, gemm_sms(f.max_sms));
  uint8_t* ws = static_cast<uint8_t*>(f.ws);
  uint8_t* x_codes = ws + pl.off_codes;
  uint8_t* x_scales = ws + pl.off_scales;

  // 1-2: quantize the activation once (programmatic dependent launches)
  QuantArgs q{};
  q.x = f.a;
  q.rows = f.M;
  q.K = f.K;
  q.fmt = f.fmt;
  q.layout = 0;
  q.dynamic = f.dynamic;
  q.g = f.g_a;
  q.codes = x_codes;
  q.scales = x_scales;
  q.rot = f.rot;
  q.rot_scale = f.rot_scale;
  q.rule = f.rule;
  // scale columns past K of real rows are still zeroed (they meet zero codes,
  // and 0 x NaN would not be 0); rows >= M only reach output columns that
  // are never stored
  q.zero_pad_rows = 0;
  // the GEMM reads the quantized activation only after its wait
  q.release_early = 1;
  cudaError_t e = launch_quantize_act(q, reinterpret_cast<unsigned*>(ws + pl.off_partial), s);
  if (e != cudaSuccess) return e;

  // 3: the swap-AB GEMM
  FParams p{};
  p.w_scales = f.w_scales;
  p.x_scales = x_scales;
  p.g_w = f.g_w;
  p.g_a = f.g_a;
  p.C = f.C;
  p.ldc = f.ldc;
  p.M = f.M;
  p.N = f.N;
  p.K = f.K;
  p.out_f32 = f.out_f32;
  p.n_tiles = pl.n_tiles;
  p.k_steps = pl.k_steps;
  p.splits = pl.splits;
  p.nmma_n = pl.nmma_n;
  p.ncb = ncb_of(nsf_of(f.K, f.fmt));
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;
  CUtensorMap mw, mx;
  if (!make_map(&mw, f.w_codes, f.N, f.K, FBM)) return cudaErrorInvalidValue;
  if (!make_map(&mx, x_codes, f.M, f.K, pl.nmma_n)) return cudaErrorInvalidValue;
  auto kern = (f.fmt == 0) ? small_m_kernel<0> : small_m_kernel<1>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.n_tiles * pl.splits));
  cfg.blockDim = dim3(kFusedThreads);
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
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, mw, mx, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4
