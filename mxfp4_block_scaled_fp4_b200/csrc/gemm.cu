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
// Design (one CTA per SM; persistent over 128 x BN output tiles, BN = 256,
// 128 or 64, or one tile per cluster of CTAs that split K between them):
//   warp 0      one thread drives TMA: packed A / W tiles (128 B of K per
//               row, 128-byte swizzle) into a shared-memory ring;
//   warp 10     one thread loads the matching scale atoms (plain bulk
//               copies: in the MMA scale order a tile's scales for one K
//               step are contiguous) into the same ring stages;
//   warps 6-9   scale staging: each warp reads a stage's scale atoms from
//               shared memory and writes them with tcgen05.st into its own
//               32-lane quarter of the stage's scale region in tensor memory
//               (every quarter gets the whole 32-row x 16-byte block of an
//               atom, the image the MMA reads), waits for the stage's code
//               tiles and then marks the stage ready.  Moving scales with
//               warp stores instead of tcgen05.cp keeps the copies out of
//               the MMA pipe: measured on B200, even one tcgen05.cp per K
//               step stalled the MMAs of every step;
//   warp 1      one thread waits for ready stages (one barrier per stage:
//               a test of a completed mbarrier is itself a round trip of
//               about 250 cycles, half the tensor time of a stage), issues
//               tcgen05.mma kind::mxf4nvf4 (128 x BN x 64 per instruction)
//               into an FP32 accumulator in tensor memory and releases ring
//               stages with tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld the accumulator (one 32-lane quarter
//               per warp), multiply by alpha, round to bf16 / keep fp32,
//               store C (split K: exchange partial sums first, below).
// Every mbarrier wait is bounded; a wait that runs out sets the watchdog
// word, the CTA stops issuing, waits (bounded) for its copies and MMAs in
// flight, frees its tensor memory and returns.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cuda_bf16.h>

#include "groups.cuh"
#include "internal.h"
#include "launch_shape.h"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int BM = 128;
constexpr int BK = 256;                 // FP4 elements of K per ring stage
constexpr int BK_BYTES = BK / 2;        // 128: one 128-byte swizzle row
constexpr int MMA_K = 64;               // FP4 elements per tcgen05.mma
constexpr int A_STAGE = BM * BK_BYTES;  // 16 KiB
constexpr int SFA_STAGE = 4 * 512;      // up to 4 scale atoms (128 rows x 4 scales)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;         // up to 256 fp32 columns
constexpr uint32_t SF_COL = 256;        // per stage: 16 columns A scales + 16 or 32 B scales
constexpr int kGemmThreads = 352;       // 11 warps: TMA, MMA, 4 epilogue, 4 scale staging, scale TMA
constexpr int GROUP_M = 16;             // tile raster: 16 M-tiles share their W tiles in L2
constexpr int kMaxGroups = kGroupedMaxGroups;   // experts of a grouped launch

// Output tiles are 128 x BN.  BN = 256 is the throughput shape; 128 and 64
// give problems with few 256-wide tiles more CTAs (and smaller split-K
// partial sums to exchange).  A W tile's scales come from one 128-row scale
// block (two for BN = 256); for BN = 64 the tile is one half of it.  The
// ring is as deep as shared memory allows, so that narrow tiles keep as
// many bytes in flight as wide ones.
// G = 1: the grouped (mixture-of-experts) form: the same ring (a group's
// tiles start on a 128-row scale block, so a tile's A scales are one
// block's atoms), and the group table follows the barriers.
template <int BN, int G = 0>
struct Tile {
  static constexpr int B_STAGE = BN * BK_BYTES;
  static constexpr int SF_BLOCKS = (BN == 256) ? 2 : 1;
  static constexpr int SFB_STAGE = SF_BLOCKS * 4 * 512;
  static constexpr int SFA_BYTES = SFA_STAGE;
  static constexpr int STAGE_BYTES = A_STAGE + B_STAGE + SFA_BYTES + SFB_STAGE;
  static constexpr int STAGES = (BN == 256) ? 4 : (BN == 128) ? 6 : 7;
  static constexpr int RING = STAGES * STAGE_BYTES;
  static constexpr int GCAP = kMaxGroups;
  static constexpr int GTAB = G ? 4 * (2 * GCAP + 2) : 0;   // group table (ints)
  static constexpr int RTAB = G ? 0 : 512;                   // reciprocals of the FP4 epilogue
  static constexpr int SMEM = RING + 1024 + 512 + GTAB + RTAB;   // ring, alignment, barriers,
                                                                 // groups, reciprocals
  // tensor-memory columns between the B scales of consecutive atoms, and
  // per stage (A scales in the first 16)
  static constexpr int SFB_ATOM_COLS = 4 * SF_BLOCKS;
  static constexpr uint32_t SF_STAGE_COLS = 16 + 16 * SF_BLOCKS;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(SF_COL + STAGES * SF_STAGE_COLS <= TMEM_COLS, "tensor memory");
  static_assert(STAGES * 4 * 8 + 4 * 8 + 8 <= 512, "barrier area");
  // split-K partial sums of S <= 8 splits, S * ceil(128 / S) rows, in the ring
  static_assert((BM + 7) * BN * 4 <= RING, "split-K exchange area");
};

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
  int splits;             // CTAs per output tile along K (a cluster), 1 = no split
  int k_per;              // K steps per split
  unsigned* watchdog;
  // grouped form (G = 1): E groups; group e is rows [offsets[e], offsets[e+1])
  // of A and C and weights rows [e N, e N + N) of the stacked W, whose
  // scales start at byte e * w_sf_bytes; g_w holds one global scale per group
  const int* offsets;
  int E;
  long long w_sf_bytes;
  int a_rowblocks;        // ceil(M / 128)
  QuantOut qo;            // OUT 2, 3: the emitted FP4 activation (C optional)
  const float* sigma_a;   // OUT 4, 5: macro-block scales of A rows [M] and W rows [N]
  const float* sigma_w;
};

// Split-K: CTA d of a tile's cluster reduces accumulator rows
// [row_begin(d), row_begin(d + 1)).
__device__ __forceinline__ int row_begin(int d, int S) { return d * BM / S; }
__device__ __forceinline__ int row_owner(int r, int S) { return ((r + 1) * S - 1) / BM; }

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mt, int& nt) {
  const int per_group = GROUP_M * p.n_tiles;
  const int group = t / per_group;
  const int first_m = group * GROUP_M;
  const int gsize = min(GROUP_M, p.m_tiles - first_m);
  const int within = t - group * per_group;
  mt = first_m + within % gsize;
  nt = within / gsize;
}

// alpha * 8 accumulator values -> 8 bf16 (one 16-byte store) / 2 float4.
template <int OUT_F32>
__device__ __forceinline__ void store8(void* C, long long off, float alpha, const float* v) {
  if (!OUT_F32) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(alpha, v[2 * j]), __fmul_rn(alpha, v[2 * j + 1]));
      w[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(C) + off) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(C) + off);
    o[0] = make_float4(__fmul_rn(alpha, v[0]), __fmul_rn(alpha, v[1]), __fmul_rn(alpha, v[2]),
                       __fmul_rn(alpha, v[3]));
    o[1] = make_float4(__fmul_rn(alpha, v[4]), __fmul_rn(alpha, v[5]), __fmul_rn(alpha, v[6]),
                       __fmul_rn(alpha, v[7]));
  }
}

// OUT: 0 = bf16 C, 1 = fp32 C, 2 / 3 = C quantized to NVFP4 / MXFP4
// (out_quant.cuh; no K split), with the bf16 C stored as well when p.C is
// not null; 4 / 5 = bf16 / fp32 C scaled by sigma_a[m] sigma_w[n] (MXFP4
// macro-block scaling; no K split) instead of alpha.
template <int FMT, int OUT, int BN, int G = 0>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                const Params p) {
  using T = Tile<BN, G>;
  constexpr int SFA_STAGE = T::SFA_BYTES;
  constexpr int STAGES = T::STAGES;
  constexpr uint32_t SF_STAGE_COLS = T::SF_STAGE_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE;
  uint8_t* sSFA = sB + STAGES * T::B_STAGE;
  uint8_t* sSFB = sSFA + STAGES * SFA_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * T::SFB_STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_loaded = empty + STAGES;
  uint64_t* ready = sf_loaded + STAGES;
  uint64_t* acc_full = ready + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* recv = drain + 1;          // split-K: partial sums pushed by the peers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* gtab = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + 512);   // G = 1
  float* r_tab = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 512 + T::GTAB);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int n_tiles_total = p.m_tiles * p.n_tiles;
  // split-K: one tile per cluster, CTA rank = its slice of the K steps;
  // otherwise persistent over the tiles with all K steps
  const bool split = p.splits > 1;
  const int S = p.splits;
  const int me = split ? static_cast<int>(cluster_ctarank()) : 0;
  const int t_first = split ? static_cast<int>(blockIdx.x) / S : static_cast<int>(blockIdx.x);
  const int t_stride = split ? n_tiles_total : static_cast<int>(gridDim.x);
  const int kb0 = me * p.k_per;
  const int kb1 = min(p.k_steps, kb0 + p.k_per);
  // split-K partial sums exchanged: rows below M, columns below N of the tile
  int rows_valid = 0, cols_valid = 0;
  if (split) {
    int mt, nt;
    tile_coords(t_first, p, mt, nt);
    rows_valid = min(BM, p.M - mt * BM);
    cols_valid = min(BN, p.N - nt * BN);
  }
  // split-K exchange: rows of one split's partial sums per owner, rounded up
  const int r_slot = (BM + S - 1) / S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_loaded[s], 1);
      mbar_init(&ready[s], 4);   // one arrival per scale-staging warp
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);   // one arrival per epilogue warp
    mbar_init(drain, 1);
    mbar_init(recv, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (split) {
      const int mine = max(0, min(row_begin(me + 1, S), rows_valid) - row_begin(me, S));
      mbar_expect_tx(recv, static_cast<uint32_t>((S - 1) * mine * cols_valid * 4));
    }
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
  // Programmatic dependent launch: the next kernel of the stream may be
  // scheduled from here on (every kernel of this library waits for its
  // predecessor before reading what that one wrote), and this kernel's
  // setup above overlapped its predecessor's tail; all its global reads and
  // writes come after the wait.  Without such a launch both are no-ops.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (G) {
    // the group table from the device-side offsets (groups.cuh)
    if (warp == 0) build_group_table<T::GCAP>(p.offsets, p.E, p.M, BM, gtab, lane);
    __syncthreads();
    n_tiles_total = gtab[p.E] * p.n_tiles;
  }
  float alpha = 1.0f;
  if (FMT == 0 && warp >= 2 && warp < 6 && !G) alpha = __fmul_rn(*p.g_a, *p.g_w);
  constexpr bool F32 = OUT == 1 || OUT == 5;       // fp32 C
  constexpr bool QOUT = OUT == 2 || OUT == 3;      // FP4 activation out
  constexpr bool MBS = OUT >= 4;                   // per-row x per-column scales
  QuantOutG qg{};
  if (QOUT && warp >= 2 && warp < 6) {
    qg = quant_out_g(p.qo, r_tab, threadIdx.x - 64);
    asm volatile("bar.sync 1, 128;" ::: "memory");   // the 4 epilogue warps
  }
  bool acc_ok = false;   // split-K epilogue: this CTA's accumulator is complete

  constexpr int kAtomsPerStage = (FMT == 0) ? 4 : 2;   // scale atoms per 256 K

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    for (int t = t_first; t < n_tiles_total; t += t_stride) {
      int mt, nt, a_row0, w_row0;
      if (G) {
        const GTile g = gtile<T::GCAP>(t, p.E, p.n_tiles, BM, gtab, GROUP_M);
        nt = g.nt;
        a_row0 = g.a_row0;
        w_row0 = g.e * p.N + nt * BN;
      } else {
        tile_coords(t, p, mt, nt);
        a_row0 = mt * BM;
        w_row0 = nt * BN;
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER)) goto producer_drain;
        {
          mbar_expect_tx(&full[stage], A_STAGE + T::B_STAGE);
          tma_load_2d(sA + stage * A_STAGE, &tm_a, kb * BK_BYTES, a_row0, &full[stage]);
          tma_load_2d(sB + stage * T::B_STAGE, &tm_w, kb * BK_BYTES, w_row0, &full[stage]);
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
        mbar_wait_drain(&full[s], (armed_parity >> s) & 1u, p.watchdog);
      }
  producer_done:;
  } else if (warp == 10 && lane == 0) {
    // ------------------------------------------------ scale producer
    // The scale atoms of a stage (contiguous in the MMA scale order) by
    // plain bulk copies, on their own barrier so that staging them into
    // tensor memory overlaps the code tiles' flight.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    for (int t = t_first; t < n_tiles_total; t += t_stride) {
      int mt, nt;
      int arb;                          // A scale row block of the tile
      const int ablocks = 1;
      const uint8_t* wsf = p.w_scales;  // this tile's weight scales
      if (G) {
        const GTile g = gtile<T::GCAP>(t, p.E, p.n_tiles, BM, gtab, GROUP_M);
        nt = g.nt;
        arb = g.a_row0 / BM;
        wsf += static_cast<long long>(g.e) * p.w_sf_bytes;
      } else {
        tile_coords(t, p, mt, nt);
        arb = mt;
      }
      const int rb0 = nt * BN / 128;
      const int wblocks = min(T::SF_BLOCKS, p.w_rowblocks - rb0);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER)) goto sf_drain;
        {
          const int cb0 = kb * kAtomsPerStage;
          const int atoms = min(kAtomsPerStage, p.ncb - cb0);
          const uint32_t sf_bytes = static_cast<uint32_t>(atoms) * 512u;
          mbar_expect_tx(&sf_loaded[stage], sf_bytes * (ablocks + wblocks));
          for (int i = 0; i < ablocks; ++i)
            bulk_load(sSFA + stage * SFA_STAGE + i * kAtomsPerStage * 512,
                      p.a_scales + (static_cast<long long>(arb + i) * p.ncb + cb0) * 512, sf_bytes,
                      &sf_loaded[stage]);
          for (int i = 0; i < wblocks; ++i)
            bulk_load(sSFB + stage * T::SFB_STAGE + i * 2048,
                      wsf + (static_cast<long long>(rb0 + i) * p.ncb + cb0) * 512, sf_bytes,
                      &sf_loaded[stage]);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    goto sf_done;
  sf_drain:
    for (int s = 0; s < STAGES; ++s)
      if (armed & (1u << s)) mbar_wait_drain(&sf_loaded[s], (armed_parity >> s) & 1u, p.watchdog);
  sf_done:;
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    for (int t = t_first; t < n_tiles_total; t += t_stride, ++it) {
      if (it > 0 && !mbar_wait(acc_empty, static_cast<uint32_t>(it - 1) & 1u, abort_flag, p.watchdog, WD_MMA_ACC))
        goto mma_drain;
      tc_fence_after();
      for (int kb = kb0; kb < kb1; ++kb) {
        // one wait per stage: the staging warps arrive on ready[] only once
        // the stage's code tiles have landed and its scales are in tensor
        // memory (a completed-barrier test alone is a ~250-cycle round trip)
        if (!mbar_wait(&ready[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL)) goto mma_drain;
        tc_fence_after();
        {
          const int n_mma = min(BK / MMA_K, (p.K - kb * BK + MMA_K - 1) / MMA_K);
          const uint32_t sfa_t = tmem + SF_COL + stage * SF_STAGE_COLS;
          const uint32_t sfb_t = sfa_t + 16;
          // descriptors of the stage's first K slice; the next slice starts
          // 32 bytes further (2 in the address field)
          const uint64_t ad0 = smem_desc(smem_u32(sA + stage * A_STAGE), 16, 1024, kLayoutSwizzle128B);
          const uint64_t bd0 = smem_desc(smem_u32(sB + stage * T::B_STAGE), 16, 1024, kLayoutSwizzle128B);
          const uint32_t acc0 = (kb > kb0) ? 1u : 0u;
          auto mma = [&](int k) {
            const uint32_t acc = (k > 0) ? 1u : acc0;
            if (FMT == 0) {
              tc_mma_nvf4(tmem + ACC_COL, ad0 + 2 * k, bd0 + 2 * k, idesc_fp4(BM, BN, false, 0, 0),
                          sfa_t + 4 * k, sfb_t + T::SFB_ATOM_COLS * k, acc);
            } else {
              const uint32_t id = 2u * (k & 1);
              tc_mma_mxf4(tmem + ACC_COL, ad0 + 2 * k, bd0 + 2 * k, idesc_fp4(BM, BN, true, id, id),
                          sfa_t + 4 * (k >> 1), sfb_t + T::SFB_ATOM_COLS * (k >> 1), acc);
            }
          };
          if (n_mma == BK / MMA_K) {
#pragma unroll
            for (int k = 0; k < BK / MMA_K; ++k) mma(k);
          } else {
            for (int k = 0; k < n_mma; ++k) mma(k);
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
  } else if (warp >= 6 && warp < 10) {
    // ----------------------------------------------------- scale staging
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = t_first; t < n_tiles_total; t += t_stride) {
      int mt, nt;
      if (G) {
        nt = gtile<T::GCAP>(t, p.E, p.n_tiles, BM, gtab, GROUP_M).nt;
      } else {
        tile_coords(t, p, mt, nt);
      }
      // BN = 64: the tile is rows 64 (nt & 1) .. +63 of its scale block,
      // words 2 (nt & 1) and 2 (nt & 1) + 1 of each 16-byte atom row
      const int half = (BN == 64) ? (nt & 1) : 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        // warp-uniform outcome: tcgen05.st below needs all 32 lanes
        if (!__all_sync(0xFFFFFFFFu,
                        mbar_wait(&sf_loaded[stage], phase, abort_flag, p.watchdog, WD_STAGING)))
          goto staging_done;
        {
          const uint32_t sfa_s = smem_u32(sSFA + stage * SFA_STAGE) + lane * 16;
          const uint32_t sfb_s = smem_u32(sSFB + stage * T::SFB_STAGE) + lane * 16;
          const uint32_t sfa_t = tmem + lane_off + SF_COL + stage * SF_STAGE_COLS;
          const uint32_t sfb_t = sfa_t + 16;
          // atom a, row `lane`: 16 bytes = 4 columns; A at columns 4a..4a+3,
          // W scale block rb at columns SFB_ATOM_COLS a + 4 rb .. + 3
          uint32_t va[4 * kAtomsPerStage], vb[4 * T::SF_BLOCKS * kAtomsPerStage];
#pragma unroll
          for (int a = 0; a < kAtomsPerStage; ++a) {
            {
              const uint4 x = lds128(sfa_s + a * 512);
              va[4 * a + 0] = x.x; va[4 * a + 1] = x.y; va[4 * a + 2] = x.z; va[4 * a + 3] = x.w;
            }
#pragma unroll
            for (int rb = 0; rb < T::SF_BLOCKS; ++rb) {
              const uint4 y = lds128(sfb_s + rb * 2048 + a * 512);
              uint32_t* o = vb + T::SFB_ATOM_COLS * a + 4 * rb;
              if (BN == 64) {
                o[0] = half ? y.z : y.x; o[1] = half ? y.w : y.y; o[2] = 0u; o[3] = 0u;
              } else {
                o[0] = y.x; o[1] = y.y; o[2] = y.z; o[3] = y.w;
              }
            }
          }
          if (kAtomsPerStage == 4) {
            tmem_st_x16(sfa_t, va);
            if (T::SF_BLOCKS == 2) tmem_st_x32(sfb_t, vb); else tmem_st_x16(sfb_t, vb);
          } else {
            tmem_st_x8(sfa_t, va);
            if (T::SF_BLOCKS == 2) tmem_st_x16(sfb_t, vb); else tmem_st_x8(sfb_t, vb);
          }
          tmem_st_wait();
        }
        // the stage is ready for the MMAs once its code tiles have landed too
        if (!__all_sync(0xFFFFFFFFu,
                        mbar_wait(&full[stage], phase, abort_flag, p.watchdog, WD_STAGING)))
          goto staging_done;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ready[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  staging_done:;
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;        // tensor-memory lanes this warp may read
    if (split) {
      // one tile; the reduction across the cluster follows below
      acc_ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, abort_flag, p.watchdog, WD_EPILOGUE));
      tc_fence_after();
    } else {
      int it = 0;
      for (int t = t_first; t < n_tiles_total; t += t_stride, ++it) {
        int mt, nt, row, row_begin = 0, row_end = p.M;
        if (G) {
          const GTile g = gtile<T::GCAP>(t, p.E, p.n_tiles, BM, gtab, GROUP_M);
          nt = g.nt;
          row = g.a_row0 + quarter * 32 + lane;
          row_begin = g.a_row_begin;
          row_end = g.a_row_end;
          if (FMT == 0) alpha = __fmul_rn(*p.g_a, p.g_w[g.e]);
        } else {
          tile_coords(t, p, mt, nt);
          row = mt * BM + quarter * 32 + lane;
        }
        // warp-uniform outcome: tcgen05.ld below needs all 32 lanes
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag,
                                               p.watchdog, WD_EPILOGUE)))
          break;
        tc_fence_after();
        const bool row_ok = row >= row_begin && row < row_end;
        const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + ACC_COL;
        const float arow = MBS ? __ldg(p.sigma_a + min(row, p.M - 1)) : alpha;
        if (!F32) {
          // bf16: the whole row fits in registers once packed, so the
          // accumulator is released before any global store is issued
          uint32_t packed[BN / 2];
#pragma unroll
          for (int c = 0; c < BN / 16; ++c) {
            uint32_t r[16];
            FP4_TMEM_LD_32x32b_X16(tbase + c * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int n = nt * BN + 16 * c + 2 * j;
              const float lo =
                  __fmul_rn(col_scale<MBS>(arow, p.sigma_w, n, p.N), __uint_as_float(r[2 * j]));
              const float hi =
                  __fmul_rn(col_scale<MBS>(arow, p.sigma_w, n + 1, p.N), __uint_as_float(r[2 * j + 1]));
              __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
              packed[8 * c + j] = *reinterpret_cast<uint32_t*>(&h);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty);
          if (QOUT) {
            const bool pad = p.qo.layout == 0 && !row_ok && row < (p.M + 127) / 128 * 128;
            quant_out_row<BN, QOUT ? OUT - 2 : 0>(p.qo, qg, packed, row, row_ok, pad, nt * BN, p.N);
          }
          if (row_ok && (!QOUT || p.C != nullptr)) {
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
                const int n = n0 + 4 * v;
                float4 o;
                o.x = __fmul_rn(col_scale<MBS>(arow, p.sigma_w, n, p.N), __uint_as_float(r[4 * v + 0]));
                o.y = __fmul_rn(col_scale<MBS>(arow, p.sigma_w, n + 1, p.N), __uint_as_float(r[4 * v + 1]));
                o.z = __fmul_rn(col_scale<MBS>(arow, p.sigma_w, n + 2, p.N), __uint_as_float(r[4 * v + 2]));
                o.w = __fmul_rn(col_scale<MBS>(arow, p.sigma_w, n + 3, p.N), __uint_as_float(r[4 * v + 3]));
                *reinterpret_cast<float4*>(out + 4 * v) = o;
              }
            }
          }
        }
      }
    }
  }

  if (split) {
    // Split-K reduction.  Every CTA of the cluster holds the partial sums of
    // its K slice for the whole tile; CTA d owns accumulator rows
    // [row_begin(d), row_begin(d + 1)).  Each epilogue thread reads its
    // row's partial sums from tensor memory once and writes them into the
    // row owner's (now idle) ring: with st.async into a peer, with plain
    // stores into its own CTA.  Then all 128 epilogue threads of the owner
    // share out its rows x 8-column groups, add the S partials in split
    // order 0..S-1 (a fixed order, so the result does not depend on
    // timing), scale by alpha and store C.  Partials from split src: the
    // 16-byte column group c4 of owned row lr at
    // ring + ((src * BN/4 + c4) * r_slot + lr) * 16.
    __syncwarp();
    cluster_sync_all();   // every CTA's MMAs and copies done: rings free
    if (warp >= 2 && warp < 6) {
      const int quarter = warp & 3;
      const int tid = threadIdx.x - 64;             // 0..127 over the epilogue warps
      int mt, nt;
      tile_coords(t_first, p, mt, nt);
      const uint32_t ring = smem_u32(sA);
      const uint32_t bar = smem_u32(recv);
      const int groups = cols_valid / 4;            // 16-byte column groups stored
      const int lo = row_begin(me, S), hi = min(row_begin(me + 1, S), rows_valid);
      if (acc_ok) {
        // 1) every row's partial sums to the row's owner
        const int r = quarter * 32 + lane;          // accumulator row (tensor-memory lane)
        const bool row_ok = r < rows_valid;
        const int owner = row_owner(r, S);
        const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + ACC_COL;
        const uint32_t off = static_cast<uint32_t>(
            (me * (BN / 4) * r_slot + (r - row_begin(owner, S))) * 16);
        const uint32_t dst = (owner == me ? ring : map_to_rank(ring, static_cast<uint32_t>(owner))) + off;
        const uint32_t dbar = map_to_rank(bar, static_cast<uint32_t>(owner));
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          FP4_TMEM_LD_32x32b_X32(tbase + c * 32, v);
          tmem_ld_wait();
          if (!row_ok) continue;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (c * 8 + j >= groups) break;
            const uint32_t d = dst + static_cast<uint32_t>((c * 8 + j) * r_slot * 16);
            if (owner != me)
              st_async_v4(d, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3], dbar);
            else
              sts128(d, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
        }
      }
      // own rows written by all four warps; peers' rows by their st.async
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const bool got = acc_ok && hi > lo &&
                       __all_sync(0xFFFFFFFFu, mbar_wait(recv, 0, abort_flag, p.watchdog, WD_EPILOGUE));
      if (!got && hi > lo && tid == 0) {
        // unwinding: the peers' pushes may still be in flight into this
        // CTA's shared memory; let them land (bounded) before it goes away
        mbar_wait_drain(recv, 0, p.watchdog);
      }
      if (got) {
        // 2) the owned rows: (row, 8-column group) units shared out, rows
        // fastest so that a warp's shared-memory reads are contiguous
        const int rows = hi - lo;
        const int units = rows * (groups / 2);
        for (int u = tid; u < units; u += 128) {
          const int lr = u % rows, g = u / rows;
          float acc[8];
#pragma unroll 1
          for (int src = 0; src < S; ++src) {
            const uint32_t a = ring + static_cast<uint32_t>(((src * (BN / 4) + 2 * g) * r_slot + lr) * 16);
            const uint4 y0 = lds128(a);
            const uint4 y1 = lds128(a + r_slot * 16);
            const float x[8] = {__uint_as_float(y0.x), __uint_as_float(y0.y), __uint_as_float(y0.z),
                                __uint_as_float(y0.w), __uint_as_float(y1.x), __uint_as_float(y1.y),
                                __uint_as_float(y1.z), __uint_as_float(y1.w)};
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = (src == 0) ? x[i] : __fadd_rn(acc[i], x[i]);
          }
          store8<F32>(p.C, (static_cast<long long>(mt) * BM + lo + lr) * p.ldc + nt * BN + 8 * g,
                          alpha, acc);
        }
      }
    }
    __syncwarp();
    cluster_sync_all();   // no CTA leaves while a peer may still write to it
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

// The driver's tensor-map encoder, looked up once (a function-local static
// is initialized once even when threads race to the first call).
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
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

bool make_f32_out_map(CUtensorMap* m, void* C, long long rows, int cols, int ldc, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldc) * 4};
  cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, C, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

template <int FMT, int OUT, int BN, int G = 0>
cudaError_t launch_typed(const CUtensorMap& ma, const CUtensorMap& mw, const Params& p, int grid,
                         cudaStream_t s) {
  auto kern = gemm_kernel<FMT, OUT, BN, G>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile<BN, G>::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (p.splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.splits;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = Tile<BN, G>::SMEM;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, ma, mw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Clusters of `size` CTAs of the BN-wide kernel that fit on the device at
// once (cached per device, width and size; 0 when the query fails).
template <int BN>
int max_clusters(int size) {
  static std::atomic<int> cache[64][9] = {};
  int dev = 0;
  if (size < 2 || size > 8 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int c = cache[dev][size].load(std::memory_order_relaxed);
  if (c == 0) {
    auto kern = gemm_kernel<0, 0, BN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile<BN>::SMEM) !=
        cudaSuccess)
      return 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = size;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(size);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = Tile<BN>::SMEM;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      return 0;
    }
    c = n > 0 ? n : -1;
    cache[dev][size].store(c, std::memory_order_relaxed);
  }
  return c > 0 ? c : 0;
}

int max_clusters_bn(int bn, int size) {
  return bn == 256 ? max_clusters<256>(size) : bn == 128 ? max_clusters<128>(size)
                                                         : max_clusters<64>(size);
}

template <int BN>
cudaError_t launch_bn(const GemmArgs& a, Params p, int splits, cudaStream_t s) {
  const int sms = gemm_sms(a.max_sms);
  CUtensorMap ma, mw;
  if (!make_code_map(&ma, a.a_codes, a.M, a.K, BM)) return cudaErrorInvalidValue;
  if (!make_code_map(&mw, a.w_codes, a.N, a.K, BN)) return cudaErrorInvalidValue;
  p.n_tiles = (a.N + BN - 1) / BN;
  p.splits = splits;
  p.k_per = (p.k_steps + splits - 1) / splits;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = (splits > 1) ? tiles * splits : std::max(1, std::min(tiles, sms));
  using L = cudaError_t (*)(const CUtensorMap&, const CUtensorMap&, const Params&, int,
                            cudaStream_t);
  static const L table[2][4] = {
      {launch_typed<0, 0, BN>, launch_typed<0, 1, BN>, launch_typed<0, 2, BN>, launch_typed<0, 3, BN>},
      {launch_typed<1, 0, BN>, launch_typed<1, 1, BN>, launch_typed<1, 2, BN>, launch_typed<1, 3, BN>}};
  if (a.out_mode >= 4) {   // macro-block scaling: MXFP4 only
    if (a.fmt != 1) return cudaErrorInvalidValue;
    return a.out_mode == 5 ? launch_typed<1, 5, BN>(ma, mw, p, grid, s)
                           : launch_typed<1, 4, BN>(ma, mw, p, grid, s);
  }
  return table[a.fmt != 0][a.out_mode](ma, mw, p, grid, s);
}

}  // namespace

int gemm_sms(int max_sms) {
  const int sms = sm_count();
  return (max_sms > 0 && max_sms < sms) ? max_sms : sms;
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s) {
  const int sms = gemm_sms(a.max_sms);
  if (takes_pair(a.M, a.N, sms)) return launch_gemm_pair(a, s);
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
  p.k_steps = (a.K + BK - 1) / BK;
  p.ncb = ncb_of(nsf_of(a.K, a.fmt));
  p.w_rowblocks = (a.N + 127) / 128;
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;
  p.qo = a.qo;
  p.sigma_a = a.sigma_a;
  p.sigma_w = a.sigma_w;
  // the FP4-emitting and the macro-block-scaled epilogues take no K split
  const Shape sh = choose_shape(p.m_tiles, a.N, p.k_steps, sms, max_clusters_bn, a.out_mode < 2);
  if (sh.bn == 64) return launch_bn<64>(a, p, sh.splits, s);
  if (sh.bn == 128) return launch_bn<128>(a, p, sh.splits, s);
  return launch_bn<256>(a, p, sh.splits, s);
}

cudaError_t launch_gemm_grouped(const GroupedArgs& a, cudaStream_t s) {
  const int sms = gemm_sms(a.max_sms);
  // groups of many rows (on average at least two 256-row tiles) take the
  // CTA-pair form; the offsets stay on the device, so the average decides
  if (a.M >= 512LL * a.E && a.N > 128 && takes_pair(a.M, a.N, sms))
    return launch_gemm_pair_grouped(a, s);
  Params p{};
  p.a_scales = a.a_scales;
  p.w_scales = a.w_scales;
  p.g_a = a.g_a;
  p.g_w = a.g_w;
  p.C = a.C;
  p.ldc = a.ldc;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  // M tiles of all groups together (a bound for the grid: each group may add
  // a partial tile at either end, its first one starting on the 128-row
  // block of its first row)
  p.m_tiles = (a.M + BM - 1) / BM + 2 * a.E;
  p.k_steps = (a.K + BK - 1) / BK;
  p.ncb = ncb_of(nsf_of(a.K, a.fmt));
  p.w_rowblocks = (a.N + 127) / 128;
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;
  p.offsets = a.offsets;
  p.E = a.E;
  p.w_sf_bytes = static_cast<long long>(p.w_rowblocks) * p.ncb * 512;
  p.a_rowblocks = (a.M + BM - 1) / BM;
  p.splits = 1;
  p.k_per = p.k_steps;
  // tiles of 128 rows x 256 columns with all of K (no split); 128 x 128
  // when N is at most 128
  const int bn = a.N > 128 ? 256 : 128;
  CUtensorMap ma, mw;
  if (!make_code_map(&ma, a.a_codes, a.M, a.K, BM)) return cudaErrorInvalidValue;
  if (!make_code_map(&mw, a.w_codes, static_cast<long long>(a.E) * a.N, a.K, bn))
    return cudaErrorInvalidValue;
  p.n_tiles = (a.N + bn - 1) / bn;
  const long long upper = static_cast<long long>(p.m_tiles) * p.n_tiles;
  const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(upper, sms)));
  if (bn == 256)
    return a.fmt == 0 ? (a.out_f32 ? launch_typed<0, 1, 256, 1>(ma, mw, p, grid, s)
                                   : launch_typed<0, 0, 256, 1>(ma, mw, p, grid, s))
                      : (a.out_f32 ? launch_typed<1, 1, 256, 1>(ma, mw, p, grid, s)
                                   : launch_typed<1, 0, 256, 1>(ma, mw, p, grid, s));
  return a.fmt == 0 ? (a.out_f32 ? launch_typed<0, 1, 128, 1>(ma, mw, p, grid, s)
                                 : launch_typed<0, 0, 128, 1>(ma, mw, p, grid, s))
                    : (a.out_f32 ? launch_typed<1, 1, 128, 1>(ma, mw, p, grid, s)
                                 : launch_typed<1, 0, 128, 1>(ma, mw, p, grid, s));
}

cudaError_t gemm_plan(int M, int N, int K, int max_sms, int* tile_m, int* tile_n, int* splits,
                      bool allow_split) {
  const int sms = gemm_sms(max_sms);
  if (sms <= 0) return cudaErrorNoDevice;
  if (takes_pair(M, N, sms)) {
    *tile_m = 2 * BM;
    *tile_n = 256;
    *splits = 1;
    return cudaSuccess;
  }
  const Shape sh = choose_shape((M + BM - 1) / BM, N, (K + BK - 1) / BK, sms, max_clusters_bn,
                                allow_split);
  *tile_m = BM;
  *tile_n = sh.bn;
  *splits = sh.splits;
  return cudaSuccess;
}

}  // namespace fp4
