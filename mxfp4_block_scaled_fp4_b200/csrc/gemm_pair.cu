// gemm_pair.cu -- the block-scaled FP4 GEMM of gemm.cu on CTA pairs
// (tcgen05 cta_group::2), used when M > 128.
//
//   C[M, N] = alpha * sum_k s_a[m, k/B] q_a[m, k] * s_w[n, k/B] q_w[n, k]
//
// (the W4A4 GEMM of the "fp4-cuda-kernel" forum post; NVFP4 / MXFP4 block
// formats as in gemm.cu.)
//
// The output is cut into 256 x 256 tiles, each computed by a cluster of two
// CTAs on the two SMs of a TPC.  CTA r of the pair holds rows r*128 .. +127
// of the tile's A slice and of its W slice in its own shared memory; one
// tcgen05.mma (M = 256, N = 256, K = 64) issued by the even CTA (the leader)
// reads A from each CTA's own half and W from both halves, and leaves
// accumulator rows r*128 .. +127 (all 256 columns) in CTA r's tensor memory,
// next to CTA r's own copy of the scales.  Per SM and per MMA that halves the
// W bytes loaded into and read out of shared memory compared with the
// one-CTA 128 x 256 tile (12 KiB -> 8 KiB of operand traffic per 128 x 256 x
// 64 step); measured on B200 it is 8-13% faster than the one-CTA kernel on
// large prefill shapes and bit-identical to it.
//
// Roles (11 warps in each CTA of the pair):
//   warp 0      TMA for this CTA: its A and W halves (plain, non-multicast
//               tiled loads onto its own `full` barrier);
//   warp 10     bulk copies of this CTA's scale atoms (the A row block of its
//               half; both W row blocks of the tile, which every SM's MMA
//               reads from its own tensor memory) onto `sf_loaded`;
//   warp 1      both CTAs: tensor-memory allocation for the pair; leader,
//               one thread: issues the pair MMAs, commits to both CTAs'
//               `empty` / `acc_full` barriers (multicast commit);
//   warps 2-5   epilogue of this CTA's 128 accumulator rows, then release
//               the accumulator on the leader's `acc_empty` (count 8);
//   warps 6-9   scale staging into this CTA's tensor memory with tcgen05.st;
//               once the stage's code tiles have landed as well, each warp
//               arrives on the leader's `ready` barrier (count 8), so the MMA
//               thread waits on one barrier for both CTAs' data.
// The hand-offs between the CTAs are plain remote mbarrier arrivals: what
// they publish is ordered by tcgen05.wait::st / tcgen05.ld waits and the
// tcgen05 thread-sync fences (tensor memory) or by an mbarrier the arriving
// warp has itself observed complete (shared memory written by TMA).  A
// release at cluster scope on the per-stage arrival was measured to cost
// ~1000 cycles per K step and to halve the kernel's speed.
// Every copy is issued and awaited by the CTA whose shared memory it fills,
// so on an abort each CTA drains its own copies.  Every wait is bounded; a
// wait that runs out sets the watchdog word and raises the abort flag of
// both CTAs, the leader waits for its MMAs in flight, and both CTAs meet at
// a final cluster barrier before the pair's tensor memory is freed.
#include <algorithm>
#include <atomic>
#include <cuda_bf16.h>

#include "groups.cuh"
#include "internal.h"
#include "out_quant.cuh"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int BM = 256;                 // tile rows (128 per CTA)
constexpr int BN = 256;                 // tile columns (128 W rows per CTA)
constexpr int HALF = 128;
constexpr int BK = 256;
constexpr int BK_BYTES = BK / 2;
constexpr int MMA_K = 64;
constexpr int STAGES = 5;
constexpr int A_STAGE = HALF * BK_BYTES;   // 16 KiB
constexpr int B_STAGE = HALF * BK_BYTES;   // 16 KiB
constexpr int SFA_STAGE = 4 * 512;
constexpr int SFB_STAGE = 2 * 4 * 512;
constexpr int RING_BYTES = STAGES * (A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE);
// bf16 epilogue staging: per epilogue warp two 32-row x 64-column buffers
// (4 KiB each, 128-byte swizzle) that TMA stores drain to C
constexpr int OUT_BUF = 32 * 128;
constexpr int OUT_BYTES = 4 * 2 * OUT_BUF;
constexpr int RTAB_BYTES = 512;          // FP4-emitting epilogue: 128 reciprocals
constexpr int SMEM_BYTES = RING_BYTES + OUT_BYTES + RTAB_BYTES + 1024 + 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SF_COL = 256;
constexpr uint32_t SF_STAGE_COLS = 48;
constexpr int kThreads = 352;       // 11 warps
constexpr int GROUP_M = 32;             // raster: 32 tile rows (8192 rows of A) share W in L2

static_assert(SF_COL + STAGES * SF_STAGE_COLS <= TMEM_COLS, "scale stages exceed tensor memory");
static_assert(SMEM_BYTES <= 227 * 1024, "ring exceeds shared memory");
static_assert(RING_BYTES % 1024 == 0, "epilogue buffers must stay 1024-byte aligned");

// The grouped (mixture-of-experts) form, G = 1: the same ring (a group's
// tiles start on a 128-row scale block, so each CTA half reads one block of
// A scales, as in the plain form); the group table takes the place of the
// reciprocals (the grouped form has no FP4 output).
template <int G>
struct PairLayout {
  static constexpr int RTAB = G ? 0 : RTAB_BYTES;
  // macro-block scaling (OUT 4, 5): the tile's 256 column scales, double
  // buffered across tiles
  static constexpr int SIGW = G ? 0 : 2 * BN * 4;
  static constexpr int GTAB = G ? 4 * (2 * kGroupedMaxGroups + 2) : 0;
  static constexpr int SMEM = RING_BYTES + OUT_BYTES + RTAB + SIGW + GTAB + 1024 + 256;
  static_assert(SMEM <= 227 * 1024, "ring exceeds shared memory");
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
  int ncb;
  int a_rowblocks;        // ceil(M / 128)
  int w_rowblocks;        // ceil(N / 128)
  unsigned* watchdog;
  QuantOut qo;            // OUT 2, 3: the emitted FP4 activation (C optional)
  const float* sigma_a;   // OUT 4, 5: macro-block scales of A rows [M] and W rows [N]
  const float* sigma_w;
  // grouped form (G = 1): group e is rows [offsets[e], offsets[e+1]) of A
  // and C and weight rows [e N, e N + N) of the stacked W, whose scales
  // start at byte e * w_sf_bytes; g_w holds one global scale per group
  const int* offsets;
  int E;
  long long w_sf_bytes;
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

// OUT: 0 = bf16 C, 1 = fp32 C, 2 / 3 = C quantized to NVFP4 / MXFP4
// (out_quant.cuh), with the bf16 C stored as well when p.C is not null;
// 4 / 5 = bf16 / fp32 C scaled by sigma_a[m] sigma_w[n] (MXFP4 macro-block
// scaling) instead of alpha.
// QROT (OUT 2, 3): the emitted activation's rotation order (0, 16, 32).
template <int FMT, int OUT, int G = 0, int QROT = 0>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_q, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  // the same 1024-aligned offset in both CTAs: the pair MMA addresses the
  // peer's operands with this CTA's descriptors
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE;
  uint8_t* sSFA = sB + STAGES * B_STAGE;
  uint8_t* sSFB = sSFA + STAGES * SFA_STAGE;
  uint8_t* sOut = sSFB + STAGES * SFB_STAGE;
  float* r_tab = reinterpret_cast<float*>(sOut + OUT_BYTES);                          // G = 0
  float* sigw = reinterpret_cast<float*>(sOut + OUT_BYTES + PairLayout<G>::RTAB);     // G = 0
  int* gtab = reinterpret_cast<int*>(sOut + OUT_BYTES + PairLayout<G>::RTAB +
                                     PairLayout<G>::SIGW);                           // G = 1
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + OUT_BYTES + PairLayout<G>::RTAB +
                                               PairLayout<G>::SIGW + PairLayout<G>::GTAB);
  uint64_t* sf_loaded = full + STAGES;
  uint64_t* empty = sf_loaded + STAGES;
  uint64_t* ready = empty + STAGES;
  uint64_t* acc_full = ready + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* sw_ready = drain + 1;   // MBS: the two column-scale buffers (4 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sw_ready + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sf_loaded[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 8);     // 4 staging warps in each CTA of the pair
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);       // 4 epilogue warps in each CTA of the pair
    mbar_init(drain, 1);
    mbar_init(&sw_ready[0], 4);
    mbar_init(&sw_ready[1], 4);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_w);
    if (!(OUT == 2 || OUT == 3) || p.C != nullptr) prefetch_tensormap(&tm_c);
    if (OUT == 2 || OUT == 3) prefetch_tensormap(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // barriers initialised and tensor memory allocated in both CTAs before any
  // remote arrival
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t peer_abort = map_to_rank(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);

  int n_tiles_total = p.m_tiles * p.n_tiles;
  if (G) {
    // the group table from the device-side offsets (groups.cuh), in both
    // CTAs of the pair alike
    if (warp == 0) build_group_table<kGroupedMaxGroups>(p.offsets, p.E, p.M, BM, gtab, lane);
    __syncthreads();
    n_tiles_total = gtab[p.E] * p.n_tiles;
  }
  const int first = static_cast<int>(cluster_id_x());
  const int stride = static_cast<int>(nclusters_x());
  constexpr int kAtomsPerStage = (FMT == 0) ? 4 : 2;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    for (int t = first; t < n_tiles_total; t += stride) {
      int a_row, w_row;   // first A row and W row of this CTA's half
      if (G) {
        const GTile g = gtile<kGroupedMaxGroups>(t, p.E, p.n_tiles, BM, gtab, GROUP_M);
        a_row = g.a_row0 + static_cast<int>(rank) * HALF;
        w_row = g.e * p.N + g.nt * BN + static_cast<int>(rank) * HALF;
      } else {
        int mt, nt;
        tile_coords(t, p, mt, nt);
        a_row = mt * BM + static_cast<int>(rank) * HALF;
        w_row = nt * BN + static_cast<int>(rank) * HALF;
      }
      for (int kb = 0; kb < p.k_steps; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER)) {
          st_cluster_u32(peer_abort, 1u);
          goto producer_drain;
        }
        {
          mbar_expect_tx(&full[stage], A_STAGE + B_STAGE);
          tma_load_2d(sA + stage * A_STAGE, &tm_a, kb * BK_BYTES, a_row, &full[stage]);
          tma_load_2d(sB + stage * B_STAGE, &tm_w, kb * BK_BYTES, w_row, &full[stage]);
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
    for (int s = 0; s < STAGES; ++s)
      if (armed & (1u << s)) mbar_wait_drain(&full[s], (armed_parity >> s) & 1u, p.watchdog);
  producer_done:;
  } else if (warp == 10 && lane == 0) {
    // ------------------------------------------------ scale-atom producer
    // A thread of its own, so that the scale copies and the code-tile
    // copies of a stage are issued in parallel (each copy instruction costs
    // its thread ~80 cycles, and this sits on the refill path of every stage)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_parity = 0;
    for (int t = first; t < n_tiles_total; t += stride) {
      int rba, nt;                     // A scale row block of this CTA's half
      const uint8_t* wsf = p.w_scales;
      if (G) {
        const GTile g = gtile<kGroupedMaxGroups>(t, p.E, p.n_tiles, BM, gtab, GROUP_M);
        rba = g.a_row0 / HALF + static_cast<int>(rank);
        nt = g.nt;
        wsf += static_cast<long long>(g.e) * p.w_sf_bytes;
      } else {
        int mt;
        tile_coords(t, p, mt, nt);
        rba = mt * 2 + static_cast<int>(rank);
      }
      const int ablocks = rba < p.a_rowblocks ? 1 : 0;
      const int rb0 = nt * 2;
      const int wblocks = min(2, p.w_rowblocks - rb0);
      const uint8_t* sfa_g = p.a_scales + static_cast<long long>(rba) * p.ncb * 512;
      const uint8_t* sfb_g = wsf + static_cast<long long>(rb0) * p.ncb * 512;
      for (int kb = 0; kb < p.k_steps; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER)) {
          st_cluster_u32(peer_abort, 1u);
          goto sf_drain;
        }
        {
          const int cb0 = kb * kAtomsPerStage;
          const int atoms = min(kAtomsPerStage, p.ncb - cb0);
          const uint32_t sf_bytes = static_cast<uint32_t>(atoms) * 512u;
          // a half made only of rows past M has no scale atoms; its
          // accumulator rows are never stored
          mbar_expect_tx(&sf_loaded[stage], sf_bytes * (ablocks + wblocks));
          for (int i = 0; i < ablocks; ++i)
            bulk_load(sSFA + stage * SFA_STAGE + i * kAtomsPerStage * 512,
                      sfa_g + (static_cast<long long>(i) * p.ncb + cb0) * 512, sf_bytes,
                      &sf_loaded[stage]);
          for (int i = 0; i < wblocks; ++i)
            bulk_load(sSFB + stage * SFB_STAGE + i * 2048,
                      sfb_g + (static_cast<long long>(i) * p.ncb + cb0) * 512, sf_bytes,
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
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------- pair MMA issuer
    // Lean loop: the pipe runs one 256 x 256 x 64 MMA per 128 cycles and an
    // issue costs this thread ~75, so everything else it does between two
    // K steps must fit in ~200 cycles or the pipe idles (measured on B200).
    // Descriptors advance by adding to their address field.  No extra
    // probes of `ready`: an mbarrier.try_wait without a suspend hint that
    // finds the phase incomplete can hold the thread for a system-defined
    // time, which measured as a 25% slower K step.
    const uint64_t a_desc0 = smem_desc(smem_u32(sA), 16, 1024, kLayoutSwizzle128B);
    const uint64_t b_desc0 = smem_desc(smem_u32(sB), 16, 1024, kLayoutSwizzle128B);
    const uint32_t sf0 = tmem + SF_COL;
    constexpr uint32_t kIdesc0 = idesc_fp4(BM, BN, FMT == 1, 0, 0);
    constexpr uint32_t kIdesc2 = idesc_fp4(BM, BN, FMT == 1, 2, 2);
    // MMAs in the last K step (K may end inside it)
    const int last_mmas = (p.K - (p.k_steps - 1) * BK + MMA_K - 1) / MMA_K;
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    for (int t = first; t < n_tiles_total; t += stride, ++it) {
      if (it > 0 && !mbar_wait(acc_empty, static_cast<uint32_t>(it - 1) & 1u, abort_flag,
                               p.watchdog, WD_MMA_ACC)) {
        st_cluster_u32(peer_abort, 1u);
        goto mma_drain;
      }
      tc_fence_after();
      for (int kb = 0; kb < p.k_steps; ++kb) {
        if (!mbar_wait(&ready[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL)) {
          st_cluster_u32(peer_abort, 1u);
          goto mma_drain;
        }
        tc_fence_after();
        int nstage = stage + 1;
        uint32_t nphase = phase;
        if (nstage == STAGES) {
          nstage = 0;
          nphase ^= 1u;
        }
        const bool has_next = kb + 1 < p.k_steps;
        {
          const int n_mma = has_next ? BK / MMA_K : last_mmas;
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(stage * (A_STAGE >> 4));
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(stage * (B_STAGE >> 4));
          const uint32_t sfa_t = sf0 + stage * SF_STAGE_COLS;
          const uint32_t sfb_t = sfa_t + 16;
#pragma unroll
          for (int k = 0; k < BK / MMA_K; ++k) {
            if (k < n_mma) {
              // 32 bytes of K per MMA = 2 units of the descriptor's address field
              const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
              if (FMT == 0)
                tc_mma_pair_nvf4(tmem + ACC_COL, ad + 2 * k, bd + 2 * k, kIdesc0, sfa_t + 4 * k,
                                 sfb_t + 8 * k, acc);
              else
                tc_mma_pair_mxf4(tmem + ACC_COL, ad + 2 * k, bd + 2 * k,
                                 (k & 1) ? kIdesc2 : kIdesc0, sfa_t + 4 * (k >> 1),
                                 sfb_t + 8 * (k >> 1), acc);
            }
          }
        }
        tc_commit_pair(&empty[stage], 0x3);
        stage = nstage;
        phase = nphase;
      }
      tc_commit_pair(acc_full, 0x3);
    }
    goto mma_done;
  mma_drain:
    tc_commit_pair(drain, 0x1);
    mbar_wait_drain(drain, 0, p.watchdog);
  mma_done:;
  } else if (warp >= 6 && warp <= 9) {
    // ----------------------------------------------------- scale staging
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = first; t < n_tiles_total; t += stride) {
      for (int kb = 0; kb < p.k_steps; ++kb) {
        if (!__all_sync(0xFFFFFFFFu,
                        mbar_wait(&sf_loaded[stage], phase, abort_flag, p.watchdog, WD_STAGING))) {
          if (lane == 0) st_cluster_u32(peer_abort, 1u);
          goto staging_done;
        }
        {
          const uint32_t sfa_s = smem_u32(sSFA + stage * SFA_STAGE) + lane * 16;
          const uint32_t sfb_s = smem_u32(sSFB + stage * SFB_STAGE) + lane * 16;
          const uint32_t sfa_t = tmem + lane_off + SF_COL + stage * SF_STAGE_COLS;
          const uint32_t sfb_t = sfa_t + 16;
          uint32_t va[4 * kAtomsPerStage], vb[8 * kAtomsPerStage];
#pragma unroll
          for (int a = 0; a < kAtomsPerStage; ++a) {
            {
              const uint4 x = lds128(sfa_s + a * 512);
              va[4 * a + 0] = x.x; va[4 * a + 1] = x.y; va[4 * a + 2] = x.z; va[4 * a + 3] = x.w;
            }
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
        // the stage's code tiles must have landed in this CTA as well before
        // the leader may issue the MMAs that read them
        if (!__all_sync(0xFFFFFFFFu,
                        mbar_wait(&full[stage], phase, abort_flag, p.watchdog, WD_STAGING))) {
          if (lane == 0) st_cluster_u32(peer_abort, 1u);
          goto staging_done;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(&ready[stage]);
          else
            mbar_arrive_remote(map_to_rank(smem_u32(&ready[stage]), 0));
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  staging_done:;
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    float alpha = 1.0f;
    if (FMT == 0) alpha = __fmul_rn(*p.g_a, *p.g_w);
    const uint32_t acc_empty_leader = map_to_rank(smem_u32(acc_empty), 0);
    uint8_t* sOutW = sOut + (warp - 2) * 2 * OUT_BUF;
    QuantOutG qg{};
    constexpr bool F32 = OUT == 1 || OUT == 5;       // fp32 C
    constexpr bool QOUT = OUT == 2 || OUT == 3;      // FP4 activation out
    constexpr bool MBS = OUT >= 4;                   // per-row x per-column scales
    if (QOUT) {
      qg = quant_out_g(p.qo, r_tab, threadIdx.x - 64);
      asm volatile("bar.sync 1, 128;" ::: "memory");   // the 4 epilogue warps
    }
    int it = 0;
    for (int t = first; t < n_tiles_total; t += stride, ++it) {
      int nt, row0, row_begin = 0, row_end = p.M;   // row0: this warp's first C row
      if (G) {
        const GTile g = gtile<kGroupedMaxGroups>(t, p.E, p.n_tiles, BM, gtab, GROUP_M);
        nt = g.nt;
        row0 = g.a_row0 + static_cast<int>(rank) * HALF + quarter * 32;
        row_begin = g.a_row_begin;
        row_end = g.a_row_end;
        if (FMT == 0) alpha = __fmul_rn(*p.g_a, p.g_w[g.e]);
      } else {
        int mt;
        tile_coords(t, p, mt, nt);
        row0 = mt * BM + static_cast<int>(rank) * HALF + quarter * 32;
      }
      const int row = row0 + lane;
      // MBS: the tile's column scales into shared memory while the MMAs run
      // (a tile's epilogue reads each of them 128 times per CTA), each warp a
      // quarter of them; the buffer alternates between tiles, and a warp
      // passes the (bounded) wait of tile t + 1 only after every epilogue
      // warp has arrived for it, i.e. has finished tile t - 1
      float* sw = sigw + (it & 1) * BN;
      if (MBS) {
        for (int j = threadIdx.x - 64; j < BN; j += 128) {
          const int n = nt * BN + j;
          sw[j] = n < p.N ? __ldg(p.sigma_w + n) : 0.0f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sw_ready[it & 1]);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sw_ready[it & 1], static_cast<uint32_t>(it >> 1) & 1u,
                                               abort_flag, p.watchdog, WD_EPILOGUE))) {
          if (lane == 0) st_cluster_u32(peer_abort, 1u);
          break;
        }
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag,
                                             p.watchdog, WD_EPILOGUE))) {
        if (lane == 0) st_cluster_u32(peer_abort, 1u);
        break;
      }
      tc_fence_after();
      const bool row_ok = row >= row_begin && row < row_end;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + ACC_COL;
      if (G && (row0 < row_begin || row0 + 32 > row_end)) {
        // grouped, a warp whose 32 rows reach outside its group: those rows
        // belong to the neighbouring groups, so C leaves by per-row stores
        // of the group's rows only (a TMA store would clip only at 0 and M);
        // warps inside the group take the TMA-store path below
        if (!F32) {
          uint32_t packed[BN / 2];
#pragma unroll
          for (int c = 0; c < BN / 16; ++c) {
            uint32_t r[16];
            FP4_TMEM_LD_32x32b_X16(tbase + c * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(alpha, __uint_as_float(r[2 * j])),
                                                       __fmul_rn(alpha, __uint_as_float(r[2 * j + 1])));
              packed[8 * c + j] = *reinterpret_cast<uint32_t*>(&h);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (leader)
              mbar_arrive(acc_empty);
            else
              mbar_arrive_remote(acc_empty_leader);
          }
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
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t r[32];
            FP4_TMEM_LD_32x32b_X32(tbase + c * 32, r);
            tmem_ld_wait();
            if (c == BN / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                if (leader)
                  mbar_arrive(acc_empty);
                else
                  mbar_arrive_remote(acc_empty_leader);
              }
            }
            const int n0 = nt * BN + c * 32;
            if (!row_ok || n0 >= p.N) continue;
            float* out = static_cast<float*>(p.C) + static_cast<long long>(row) * p.ldc + n0;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              if (n0 + 4 * v < p.N)
                *reinterpret_cast<float4*>(out + 4 * v) =
                    make_float4(__fmul_rn(alpha, __uint_as_float(r[4 * v + 0])),
                                __fmul_rn(alpha, __uint_as_float(r[4 * v + 1])),
                                __fmul_rn(alpha, __uint_as_float(r[4 * v + 2])),
                                __fmul_rn(alpha, __uint_as_float(r[4 * v + 3])));
            }
          }
        }
        continue;
      }
      // MBS: the row's scale (the column's comes with each value)
      const float arow = MBS ? __ldg(p.sigma_a + min(row, p.M - 1)) : alpha;
      if (!F32) {
        uint32_t packed[BN / 2];
#pragma unroll
        for (int c = 0; c < BN / 16; ++c) {
          uint32_t r[16];
          FP4_TMEM_LD_32x32b_X16(tbase + c * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int jc = 16 * c + 2 * j;   // column within the tile
            const float lo = __fmul_rn(MBS ? __fmul_rn(arow, sw[jc]) : arow, __uint_as_float(r[2 * j]));
            const float hi =
                __fmul_rn(MBS ? __fmul_rn(arow, sw[jc + 1]) : arow, __uint_as_float(r[2 * j + 1]));
            __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
            packed[8 * c + j] = *reinterpret_cast<uint32_t*>(&h);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(acc_empty);
          else
            mbar_arrive_remote(acc_empty_leader);
        }
        // C rows row0 .. row0+31 leave through this warp's two swizzled
        // buffers and 64-column TMA stores (rows past M and columns past N
        // are clipped by the store)
        if (row0 < p.M && (!QOUT || p.C != nullptr)) {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) {
            const int n0 = nt * BN + 64 * c;
            if (n0 < p.N) {
              uint8_t* buf = sOutW + (c & 1) * OUT_BUF;
              // the buffer's previous store must have finished reading it
              if (lane == 0) bulk_wait_read_1();
              __syncwarp();
              const uint32_t rowaddr = smem_u32(buf) + lane * 128;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                sts128(rowaddr + ((j ^ (lane & 7)) << 4), packed[32 * c + 4 * j],
                       packed[32 * c + 4 * j + 1], packed[32 * c + 4 * j + 2],
                       packed[32 * c + 4 * j + 3]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tm_c, buf, n0, row0);
                bulk_commit();
              }
            }
          }
        }
        if (QOUT) {
          // the codes of rows row0 .. row0+31 (128 bytes each) leave through
          // this warp's second buffer and one TMA store (rows past M and
          // bytes past N / 2 are clipped by the store); the scales by word
          // stores.  (The next tile's first C chunk uses the first buffer,
          // and its second chunk waits for this store as for any other.)
          const bool pad = p.qo.layout == 0 && !row_ok && row < p.a_rowblocks * HALF;
          uint8_t* qbuf = sOutW + OUT_BUF;
          if (lane == 0) bulk_wait_read_0();   // every earlier store has read its buffer
          __syncwarp();
          const uint32_t srow = row0 < p.M ? smem_u32(qbuf) + lane * 128 : 0u;
          quant_out_row<BN, QOUT ? OUT - 2 : 0, QROT>(p.qo, qg, packed, row, row_ok, pad, nt * BN, p.N,
                                                srow, lane & 7);
          if (row0 < p.M) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tm_q, qbuf, nt * (BN / 2), row0);
              bulk_commit();
            }
          }
        }
      } else {
        // fp32: 32-column chunks leave through the warp's two swizzled
        // buffers (32 rows x 128 bytes each) and TMA stores (clipped at M
        // and N), so that the warp's writes are whole 128-byte rows issued
        // by the copy engine instead of 32 scattered 16-byte stores per
        // instruction; the accumulator is released after its last chunk is
        // read
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          FP4_TMEM_LD_32x32b_X32(tbase + c * 32, r);
          tmem_ld_wait();
          if (c == BN / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (leader)
                mbar_arrive(acc_empty);
              else
                mbar_arrive_remote(acc_empty_leader);
            }
          }
          const int n0 = nt * BN + c * 32;
          if (row0 >= p.M || n0 >= p.N) continue;   // warp-uniform
          uint8_t* buf = sOutW + (c & 1) * OUT_BUF;
          // the buffer's previous store must have finished reading it
          if (lane == 0) bulk_wait_read_1();
          __syncwarp();
          const uint32_t rowaddr = smem_u32(buf) + lane * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int jc = c * 32 + 4 * j;   // column within the tile
            sts128(rowaddr + ((j ^ (lane & 7)) << 4),
                   __float_as_uint(__fmul_rn(MBS ? __fmul_rn(arow, sw[jc]) : arow, __uint_as_float(r[4 * j + 0]))),
                   __float_as_uint(__fmul_rn(MBS ? __fmul_rn(arow, sw[jc + 1]) : arow, __uint_as_float(r[4 * j + 1]))),
                   __float_as_uint(__fmul_rn(MBS ? __fmul_rn(arow, sw[jc + 2]) : arow, __uint_as_float(r[4 * j + 2]))),
                   __float_as_uint(__fmul_rn(MBS ? __fmul_rn(arow, sw[jc + 3]) : arow, __uint_as_float(r[4 * j + 3]))));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_c, buf, n0, row0);
            bulk_commit();
          }
        }
      }
    }
    // every TMA store of this warp has landed before the CTA goes away
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // neither CTA leaves (or frees tensor memory) while the other may still
  // arrive on its barriers or the leader's MMAs may still touch its memory
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------ host side

template <int FMT, int OUT, int G = 0, int QROT = 0>
cudaError_t launch_typed(const CUtensorMap& ma, const CUtensorMap& mw, const CUtensorMap& mc,
                         const CUtensorMap& mq,
                         const Params& p, int tiles, int max_sms, cudaStream_t s) {
  auto kern = gemm_pair_kernel<FMT, OUT, G, QROT>;
  constexpr int SMEM_BYTES = PairLayout<G>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // pairs that fit on the device at once (cached per device and form)
  static std::atomic<int> max_pairs[64] = {};
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int fit = max_pairs[dev].load(std::memory_order_relaxed);
  if (fit <= 0) {
    cfg.gridDim = dim3(2);
    e = cudaOccupancyMaxActiveClusters(&fit, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (fit <= 0) return cudaErrorInvalidConfiguration;
    max_pairs[dev].store(fit, std::memory_order_relaxed);
  }
  const int pairs = std::max(1, std::min({tiles, fit, gemm_sms(max_sms) / 2}));
  cfg.gridDim = dim3(2 * pairs);
  e = cudaLaunchKernelEx(&cfg, kern, ma, mw, mc, mq, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_pair_grouped(const GroupedArgs& a, cudaStream_t s) {
  CUtensorMap ma, mw;
  if (!make_code_map(&ma, a.a_codes, a.M, a.K, HALF)) return cudaErrorInvalidValue;
  if (!make_code_map(&mw, a.w_codes, static_cast<long long>(a.E) * a.N, a.K, HALF))
    return cudaErrorInvalidValue;
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
  // 256-row tiles of all groups together (a bound for the grid: each group
  // may add a partial tile at either end, its first one starting on the
  // 128-row block of its first row)
  p.m_tiles = (a.M + BM - 1) / BM + 2 * a.E;
  p.n_tiles = (a.N + BN - 1) / BN;
  p.k_steps = (a.K + BK - 1) / BK;
  p.ncb = ncb_of(nsf_of(a.K, a.fmt));
  p.a_rowblocks = (a.M + HALF - 1) / HALF;
  p.w_rowblocks = (a.N + HALF - 1) / HALF;
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;
  p.offsets = a.offsets;
  p.E = a.E;
  p.w_sf_bytes = static_cast<long long>(p.w_rowblocks) * p.ncb * 512;
  // C of all groups: warps whose rows lie inside their group store by TMA
  CUtensorMap mc;
  if (a.out_f32 ? !make_f32_out_map(&mc, a.C, a.M, a.N, a.ldc, 32)
                : !make_bf16_out_map(&mc, a.C, a.M, a.N, a.ldc, 32))
    return cudaErrorInvalidValue;
  const int tiles = p.m_tiles * p.n_tiles;
  if (a.fmt == 0)
    return a.out_f32 ? launch_typed<0, 1, 1>(ma, mw, mc, ma, p, tiles, a.max_sms, s)
                     : launch_typed<0, 0, 1>(ma, mw, mc, ma, p, tiles, a.max_sms, s);
  return a.out_f32 ? launch_typed<1, 1, 1>(ma, mw, mc, ma, p, tiles, a.max_sms, s)
                   : launch_typed<1, 0, 1>(ma, mw, mc, ma, p, tiles, a.max_sms, s);
}

cudaError_t launch_gemm_pair(const GemmArgs& a, cudaStream_t s) {
  CUtensorMap ma, mw, mc, mq;
  if (!make_code_map(&ma, a.a_codes, a.M, a.K, HALF)) return cudaErrorInvalidValue;
  if (!make_code_map(&mw, a.w_codes, a.N, a.K, HALF)) return cudaErrorInvalidValue;
  const bool f32 = a.out_mode == 1 || a.out_mode == 5;
  const bool qout = a.out_mode == 2 || a.out_mode == 3;
  if (qout && !a.C)
    mc = ma;   // unused: no bf16 C beside the FP4 output
  else if (f32 ? !make_f32_out_map(&mc, a.C, a.M, a.N, a.ldc, 32)
               : !make_bf16_out_map(&mc, a.C, a.M, a.N, a.ldc, 32))
    return cudaErrorInvalidValue;
  // the emitted codes [M, N / 2]: 128-byte x 32-row boxes, one per epilogue
  // warp and tile (unused otherwise)
  if (!qout)
    mq = ma;
  else if (!make_code_map(&mq, a.qo.codes, a.M, a.N, 32))
    return cudaErrorInvalidValue;
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
  p.a_rowblocks = (a.M + HALF - 1) / HALF;
  p.w_rowblocks = (a.N + HALF - 1) / HALF;
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;
  p.qo = a.qo;
  p.sigma_a = a.sigma_a;
  p.sigma_w = a.sigma_w;
  const int tiles = p.m_tiles * p.n_tiles;
  using L = cudaError_t (*)(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const CUtensorMap&, const Params&, int, int, cudaStream_t);
  static const L table[2][2] = {{launch_typed<0, 0>, launch_typed<0, 1>},
                                {launch_typed<1, 0>, launch_typed<1, 1>}};
  // the FP4-emitting epilogue, by operand format, output format and rotation
  static const L qtable[2][2][3] = {
      {{launch_typed<0, 2, 0, 0>, launch_typed<0, 2, 0, 16>, launch_typed<0, 2, 0, 32>},
       {launch_typed<0, 3, 0, 0>, launch_typed<0, 3, 0, 16>, launch_typed<0, 3, 0, 32>}},
      {{launch_typed<1, 2, 0, 0>, launch_typed<1, 2, 0, 16>, launch_typed<1, 2, 0, 32>},
       {launch_typed<1, 3, 0, 0>, launch_typed<1, 3, 0, 16>, launch_typed<1, 3, 0, 32>}}};
  if (a.out_mode == 2 || a.out_mode == 3) {
    const int ri = a.qo.rot == 32 ? 2 : (a.qo.rot == 16 ? 1 : 0);
    return qtable[a.fmt != 0][a.out_mode - 2][ri](ma, mw, mc, mq, p, tiles, a.max_sms, s);
  }
  if (a.out_mode >= 4) {   // macro-block scaling: MXFP4 only
    if (a.fmt != 1) return cudaErrorInvalidValue;
    return a.out_mode == 5 ? launch_typed<1, 5>(ma, mw, mc, ma, p, tiles, a.max_sms, s)
                           : launch_typed<1, 4>(ma, mw, mc, ma, p, tiles, a.max_sms, s);
  }
  return table[a.fmt != 0][a.out_mode](ma, mw, mc, mq, p, tiles, a.max_sms, s);
}

}  // namespace fp4
