// fused.cu -- small-M (decode) W4A4 path: the bf16 activation is quantized
// inside the GEMM kernel, never written to global memory in FP4 form.
//
// "FP4 n'existe pas", runtime survey: quantization, scaling, matmul and
// de-scaling fused in one launch; the small-M regime cuBLAS refuses:
// "Hardware FP4 inference for speech on Blackwell", section "Do the FP4
// tensor cores even engage?".  Same arithmetic as fp4_quantize_act followed
// by fp4_gemm (bit-identical codes and scales), up to FP32 summation order.
//
// One or two launches per call:
//  prologue  (DYNAMIC global scale only) one partial amax per CTA.  Every
//            launch is a programmatic dependent of the one before it, and
//            every kernel here releases its dependent early, so a kernel's
//            weight streaming starts while its predecessor still runs; a
//            kernel reads the activation only after griddepcontrol.wait.
//  main      swap-AB: the weights are the 128-row "A" operand of
//            tcgen05.mma kind::mxf4nvf4 and the <= 32 activation rows are the
//            16- or 32-wide "B" operand.  Grid = N/128 weight tiles x S
//            split-K slices, S chosen so the grid fits one wave.  Per CTA:
//     warp 0     TMA: weight tiles (16 KiB per 256 K) + their scale atoms
//                through a 4-stage ring;
//     warp 1     MMA issuer;
//     warps 2-5  after griddepcontrol.wait: global scale; then per 256-K
//                step, quantize the activation rows into shared memory
//                (128-byte swizzled K-major rows, the MMA's B layout) and
//                their scales into tensor memory (tcgen05.st), loads of
//                the next step in flight meanwhile; finally the epilogue.
//     Weight scales go to tensor memory with tcgen05.cp from the MMA
//     thread: at decode sizes the tensor pipe has slack for it.
//  With S > 1 slices the S CTAs of a weight tile form a thread-block
//  cluster: each leaves its FP32 partial in shared memory and CTA s sums
//  rows m = s, s + S, ... over the S partials in slice order through
//  distributed shared memory (deterministic, no global round trip).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "codec.cuh"
#include "ptx.cuh"

namespace fp4 {

namespace {

constexpr int FBM = 128;                 // weight rows per tile
constexpr int FBK = 256;                 // K per ring stage
constexpr int FBK_BYTES = FBK / 2;
constexpr int FSTAGES = 4;
constexpr int FW_STAGE = FBM * FBK_BYTES;   // 16 KiB
constexpr int FSF_STAGE = 4 * 512;          // up to 4 weight-scale atoms
constexpr int kMaxSplits = 8;               // portable cluster size
constexpr int kMaxStepsPerSplit = 26;       // activation scales of a slice fit tensor memory
constexpr int kFusedThreads = 192;          // TMA, MMA, 4 worker warps
constexpr int kTargetCtas = 148;            // SMs of a B200
constexpr int kSmemPerSm = 227 * 1024;      // shared memory a B200 SM offers to CTAs
constexpr int kStageBudget = 64 * 1024;     // bf16 activation staging (two buffers)
constexpr int kPrologueThreads = 256;
constexpr int kMaxPrologueCtas = 148;
// Tensor-memory columns.  Every scale-factor address an MMA gets is a
// multiple of 4 columns (16 bytes): a misaligned-address fault was seen on
// B200 when scales sat at columns 4i + k.
constexpr uint32_t F_ACC_COL = 0;           // <= 32 fp32 columns
constexpr uint32_t F_SFA_COL = 32;          // weight scales: 16 columns per ring stage
constexpr uint32_t F_SFB_COL = 96;          // activation scales: 16 columns per K step
inline int tmem_cols_for(int steps) { return (F_SFB_COL + 16 * steps) <= 256 ? 256 : 512; }

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

struct Plan {
  int n_tiles, k_steps, splits, steps_max, nmma_n;
  int smem_bytes, tmem_cols, group;
  bool ok;
};

// Steps of bf16 activation staged per group (double-buffered cp.async).
int group_steps(int M, int steps) {
  const int per_step = M * FBK * 2;                 // bf16 bytes of one 256-K step
  return std::max(1, std::min(steps, kStageBudget / (2 * per_step)));
}

int plan_smem(int M, int steps, int nmma_n) {
  const int gs = group_steps(M, steps);
  return 1024 + FSTAGES * (FW_STAGE + FSF_STAGE) + steps * nmma_n * FBK_BYTES +
         steps * nmma_n * 16 + 2 * gs * M * FBK * 2 + 256;
}

// Split count: the largest S <= 8 whose whole grid (N/128 tiles x S) fits in
// one wave, counting two CTAs per SM when shared and tensor memory allow.
Plan make_plan(int M, int N, int K) {
  Plan p{};
  p.n_tiles = (N + FBM - 1) / FBM;
  p.k_steps = (K + FBK - 1) / FBK;
  p.nmma_n = M <= 16 ? 16 : 32;
  int best = 0;
  for (int s = 1; s <= kMaxSplits && s <= p.k_steps; ++s) {
    const int steps = (p.k_steps + s - 1) / s;
    if (steps > kMaxStepsPerSplit) continue;
    const int smem = plan_smem(M, steps, p.nmma_n);
    if (smem > kSmemPerSm) continue;
    const int per_sm = (smem <= kSmemPerSm / 2 && tmem_cols_for(steps) <= 256) ? 2 : 1;
    if (best == 0 || p.n_tiles * s <= kTargetCtas * per_sm) best = s;
  }
  p.ok = best > 0;
  p.splits = best > 0 ? best : 1;
  p.steps_max = (p.k_steps + p.splits - 1) / p.splits;
  p.group = group_steps(M, p.steps_max);
  p.smem_bytes = plan_smem(M, p.steps_max, p.nmma_n);
  p.tmem_cols = tmem_cols_for(p.steps_max);
  return p;
}

struct FParams {
  const uint16_t* a;
  const uint8_t* w_scales;
  const float* g_w;
  float* g_a;
  const unsigned* amax_partial;
  void* C;
  long long ldc;
  int M, N, K;
  int dynamic, out_f32;
  int n_tiles, k_steps, splits, steps_max, nmma_n, ncb, n_partial, tmem_cols, group;
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
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_peer_f32(uint32_t local_saddr, uint32_t rank) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_saddr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void store_out(const FParams& p, int m, int n, float c) {
  if (p.out_f32)
    static_cast<float*>(p.C)[m * p.ldc + n] = c;
  else
    static_cast<__nv_bfloat16*>(p.C)[m * p.ldc + n] = __float2bfloat16_rn(c);
}

// ------------------------------------------------------------ prologue

// DYNAMIC global scale: one partial amax per CTA.  Launched as a
// programmatic dependent of the previous kernel, it lets the main kernel
// launch at once, so the weights start streaming while this runs.
__global__ void __launch_bounds__(kPrologueThreads)
    fused_amax_kernel(const uint4* __restrict__ a, long long n_vec,
                      unsigned* __restrict__ partial) {
  grid_dep_launch();   // the main kernel may launch and prefetch weights
  grid_dep_wait();     // the kernel that wrote `a` (if any) has finished
  unsigned m = 0;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    m = __vmaxu2(m, mag_max8(ld_nc16(a + i)));
  m = fold_u16x2(m);
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
  uint8_t* sScr = sAct + p.steps_max * act_chunk;             // per step: nmma_n x 16 scale bytes
  const int scr_step = p.nmma_n * 16;
  uint8_t* sX = sScr + p.steps_max * scr_step;                // bf16 staging, two group buffers
  const int x_row = p.group * FBK * 2;                        // bytes of one row in a buffer
  const int x_buf = p.M * x_row;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + 2 * x_buf);
  uint64_t* full = bars;
  uint64_t* empty = full + FSTAGES;
  uint64_t* sf_loaded = empty + FSTAGES;
  uint64_t* sf_full = sf_loaded + FSTAGES;
  uint64_t* acc_full = sf_full + FSTAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

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
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_w);
  }
  __syncthreads();
  // every CTA of this grid is resident: the next kernel in the stream may
  // launch now and start streaming its own weights into free SM resources
  grid_dep_launch();
  // tensor memory is allocated by warp 1 while warp 0 already streams
  // weights; warps 1-5 meet on named barrier 2 before using it
  uint32_t tmem = 0;
  if (warp >= 1) {
    if (warp == 1) {
      tmem_alloc(tmem_slot, static_cast<uint32_t>(p.tmem_cols));
      tmem_relinquish();
    }
    tc_fence_before();
    asm volatile("bar.sync 2, 160;" ::: "memory");
    tc_fence_after();
    tmem = *tmem_slot;
  }
  bool epilogue_ok = false;   // workers: the accumulator was read
  float alpha = 1.0f;         // workers: g_a * g_w (NVFP4) or 1

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      uint32_t armed = 0, armed_parity = 0;
      for (int i = 0; i < n_steps; ++i) {
        const int stage = i % FSTAGES;
        const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.watchdog, WD_PRODUCER)) break;
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
      if (*abort_flag) {
        for (int s = 0; s < FSTAGES; ++s)
          if (armed & (1u << s)) {
            mbar_wait_drain(&sf_loaded[s], (armed_parity >> s) & 1u, p.watchdog);
            mbar_wait_drain(&full[s], (armed_parity >> s) & 1u, p.watchdog);
          }
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
        // sf_full[stage]: the workers wrote this step's activation (codes and
        // scales) and the stage's weight scales
        ok = mbar_wait(&full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL) &&
             mbar_wait(&sf_full[stage], phase, abort_flag, p.watchdog, WD_MMA_FULL);
        if (!ok) break;
        tc_fence_after();
        const int kglob = (s_lo + i) * FBK;
        const int n_mma = min(4, (p.K - kglob + 63) / 64);
        const uint32_t w_s = smem_u32(sW + stage * FW_STAGE);
        const uint32_t x_s = smem_u32(sAct + i * act_chunk);
        const uint32_t sfa = tmem + F_SFA_COL + stage * 16;
        const uint32_t sfb = tmem + F_SFB_COL + i * 16;
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
    const int wt = threadIdx.x - 64;                 // 0..127
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    grid_dep_wait();                                 // amax prologue finished and visible
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
    // The activation slice (rows < M, K range of this split) is staged in
    // groups of p.group steps: cp.async brings group g+1 while group g is
    // quantized from shared memory into the MMA's B layout (codes) and the
    // scale scratch; the group's scales then go to tensor memory.  Per step
    // the workers also move the stage's weight scales into tensor memory and
    // then signal the MMA thread.  Every worker warp runs every iteration
    // and every named barrier (an abort skips work, never a barrier).
    const int k0 = s_lo * FBK;
    const int chunks_per_row = p.group * FBK / 8;     // 16-byte pieces per row and group
    auto stage_group = [&](int grp) {
      const uint32_t dst0 = smem_u32(sX + (grp & 1) * x_buf);
      const int total = p.M * chunks_per_row;
      for (int c = wt; c < total; c += 128) {
        const int m = c / chunks_per_row;
        const int kk = (c - m * chunks_per_row) * 8 + grp * p.group * FBK;   // within the slice
        const int kg = k0 + kk;
        const bool in = kk < n_steps * FBK && kg < p.K;
        const uint16_t* src = p.a + (in ? static_cast<long long>(m) * p.K + kg : 0);
        cp_async16(dst0 + m * x_row + (kk - grp * p.group * FBK) * 2, src, in ? 16u : 0u);
      }
      cp_async_commit();
    };
    const int n_groups = (n_steps + p.group - 1) / p.group;
    if (n_groups > 0) stage_group(0);
    for (int i = 0; i < n_steps; ++i) {
      const int stage = i % FSTAGES;
      const uint32_t phase = static_cast<uint32_t>(i / FSTAGES) & 1u;
      if (i % p.group == 0) {
        const int grp = i / p.group;
        if (grp + 1 < n_groups) {
          stage_group(grp + 1);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        workers_sync();                             // group grp is in shared memory
        const uint8_t* xb = sX + (grp & 1) * x_buf;
        const int g_steps = min(p.group, n_steps - i);
        // Only rows m < M are quantized: padding rows feed only output
        // columns that are never stored.  Each thread takes 4 independent
        // 16-value units per batch (loads, then math, then stores) so their
        // long rounding chains interleave.
        const int per_step = p.M * 16;
        const int units = g_steps * per_step;
        const int padded = (units + 511) / 512 * 512;   // whole warps in every batch
        for (int base = 0; base < padded; base += 512) {
          uint4 x0[4], x1[4];
          int step_of[4], m_of[4], ku_of[4];
          bool act[4], live[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int u = base + j * 128 + wt;
            act[j] = u < units;
            const int uu = act[j] ? u : 0;
            const int sl = uu / per_step;
            const int r = uu - sl * per_step;
            m_of[j] = r >> 4;
            ku_of[j] = r & 15;
            step_of[j] = i + sl;
            const int kg = k0 + step_of[j] * FBK + ku_of[j] * 16;
            live[j] = act[j] && kg < p.K;
            x0[j] = x1[j] = make_uint4(0, 0, 0, 0);
            if (live[j]) {
              const uint32_t src = smem_u32(xb + m_of[j] * x_row + (sl * FBK + ku_of[j] * 16) * 2);
              x0[j] = lds128(src);
              x1[j] = lds128(src + 16);
            }
          }
          uint2 q[4];
          unsigned sb[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            unsigned mm = fold_u16x2(__vmaxu2(mag_max8(x0[j]), mag_max8(x1[j])));
            float rr;
            if (FMT == 0) {
              sb[j] = nvfp4_scale(mm, g, six_g, &rr);
              q[j] = (rr == 0.0f) ? make_uint2(0, 0)
                                  : make_uint2(quant8(x0[j].x, x0[j].y, x0[j].z, x0[j].w, rr),
                                               quant8(x1[j].x, x1[j].y, x1[j].z, x1[j].w, rr));
            } else {
              mm = max(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, 1));   // 32-value block = lane pair
              sb[j] = mxfp4_scale(mm, &rr);
              q[j] = make_uint2(quant8(x0[j].x, x0[j].y, x0[j].z, x0[j].w, rr),
                                quant8(x1[j].x, x1[j].y, x1[j].z, x1[j].w, rr));
              if (!live[j]) sb[j] = 0;
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (!act[j]) continue;
            const int m = m_of[j], ku = ku_of[j], step = step_of[j];
            // codes: byte ku*8 of row m in the step's chunk, 128-byte swizzle
            const int kb = ku * 8;
            const int off = step * act_chunk + (m >> 3) * 1024 + (m & 7) * 128 +
                            ((((kb >> 4) ^ (m & 7)) << 4) | (kb & 15));
            *reinterpret_cast<uint2*>(sAct + off) = q[j];
            uint8_t* scr = sScr + step * scr_step;
            if (FMT == 0)
              scr[m * 16 + ku] = static_cast<uint8_t>(sb[j]);
            else if ((ku & 1) == 0)
              scr[m * 16 + (ku >> 1)] = static_cast<uint8_t>(sb[j]);
          }
        }
        fence_proxy_async_smem();      // generic-proxy writes -> visible to the tensor core
        workers_sync();
        // the group's activation scales -> tensor memory: lane i holds row i;
        // word c of a step's row goes to column 16 step + 4 c (4-aligned)
        if (!*abort_flag) {
          for (int sl = 0; sl < g_steps; ++sl) {
            uint4 w = make_uint4(0, 0, 0, 0);
            if (lane < p.M)
              w = *reinterpret_cast<const uint4*>(sScr + (i + sl) * scr_step + lane * 16);
            uint32_t bw[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) bw[j] = 0u;
            bw[0] = w.x;
            bw[4] = w.y;
            if (FMT == 0) {
              bw[8] = w.z;
              bw[12] = w.w;
            }
            tmem_st_x16(tmem + lane_off + F_SFB_COL + (i + sl) * 16, bw);
          }
        }
      }
      // weight scales of this stage -> tensor memory (every quarter gets the
      // 32-row x 16-byte block of each atom); the wait on sf_loaded also
      // keeps this arrival within one phase of the MMA thread's wait
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait(&sf_loaded[stage], phase, abort_flag, p.watchdog, WD_STAGING)))
        continue;
      {
        const uint32_t src = smem_u32(sSF + stage * FSF_STAGE) + lane * 16;
        uint32_t v[16];
#pragma unroll
        for (int a = 0; a < kAtoms; ++a) {
          const uint4 x = lds128(src + a * 512);
          v[4 * a] = x.x; v[4 * a + 1] = x.y; v[4 * a + 2] = x.z; v[4 * a + 3] = x.w;
        }
        if (kAtoms == 4) tmem_st_x16(tmem + lane_off + F_SFA_COL + stage * 16, v);
        else tmem_st_x8(tmem + lane_off + F_SFA_COL + stage * 16, v);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[stage]);
    }
    // (4) accumulator -> C directly (one slice) or -> this CTA's partial
    //     in shared memory (several slices: a cluster reduces them below)
    {
      const bool done =
          __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, abort_flag, p.watchdog, WD_EPILOGUE));
      workers_sync();
      epilogue_ok = done && !*abort_flag;
    }
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
        const float alpha1 = (FMT == 0) ? __fmul_rn(g, *p.g_w) : 1.0f;
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < 32; ++m)
            if (m < p.M) store_out(p, m, n, __fmul_rn(alpha1, __uint_as_float(r[m])));
        }
      } else {
        float* part = reinterpret_cast<float*>(sW);  // the ring is idle now
#pragma unroll
        for (int m = 0; m < 32; ++m)
          if (m < p.M) part[m * FBM + nloc] = __uint_as_float(r[m]);
      }
    }
    alpha = (FMT == 0) ? __fmul_rn(g, *p.g_w) : 1.0f;
  }

  if (p.splits > 1) {
    // every CTA of the tile's cluster has written its partial sums
    cluster_sync_all();
    if (warp >= 2 && epilogue_ok) {
      const int wt = threadIdx.x - 64;
      const int n = tile * FBM + wt;
      const uint32_t base = smem_u32(sW) + wt * 4;
      // CTA `split` reduces rows m = split, split + S, ... in slice order
      for (int m = split; m < p.M; m += p.splits) {
        float acc = 0.0f;
        for (int s = 0; s < p.splits; ++s)
          acc = __fadd_rn(acc, ld_peer_f32(base + m * FBM * 4, static_cast<uint32_t>(s)));
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
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
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

bool fused_supported(int M, int N, int K) {
  if (M < 1 || M > 32 || N < 1 || K < 1) return false;
  return make_plan(M, N, K).ok;
}

size_t fused_workspace_bytes(int M, int N, int K, int fmt) {
  (void)M;
  (void)N;
  (void)K;
  (void)fmt;
  return align256(static_cast<size_t>(kMaxPrologueCtas) * sizeof(unsigned));
}

cudaError_t launch_gemm_fused(const FusedArgs& f, cudaStream_t s) {
  const Plan pl = make_plan(f.M, f.N, f.K);
  if (!pl.ok) return cudaErrorInvalidValue;
  FParams p{};
  p.a = static_cast<const uint16_t*>(f.a);
  p.w_scales = f.w_scales;
  p.g_w = f.g_w;
  p.g_a = f.g_a;
  p.amax_partial = static_cast<const unsigned*>(f.ws);
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
  p.tmem_cols = pl.tmem_cols;
  p.group = pl.group;
  p.ncb = ncb_of(nsf_of(f.K, f.fmt));
  p.watchdog = watchdog_ptr();
  if (!p.watchdog) return cudaErrorInvalidSymbol;

  cudaError_t e;
  if (f.dynamic) {
    const long long n_vec = static_cast<long long>(f.M) * f.K / 8;
    const int blocks = static_cast<int>(std::min<long long>(
        kMaxPrologueCtas,
        std::max<long long>(1, (n_vec + kPrologueThreads * 2 - 1) / (kPrologueThreads * 2))));
    p.n_partial = blocks;
    cudaLaunchConfig_t pc{};
    pc.gridDim = dim3(static_cast<unsigned>(blocks));
    pc.blockDim = dim3(kPrologueThreads);
    pc.stream = s;
    cudaLaunchAttribute pa[1];
    pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pa[0].val.programmaticStreamSerializationAllowed = 1;
    pc.attrs = pa;
    pc.numAttrs = 1;
    e = cudaLaunchKernelEx(&pc, fused_amax_kernel, static_cast<const uint4*>(f.a), n_vec,
                           static_cast<unsigned*>(f.ws));
    if (e != cudaSuccess) return e;
  }

  CUtensorMap mw;
  if (!make_w_map(&mw, f.w_codes, f.N, f.K)) return cudaErrorInvalidValue;
  auto kern = (f.fmt == 0) ? fused_kernel<0> : fused_kernel<1>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem_bytes);
  if (e != cudaSuccess) return e;
  if (pl.splits > 1) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.n_tiles * pl.splits));
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(pl.smem_bytes);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pl.splits > 1) {
    // the S slices of a weight tile form one cluster and reduce through
    // distributed shared memory
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(pl.splits);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  cfg.attrs = na ? attr : nullptr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, mw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4
