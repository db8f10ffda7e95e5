// internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace fp4 {

constexpr int kAmaxSlots = 1024;   // partial maxima of the global-scale reduction
constexpr int kGroupedMaxGroups = 256;   // groups (experts) of one fp4_gemm_grouped call

// Workspace bytes the activation quantizer needs (the DYNAMIC reduction's
// partial maxima); one rule for every entry point that quantizes.
inline size_t quant_workspace_bytes() { return static_cast<size_t>(kAmaxSlots) * sizeof(unsigned); }

// Streaming multiprocessors of the current device (cached per device).
int sm_count();

// Device address of the watchdog word on the current device (cached per
// device; nullptr if the symbol lookup fails).
unsigned* watchdog_ptr();

// Scale-layout geometry.
inline int nsf_of(int K, int fmt) { return K / (fmt == 0 ? 16 : 32); }
inline int ncb_of(int nsf) { return (nsf + 3) / 4; }
inline long long rows_pad128(long long rows) { return (rows + 127) / 128 * 128; }

// amax over a bf16 tensor of n elements (n % 8 == 0): writes one partial
// maximum (bf16 magnitude bits) per CTA into `partial`; *n_used = CTAs.
// pdl: launch as a programmatic dependent of the previous kernel (the
// kernels release their own dependents at once and wait for their
// predecessor before reading their input).
cudaError_t launch_amax(const void* x, long long n, unsigned* partial, int* n_used,
                        cudaStream_t s, bool pdl = false);
// The same over the rotated values of a [rows, K] tensor (rot = 16 or 32,
// times scale): one partial maximum per CTA as binary32 magnitude bits.
cudaError_t launch_amax_rot(const void* x, long long rows, int K, int rot, float scale,
                            unsigned* partial, int* n_used, cudaStream_t s, bool pdl = false);

struct QuantArgs {
  const void* x;        // bf16 [rows, K]
  long long rows;
  int K;
  int fmt;              // 0 NVFP4, 1 MXFP4
  int layout;           // 0 MMA, 1 row-major
  int dynamic;          // NVFP4: 1 = g from partial maxima, 0 = read *g
  float* g;
  const unsigned* partial;
  int n_partial;
  uint8_t* codes;
  uint8_t* scales;
  // MMA layout: also zero the scales of rows [rows, rows rounded up to 128).
  // The small-M GEMM never reads those rows' scales, so its chain skips it.
  int zero_pad_rows = 1;
  // Release the next kernel of the stream at once (programmatic dependent
  // launch) instead of at completion.  Only for a dependent known to read
  // this pass's output after its griddepcontrol.wait: the small-M GEMM may
  // stream its weights before that wait, so a pass that could be writing
  // weights must never release it early.
  int release_early = 0;
  // DYNAMIC, small tensors: every quantize CTA takes the magnitude maximum
  // of the whole tensor itself (no amax pass, no partial maxima)
  int self_amax = 0;
  // x is 32-byte aligned: a lane's 32 contiguous bytes come in one load
  // (set by launch_quantize)
  int wide = 0;
  // The status word a non-finite DYNAMIC maximum is reported in (set by
  // launch_quantize when null).
  unsigned* status = nullptr;
  // Online rotation: 0 (none), 16 or 32 (block-diagonal Walsh-Hadamard of
  // that order along K, then a multiply by rot_scale = 2^-shift).  The
  // partial maxima of a rotated tensor's amax pass are binary32 bits.
  int rot = 0;
  float rot_scale = 1.0f;
  // MXFP4 scale rule: 0 = OCP (floor(log2 amax) - 2), 1 = overflow-aware.
  int rule = 0;
  // MXFP4 macro-block scaling: one binary32 scale per row, written by the
  // row pass and read by the quantize pass (rot must be 0)
  float* mbs_sigma = nullptr;
};
cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t s, bool pdl = false);

// DYNAMIC tensors of at most this many bytes skip the amax pass: every
// quantize CTA reads the whole tensor for the global amax itself.  Measured
// on B200 (CUDA graph): 1 x 2880 4.4 -> 3.5 us; at 16 x 2880 (92 KB) the
// programmatic-dependent amax pass is cheaper (4.6 vs 5.0 us), so the limit
// covers single rows.
constexpr long long kSelfAmaxBytes = 32 << 10;

// Activation quantization: the amax pass (DYNAMIC; partial maxima into
// `partial`, kAmaxSlots entries) and the quantize pass, each a programmatic
// dependent of the kernel before it.  (One kernel on one thread-block
// cluster, reducing the amax over distributed shared memory, measured
// slower on B200 for every size: 16 SMs cannot match the full chip's
// bandwidth, and two launches cost ~5 us whatever the size.)
cudaError_t launch_quantize_act(QuantArgs a, unsigned* partial, cudaStream_t s);

}  // namespace fp4
#include "out_quant.cuh"
namespace fp4 {

struct GemmArgs {
  const uint8_t* a_codes; const uint8_t* a_scales; const float* g_a;
  const uint8_t* w_codes; const uint8_t* w_scales; const float* g_w;
  // MXFP4 macro-block scaling: per-row scales of A [M] and W [N] (both
  // null otherwise); C = sigma_a[m] * sigma_w[n] * acc
  const float* sigma_a = nullptr; const float* sigma_w = nullptr;
  int M, N, K, fmt;
  void* C; int ldc;
  int out_mode;         // 0 bf16 C, 1 fp32 C, 2 / 3 NVFP4 / MXFP4 activation (+ bf16 C if C)
  int max_sms;          // SMs the launch shape is chosen for, 0 = the device's
  QuantOut qo;          // out_mode 2, 3
};
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s);
// The shape launch_gemm takes: tile rows x columns, CTAs per tile along K.
// allow_split = false: the shape the FP4-emitting epilogue takes (no K split).
cudaError_t gemm_plan(int M, int N, int K, int max_sms, int* tile_m, int* tile_n, int* splits,
                      bool allow_split = true);
// The SMs a GEMM's launch shape is chosen for: max_sms when 0 < max_sms <
// the device's count, else the device's.
int gemm_sms(int max_sms);
// The CTA-pair kernel (256 x 256 tiles); launch_gemm takes it for M > 128
// when its tiles keep at least half the SMs busy.
cudaError_t launch_gemm_pair(const GemmArgs& a, cudaStream_t s);

// The grouped (mixture-of-experts) GEMM: group e multiplies rows
// [offsets[e], offsets[e+1]) of A by weight e of the stacked W (E x [N, K],
// per-expert scale blocks of w_sf_bytes, global scales g_w[e]); offsets is
// a device array of E + 1 ints.
struct GroupedArgs {
  const uint8_t* a_codes; const uint8_t* a_scales; const float* g_a;
  const uint8_t* w_codes; const uint8_t* w_scales; const float* g_w;
  const int* offsets;
  int E, M, N, K, fmt;
  void* C; int ldc; int out_f32;
  int max_sms;
};
cudaError_t launch_gemm_grouped(const GroupedArgs& a, cudaStream_t s);
// Its CTA-pair form (256 x 256 tiles), for groups of many rows.
cudaError_t launch_gemm_pair_grouped(const GroupedArgs& a, cudaStream_t s);

// Tensor map of packed FP4 codes [rows, K/2] bytes as a 2-D uint8 tensor:
// box of 128 bytes of K by box_rows rows, 128-byte swizzle, out-of-range
// rows and columns read as zero codes.
bool make_code_map(CUtensorMap* m, const uint8_t* base, long long rows, int K, int box_rows);

// Tensor map of a bf16 output C [rows, cols] with row pitch ldc elements:
// box of 64 columns (128 bytes) by box_rows rows, 128-byte swizzle.
bool make_bf16_out_map(CUtensorMap* m, void* C, long long rows, int cols, int ldc, int box_rows);
// The same for an fp32 C: box of 32 columns (128 bytes) by box_rows rows.
bool make_f32_out_map(CUtensorMap* m, void* C, long long rows, int cols, int ldc, int box_rows);

struct FusedArgs {
  const void* a;        // bf16 [M, K]
  const uint8_t* w_codes; const uint8_t* w_scales; const float* g_w;
  int M, N, K, fmt, dynamic;
  float* g_a;
  void* C; int ldc; int out_f32;
  void* ws; size_t ws_bytes;
  int max_sms;          // SMs the launch shape is chosen for, 0 = the device's
  int rot = 0;          // activation rotation (QuantArgs::rot), its scale, MXFP4 rule
  float rot_scale = 1.0f;
  int rule = 0;
};
size_t fused_workspace_bytes(int M, int N, int K, int fmt);
// Shapes the fused path takes: 1 <= M <= 32 and K up to 8 slices of 8192.
bool fused_supported(int M, int N, int K);
cudaError_t launch_gemm_fused(const FusedArgs& a, cudaStream_t s);
// The one-kernel path of launch_gemm_fused (M <= 32, M * K <= 128K values,
// K slices of at most 8 steps of 256).
bool decode_supported(int M, int N, int K, int max_sms);
cudaError_t launch_decode(const FusedArgs& a, cudaStream_t s);

}  // namespace fp4
