// api.cu -- the extern "C" boundary: argument checks, workspace layout,
// status strings.  Every computing step runs in the kernels of
// quantize.cu, gemm.cu and fused.cu.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "fp4.h"
#include "internal.h"
#include "ptx.cuh"

namespace fp4 {

// The status word: kernels OR a bit into it when a bounded wait runs out
// (the WD_* codes of ptx.cuh) or when a DYNAMIC amax meets a non-finite
// input (WD_NONFINITE).
static __device__ unsigned int g_watchdog = 0;
// Where fp4_device_status's exchange leaves the word it took.  One slot for
// all callers: g_status_mutex keeps a second call's exchange from
// overwriting it before the first call has copied it out.
static __device__ unsigned int g_status_taken = 0;
static std::mutex g_status_mutex;

// Takes the status word and clears it in one atomic exchange, so that a bit
// a kernel on another stream sets meanwhile is never lost.
__global__ void status_take_kernel(unsigned* wd, unsigned* taken) {
  *taken = atomicExch(wd, 0u);
}

// The word's address on the current device (looked up once per device;
// concurrent first calls store the same address).
unsigned* watchdog_ptr() {
  static std::atomic<unsigned*> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  unsigned* p = cached[dev].load(std::memory_order_acquire);
  if (!p) {
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_watchdog) != cudaSuccess) return nullptr;
    p = static_cast<unsigned*>(q);
    cached[dev].store(p, std::memory_order_release);
  }
  return p;
}

// The watchdog self-test: one warp waits on an mbarrier that nothing
// arrives on, with a bounded wait of limit_ns, and returns.
__global__ void watchdog_selftest_kernel(unsigned* wd, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, wd, WD_SELFTEST, limit_ns);
}

}  // namespace fp4

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

fp4_status_t check_format(fp4_format_t f) {
  return (f == FP4_NVFP4 || f == FP4_MXFP4) ? FP4_OK : FP4_ERR_INVALID_ARG;
}

fp4_status_t check_rows_k(long long rows, int K) {
  if (rows < 0 || K <= 0) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (K % 32 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
  return FP4_OK;
}

fp4_status_t device_ok() {
  static std::atomic<int> cached[64] = {};   // 0 unknown, 1 ok, 2 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP4_ERR_NO_DEVICE;
  int c = cached[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return FP4_ERR_NO_DEVICE;
    c = (major == 10) ? 1 : 2;
    cached[dev].store(c, std::memory_order_relaxed);
  }
  return c == 1 ? FP4_OK : FP4_ERR_NO_DEVICE;
}

size_t quant_ws_bytes() { return fp4::quant_workspace_bytes(); }

fp4_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA; }

// Quantizer options -> (rotation order, 2^-shift, rule); weights take the
// smaller shift of the rotation, activations the larger (they add up to
// log2(n)).
struct Opts {
  int rot = 0;
  float rot_scale = 1.0f;
  int rule = 0;
  float* mbs = nullptr;
};
fp4_status_t parse_opts(const fp4_quant_opts_t* o, fp4_format_t fmt, bool weights, Opts* out) {
  *out = Opts{};
  if (!o) return FP4_OK;
  if (o->hadamard != 0 && o->hadamard != 16 && o->hadamard != 32) return FP4_ERR_INVALID_ARG;
  if (o->mx_rule != FP4_MX_RULE_OCP && o->mx_rule != FP4_MX_RULE_OAS) return FP4_ERR_INVALID_ARG;
  if (fmt == FP4_NVFP4 && o->mx_rule != FP4_MX_RULE_OCP) return FP4_ERR_INVALID_ARG;
  if (o->mbs_scale) {
    if (fmt != FP4_MXFP4 || o->hadamard != 0) return FP4_ERR_INVALID_ARG;
    if (!aligned4(o->mbs_scale)) return FP4_ERR_MISALIGNED;
    out->mbs = o->mbs_scale;
  }
  out->rot = o->hadamard;
  out->rule = o->mx_rule == FP4_MX_RULE_OAS ? 1 : 0;
  if (o->hadamard) {
    const int lg = o->hadamard == 16 ? 4 : 5;
    const int shift = weights ? lg / 2 : (lg + 1) / 2;
    out->rot_scale = 1.0f / static_cast<float>(1 << shift);
  }
  return FP4_OK;
}

fp4_status_t quantize_common(const void* x, int rows, int K, fp4_format_t fmt,
                             fp4_scale_layout_t layout, fp4_global_mode_t gmode,
                             const fp4_quant_opts_t* opts, bool weights, float* g,
                             uint8_t* codes, uint8_t* scales, void* ws, size_t ws_bytes,
                             void* stream) {
  fp4_status_t st;
  if ((st = check_format(fmt)) != FP4_OK) return st;
  if (layout != FP4_SCALES_MMA && layout != FP4_SCALES_ROWMAJOR) return FP4_ERR_INVALID_ARG;
  if (gmode != FP4_GLOBAL_DYNAMIC && gmode != FP4_GLOBAL_STATIC) return FP4_ERR_INVALID_ARG;
  Opts op;
  if ((st = parse_opts(opts, fmt, weights, &op)) != FP4_OK) return st;
  if ((st = check_rows_k(rows, K)) != FP4_OK) return st;
  if (rows == 0) return FP4_OK;   // nothing is read or written
  const bool nv = fmt == FP4_NVFP4;
  const bool dyn = nv && gmode == FP4_GLOBAL_DYNAMIC;
  if (!x || !codes || !scales || (nv && !g) || (dyn && !ws)) return FP4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (nv && !aligned4(g)) ||
      (dyn && !aligned16(ws)))
    return FP4_ERR_MISALIGNED;
  if (dyn && ws_bytes < quant_ws_bytes()) return FP4_ERR_WORKSPACE_TOO_SMALL;
  if ((st = device_ok()) != FP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fp4::QuantArgs a{};
  a.x = x;
  a.rows = rows;
  a.K = K;
  a.fmt = fmt;
  a.layout = layout;
  a.dynamic = dyn ? 1 : 0;
  a.g = g;
  a.codes = codes;
  a.scales = scales;
  a.rot = op.rot;
  a.rot_scale = op.rot_scale;
  a.rule = op.rule;
  a.mbs_sigma = op.mbs;
  // The amax pass (DYNAMIC) and the quantize pass, each a programmatic
  // dependent of the kernel before it (each waits for its predecessor before
  // reading), so its launch overlaps the predecessor's tail.  No pass
  // releases its own dependent early: a fused GEMM may read weights before
  // its wait.
  return from_cuda(fp4::launch_quantize_act(a, static_cast<unsigned*>(ws), s));
}

}  // namespace

extern "C" {

size_t fp4_packed_bytes(int rows, int K) {
  if (rows < 0 || K <= 0 || K % 2) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(K / 2);
}

size_t fp4_scale_bytes(int rows, int K, fp4_format_t fmt, fp4_scale_layout_t layout) {
  if (check_format(fmt) != FP4_OK || check_rows_k(rows, K) != FP4_OK) return 0;
  const int nsf = fp4::nsf_of(K, fmt);
  if (layout == FP4_SCALES_ROWMAJOR) return static_cast<size_t>(rows) * nsf;
  if (layout != FP4_SCALES_MMA) return 0;
  return static_cast<size_t>((rows + 127) / 128) * fp4::ncb_of(nsf) * 512u;
}

size_t fp4_workspace_bytes(int M, int N, int K, fp4_format_t fmt) {
  size_t w = quant_ws_bytes();
  if (M > 0 && N > 0 && K > 0 && K % 32 == 0 && check_format(fmt) == FP4_OK) {
    const size_t f = fp4::fused_workspace_bytes(M, N, K, fmt);
    if (f > w) w = f;
  }
  return w;
}

fp4_status_t fp4_quantize_act(const void* x, int rows, int K, fp4_format_t fmt,
                              fp4_scale_layout_t layout, fp4_global_mode_t gmode, float* g,
                              uint8_t* codes, uint8_t* scales, void* ws, size_t ws_bytes,
                              void* stream) {
  return quantize_common(x, rows, K, fmt, layout, gmode, nullptr, false, g, codes, scales, ws,
                         ws_bytes, stream);
}

fp4_status_t fp4_quantize_act_ex(const void* x, int rows, int K, fp4_format_t fmt,
                                 fp4_scale_layout_t layout, fp4_global_mode_t gmode,
                                 const fp4_quant_opts_t* opts, float* g, uint8_t* codes,
                                 uint8_t* scales, void* ws, size_t ws_bytes, void* stream) {
  return quantize_common(x, rows, K, fmt, layout, gmode, opts, false, g, codes, scales, ws,
                         ws_bytes, stream);
}

fp4_status_t fp4_quantize_weights(const void* w, int N, int K, fp4_format_t fmt, uint8_t* codes,
                                  uint8_t* scales, float* g, void* ws, size_t ws_bytes,
                                  void* stream) {
  return quantize_common(w, N, K, fmt, FP4_SCALES_MMA, FP4_GLOBAL_DYNAMIC, nullptr, true, g,
                         codes, scales, ws, ws_bytes, stream);
}

fp4_status_t fp4_quantize_weights_ex(const void* w, int N, int K, fp4_format_t fmt,
                                     const fp4_quant_opts_t* opts, uint8_t* codes,
                                     uint8_t* scales, float* g, void* ws, size_t ws_bytes,
                                     void* stream) {
  return quantize_common(w, N, K, fmt, FP4_SCALES_MMA, FP4_GLOBAL_DYNAMIC, opts, true, g, codes,
                         scales, ws, ws_bytes, stream);
}

fp4_status_t fp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                      const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w, int M,
                      int N, int K, fp4_format_t fmt, void* C, int ldc, fp4_out_t out, void* ws,
                      size_t ws_bytes, int max_sms, void* stream) {
  (void)ws;
  (void)ws_bytes;
  fp4_status_t st;
  if ((st = check_format(fmt)) != FP4_OK) return st;
  if (out != FP4_OUT_BF16 && out != FP4_OUT_F32) return FP4_ERR_INVALID_ARG;
  if (max_sms < 0) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || (st = check_rows_k(M, K)) != FP4_OK) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (N % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return FP4_OK;   // nothing is read or written
  const bool nv = fmt == FP4_NVFP4;
  if (!a_codes || !a_scales || !w_codes || !w_scales || !C || (nv && (!g_a || !g_w)))
    return FP4_ERR_INVALID_ARG;
  if (ldc < N) return FP4_ERR_INVALID_ARG;
  const int esize = out == FP4_OUT_F32 ? 4 : 2;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(C) || (static_cast<long long>(ldc) * esize) % 16 != 0 ||
      (nv && (!aligned4(g_a) || !aligned4(g_w))))
    return FP4_ERR_MISALIGNED;
  if ((st = device_ok()) != FP4_OK) return st;
  fp4::GemmArgs a{};
  a.a_codes = a_codes;
  a.a_scales = a_scales;
  a.g_a = g_a;
  a.w_codes = w_codes;
  a.w_scales = w_scales;
  a.g_w = g_w;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = fmt;
  a.C = C;
  a.ldc = ldc;
  a.out_mode = out == FP4_OUT_F32 ? 1 : 0;
  a.max_sms = max_sms;
  return from_cuda(fp4::launch_gemm(a, static_cast<cudaStream_t>(stream)));
}

fp4_status_t fp4_gemm_quant(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                            const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                            int M, int N, int K, fp4_format_t fmt, fp4_format_t out_fmt,
                            fp4_scale_layout_t out_layout, const fp4_quant_opts_t* out_opts,
                            const float* g_out, uint8_t* out_codes, uint8_t* out_scales, void* C,
                            int ldc, void* ws, size_t ws_bytes, int max_sms, void* stream) {
  (void)ws;
  (void)ws_bytes;
  fp4_status_t st;
  if ((st = check_format(fmt)) != FP4_OK || (st = check_format(out_fmt)) != FP4_OK) return st;
  if (out_layout != FP4_SCALES_MMA && out_layout != FP4_SCALES_ROWMAJOR) return FP4_ERR_INVALID_ARG;
  Opts op;
  if ((st = parse_opts(out_opts, out_fmt, false, &op)) != FP4_OK) return st;
  if (op.mbs) return FP4_ERR_INVALID_ARG;   // no macro-block scaling in the emitting epilogue
  if (max_sms < 0) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || (st = check_rows_k(M, K)) != FP4_OK) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (N % 32 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;   // N is the next layer's K
  if (M == 0 || N == 0) return FP4_OK;
  const bool nv = fmt == FP4_NVFP4, nv_out = out_fmt == FP4_NVFP4;
  if (!a_codes || !a_scales || !w_codes || !w_scales || !out_codes || !out_scales ||
      (nv && (!g_a || !g_w)) || (nv_out && !g_out))
    return FP4_ERR_INVALID_ARG;
  if (C && ldc < N) return FP4_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(out_codes) || !aligned16(out_scales) ||
      (C && (!aligned16(C) || (static_cast<long long>(ldc) * 2) % 16 != 0)) ||
      (nv && (!aligned4(g_a) || !aligned4(g_w))) || (nv_out && !aligned4(g_out)))
    return FP4_ERR_MISALIGNED;
  if ((st = device_ok()) != FP4_OK) return st;
  fp4::GemmArgs a{};
  a.a_codes = a_codes;
  a.a_scales = a_scales;
  a.g_a = g_a;
  a.w_codes = w_codes;
  a.w_scales = w_scales;
  a.g_w = g_w;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = fmt;
  a.C = C;
  a.ldc = C ? ldc : N;
  a.out_mode = nv_out ? 2 : 3;
  a.max_sms = max_sms;
  a.qo.codes = out_codes;
  a.qo.scales = out_scales;
  a.qo.g = g_out;
  a.qo.fmt = nv_out ? 0 : 1;
  a.qo.layout = out_layout == FP4_SCALES_ROWMAJOR ? 1 : 0;
  a.qo.rule = op.rule;
  a.qo.rot = op.rot;
  a.qo.rot_scale = op.rot_scale;
  a.qo.nsf = fp4::nsf_of(N, a.qo.fmt);
  a.qo.ncb = fp4::ncb_of(a.qo.nsf);
  return from_cuda(fp4::launch_gemm(a, static_cast<cudaStream_t>(stream)));
}

fp4_status_t fp4_gemm_mbs(const uint8_t* a_codes, const uint8_t* a_scales, const float* sigma_a,
                          const uint8_t* w_codes, const uint8_t* w_scales, const float* sigma_w,
                          int M, int N, int K, void* C, int ldc, fp4_out_t out, void* ws,
                          size_t ws_bytes, int max_sms, void* stream) {
  (void)ws;
  (void)ws_bytes;
  fp4_status_t st;
  if (out != FP4_OUT_BF16 && out != FP4_OUT_F32) return FP4_ERR_INVALID_ARG;
  if (max_sms < 0) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || (st = check_rows_k(M, K)) != FP4_OK) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (N % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return FP4_OK;
  if (!a_codes || !a_scales || !w_codes || !w_scales || !C || !sigma_a || !sigma_w)
    return FP4_ERR_INVALID_ARG;
  if (ldc < N) return FP4_ERR_INVALID_ARG;
  const int esize = out == FP4_OUT_F32 ? 4 : 2;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(C) || (static_cast<long long>(ldc) * esize) % 16 != 0 || !aligned4(sigma_a) ||
      !aligned4(sigma_w))
    return FP4_ERR_MISALIGNED;
  if ((st = device_ok()) != FP4_OK) return st;
  fp4::GemmArgs a{};
  a.a_codes = a_codes;
  a.a_scales = a_scales;
  a.w_codes = w_codes;
  a.w_scales = w_scales;
  a.sigma_a = sigma_a;
  a.sigma_w = sigma_w;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = FP4_MXFP4;
  a.C = C;
  a.ldc = ldc;
  a.out_mode = out == FP4_OUT_F32 ? 5 : 4;
  a.max_sms = max_sms;
  return from_cuda(fp4::launch_gemm(a, static_cast<cudaStream_t>(stream)));
}

fp4_status_t fp4_gemm_grouped(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                              const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                              const int* offsets, int E, int M, int N, int K, fp4_format_t fmt,
                              void* C, int ldc, fp4_out_t out, void* ws, size_t ws_bytes,
                              int max_sms, void* stream) {
  (void)ws;
  (void)ws_bytes;
  fp4_status_t st;
  if ((st = check_format(fmt)) != FP4_OK) return st;
  if (out != FP4_OUT_BF16 && out != FP4_OUT_F32) return FP4_ERR_INVALID_ARG;
  if (max_sms < 0) return FP4_ERR_INVALID_ARG;
  if (E < 1 || E > fp4::kGroupedMaxGroups) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || (st = check_rows_k(M, K)) != FP4_OK) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (N % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return FP4_OK;   // nothing is read or written
  const bool nv = fmt == FP4_NVFP4;
  if (!a_codes || !a_scales || !w_codes || !w_scales || !offsets || !C ||
      (nv && (!g_a || !g_w)))
    return FP4_ERR_INVALID_ARG;
  if (ldc < N) return FP4_ERR_INVALID_ARG;
  const int esize = out == FP4_OUT_F32 ? 4 : 2;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(C) || !aligned4(offsets) || (static_cast<long long>(ldc) * esize) % 16 != 0 ||
      (nv && (!aligned4(g_a) || !aligned4(g_w))))
    return FP4_ERR_MISALIGNED;
  if ((st = device_ok()) != FP4_OK) return st;
  fp4::GroupedArgs a{};
  a.a_codes = a_codes;
  a.a_scales = a_scales;
  a.g_a = g_a;
  a.w_codes = w_codes;
  a.w_scales = w_scales;
  a.g_w = g_w;
  a.offsets = offsets;
  a.E = E;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = fmt;
  a.C = C;
  a.ldc = ldc;
  a.out_f32 = out == FP4_OUT_F32;
  a.max_sms = max_sms;
  return from_cuda(fp4::launch_gemm_grouped(a, static_cast<cudaStream_t>(stream)));
}

fp4_status_t fp4_gemm_plan(int M, int N, int K, fp4_format_t fmt, int max_sms, int* tile_m,
                           int* tile_n, int* splits) {
  fp4_status_t st;
  if ((st = check_format(fmt)) != FP4_OK) return st;
  if (M < 0 || N < 0 || (st = check_rows_k(M, K)) != FP4_OK) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (N % 8 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (!tile_m || !tile_n || !splits || max_sms < 0) return FP4_ERR_INVALID_ARG;
  if ((st = device_ok()) != FP4_OK) return st;
  return from_cuda(fp4::gemm_plan(M, N, K, max_sms, tile_m, tile_n, splits));
}

fp4_status_t fp4_gemm_fused(const void* x, const uint8_t* w_codes, const uint8_t* w_scales,
                            const float* g_w, int M, int N, int K, fp4_format_t fmt,
                            fp4_global_mode_t gmode, float* g_a, void* C, int ldc, fp4_out_t out,
                            void* ws, size_t ws_bytes, int max_sms, void* stream) {
  return fp4_gemm_fused_ex(x, w_codes, w_scales, g_w, M, N, K, fmt, gmode, nullptr, g_a, C, ldc,
                           out, ws, ws_bytes, max_sms, stream);
}

fp4_status_t fp4_gemm_fused_ex(const void* x, const uint8_t* w_codes, const uint8_t* w_scales,
                               const float* g_w, int M, int N, int K, fp4_format_t fmt,
                               fp4_global_mode_t gmode, const fp4_quant_opts_t* opts, float* g_a,
                               void* C, int ldc, fp4_out_t out, void* ws, size_t ws_bytes,
                               int max_sms, void* stream) {
  fp4_status_t st;
  if ((st = check_format(fmt)) != FP4_OK) return st;
  Opts op;
  if ((st = parse_opts(opts, fmt, false, &op)) != FP4_OK) return st;
  if (op.mbs) return FP4_ERR_INVALID_ARG;   // the fused path has no macro-block scaling
  if (out != FP4_OUT_BF16 && out != FP4_OUT_F32) return FP4_ERR_INVALID_ARG;
  if (gmode != FP4_GLOBAL_DYNAMIC && gmode != FP4_GLOBAL_STATIC) return FP4_ERR_INVALID_ARG;
  if (max_sms < 0) return FP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || (st = check_rows_k(M, K)) != FP4_OK) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (N % 8 != 0 || M > 32) return FP4_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return FP4_OK;   // nothing is read or written
  if (!fp4::fused_supported(M, N, K)) return FP4_ERR_UNSUPPORTED_SHAPE;
  const bool nv = fmt == FP4_NVFP4;
  if (!x || !w_codes || !w_scales || !C || !ws || (nv && (!g_a || !g_w)))
    return FP4_ERR_INVALID_ARG;
  if (ldc < N) return FP4_ERR_INVALID_ARG;
  const int esize = out == FP4_OUT_F32 ? 4 : 2;
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(C) ||
      !aligned16(ws) || (static_cast<long long>(ldc) * esize) % 16 != 0 ||
      (nv && (!aligned4(g_a) || !aligned4(g_w))))
    return FP4_ERR_MISALIGNED;
  if (ws_bytes < fp4::fused_workspace_bytes(M, N, K, fmt)) return FP4_ERR_WORKSPACE_TOO_SMALL;
  if ((st = device_ok()) != FP4_OK) return st;
  fp4::FusedArgs a{};
  a.a = x;
  a.w_codes = w_codes;
  a.w_scales = w_scales;
  a.g_w = g_w;
  a.M = M;
  a.N = N;
  a.K = K;
  a.fmt = fmt;
  a.dynamic = (nv && gmode == FP4_GLOBAL_DYNAMIC) ? 1 : 0;
  a.g_a = g_a;
  a.C = C;
  a.ldc = ldc;
  a.out_f32 = out == FP4_OUT_F32;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.max_sms = max_sms;
  a.rot = op.rot;
  a.rot_scale = op.rot_scale;
  a.rule = op.rule;
  return from_cuda(fp4::launch_gemm_fused(a, static_cast<cudaStream_t>(stream)));
}

fp4_status_t fp4_watchdog_selftest(unsigned long long limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return FP4_ERR_INVALID_ARG;
  fp4_status_t st;
  if ((st = device_ok()) != FP4_OK) return st;
  unsigned* wd = fp4::watchdog_ptr();
  if (!wd) return FP4_ERR_CUDA;
  fp4::watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(wd, limit_ns);
  return from_cuda(cudaGetLastError());
}

fp4_status_t fp4_device_status(unsigned* code, void* stream) {
  if (!code) return FP4_ERR_INVALID_ARG;
  fp4_status_t st;
  if ((st = device_ok()) != FP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned* wd = fp4::watchdog_ptr();
  std::lock_guard<std::mutex> lock(fp4::g_status_mutex);
  void* taken = nullptr;
  if (!wd || cudaGetSymbolAddress(&taken, fp4::g_status_taken) != cudaSuccess) return FP4_ERR_CUDA;
  fp4::status_take_kernel<<<1, 1, 0, s>>>(wd, static_cast<unsigned*>(taken));
  if (cudaGetLastError() != cudaSuccess) return FP4_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, fp4::g_status_taken, sizeof v, 0, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return FP4_ERR_CUDA;
  *code = v;
  if (v & ~static_cast<unsigned>(fp4::WD_NONFINITE)) return FP4_ERR_DEVICE_TIMEOUT;
  return v ? FP4_ERR_NONFINITE : FP4_OK;
}

const char* fp4_status_string(fp4_status_t s) {
  switch (s) {
    case FP4_OK: return "ok";
    case FP4_ERR_INVALID_ARG: return "invalid argument";
    case FP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case FP4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case FP4_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case FP4_ERR_CUDA: return "CUDA error";
    case FP4_ERR_DEVICE_TIMEOUT: return "a device-side bounded wait timed out";
    case FP4_ERR_NO_DEVICE: return "no sm_100 device is current";
    case FP4_ERR_NONFINITE: return "a dynamic global-scale reduction met an Inf or NaN input";
  }
  return "unknown status";
}

}  // extern "C"
