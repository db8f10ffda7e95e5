// fused.cu -- small-M (decode) entry: quantize the activation on the fly and
// multiply with pre-quantized weights.
//
// First version: the activation is quantized into the workspace (amax pass,
// quantize pass) and the tcgen05 GEMM consumes it.  Same arithmetic as
// fp4_quantize_act + fp4_gemm.
#include <algorithm>

#include "internal.h"

namespace fp4 {

namespace {
size_t align256(size_t b) { return (b + 255) / 256 * 256; }
}  // namespace

size_t fused_workspace_bytes(int M, int N, int K, int fmt) {
  (void)N;
  const int nsf = nsf_of(K, fmt);
  const size_t partial = static_cast<size_t>(kAmaxSlots) * sizeof(unsigned);
  const size_t codes = static_cast<size_t>(M) * (K / 2);
  const size_t scales = static_cast<size_t>(rows_pad128(M) / 128) * ncb_of(nsf) * 512;
  return align256(partial) + align256(codes) + align256(scales);
}

cudaError_t launch_gemm_fused(const FusedArgs& f, cudaStream_t s) {
  uint8_t* ws = static_cast<uint8_t*>(f.ws);
  const int nsf = nsf_of(f.K, f.fmt);
  unsigned* partial = reinterpret_cast<unsigned*>(ws);
  uint8_t* codes = ws + align256(static_cast<size_t>(kAmaxSlots) * sizeof(unsigned));
  uint8_t* scales = codes + align256(static_cast<size_t>(f.M) * (f.K / 2));
  (void)nsf;
  QuantArgs q{};
  q.x = f.a;
  q.rows = f.M;
  q.K = f.K;
  q.fmt = f.fmt;
  q.layout = 0;
  q.dynamic = f.dynamic;
  q.g = f.g_a;
  q.codes = codes;
  q.scales = scales;
  if (f.dynamic) {
    int used = 0;
    cudaError_t e = launch_amax(f.a, static_cast<long long>(f.M) * f.K, partial, &used, s);
    if (e != cudaSuccess) return e;
    q.partial = partial;
    q.n_partial = used;
  }
  cudaError_t e = launch_quantize(q, s);
  if (e != cudaSuccess) return e;
  GemmArgs g{};
  g.a_codes = codes;
  g.a_scales = scales;
  g.g_a = f.g_a;
  g.w_codes = f.w_codes;
  g.w_scales = f.w_scales;
  g.g_w = f.g_w;
  g.M = f.M;
  g.N = f.N;
  g.K = f.K;
  g.fmt = f.fmt;
  g.C = f.C;
  g.ldc = f.ldc;
  g.out_f32 = f.out_f32;
  return launch_gemm(g, s);
}

}  // namespace fp4
