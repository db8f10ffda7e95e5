// noalloc.cu -- fp4_quantize_act_noalloc: activation quantization for
// callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: engines that
// reserve all device memory up front for weights and caches and forbid
// later allocations, plug-ins running inside a host framework that owns the
// allocator and gives them no scratch, and real-time paths that cannot
// afford cudaMalloc's implicit device synchronization.  This entry
// point quantizes exactly like fp4_quantize_act, but the scratch that the
// DYNAMIC global-scale reduction needs (one partial maximum per amax CTA)
// lives in a fixed file-scope device array instead of a caller workspace.
//
// The array is kNoAllocScratchBytes (4 KiB) and exists on every GPU that
// loads the library, until the process exits.  All calls share it, so two
// calls that overlap on the GPU (different streams, or different host
// threads on the same device) race on it.  It keeps the last call's
// contents; nothing in it needs clearing, because every call writes each
// slot it later reads.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp4.h"
#include "internal.h"

namespace fp4 {
namespace {

constexpr size_t kNoAllocScratchBytes = 4096;
static_assert(kNoAllocScratchBytes >= static_cast<size_t>(kAmaxSlots) * sizeof(unsigned),
              "the scratch must hold every partial maximum of the amax pass");
// (the size check in the entry point compares quant_workspace_bytes(), the
// rule fp4_quantize_act applies, with this limit)

// Device-side scratch.  In host code this name is only a host-side stand-in
// for the symbol, never a device address: its address on a device comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[64] = {nullptr};

// Looks up the scratch array's device address on the current device (once
// per device, with that device current).
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace fp4

extern "C" fp4_status_t fp4_quantize_act_noalloc(const void* x, int rows, int K,
                                                 fp4_format_t fmt, fp4_scale_layout_t layout,
                                                 fp4_global_mode_t gmode, float* g,
                                                 uint8_t* codes, uint8_t* scales, void* stream) {
  if (fmt != FP4_NVFP4 && fmt != FP4_MXFP4) return FP4_ERR_INVALID_ARG;
  if (layout != FP4_SCALES_MMA && layout != FP4_SCALES_ROWMAJOR) return FP4_ERR_INVALID_ARG;
  if (gmode != FP4_GLOBAL_DYNAMIC && gmode != FP4_GLOBAL_STATIC) return FP4_ERR_INVALID_ARG;
  if (rows < 0 || K <= 0 || K % 32 != 0) return FP4_ERR_UNSUPPORTED_SHAPE;
  // the scratch fp4_quantize_act needs (the same rule) must fit the array
  if (fp4::quant_workspace_bytes() > fp4::kNoAllocScratchBytes) return FP4_ERR_WORKSPACE_TOO_SMALL;
  if (rows == 0) return FP4_OK;
  const bool dyn = fmt == FP4_NVFP4 && gmode == FP4_GLOBAL_DYNAMIC;
  void* scratch = nullptr;
  if (dyn && fp4::scratch_for_current_device(&scratch) != cudaSuccess) return FP4_ERR_CUDA;
  return fp4_quantize_act(x, rows, K, fmt, layout, gmode, g, codes, scales, scratch,
                          dyn ? fp4::kNoAllocScratchBytes : 0, stream);
}
