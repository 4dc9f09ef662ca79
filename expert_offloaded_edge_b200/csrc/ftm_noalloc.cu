// Whole-layer forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside a CUDA
// graph being captured, allocator-free embedded runtimes, or engines whose
// memory is fully reserved up front.  ftm_moe_layer_forward_noalloc serves
// them: its scratch (routing ids, gates, permutation, gathered activations,
// the SwiGLU intermediate and the expert outputs) lives in one file-scope
// device array of kNoAllocScratchBytes bytes, owned by the library and kept
// on every GPU that loads it until the process exits.
//
// In host code the array's name is only a host-side stand-in, never a device
// address.  The real address is looked up once per device, with that device
// current, by cudaGetSymbolAddress on the first call made on the device; that
// first call should therefore come before any stream capture.
#include <stdio.h>

#include <mutex>

#include "ftm_common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

}  // namespace

extern "C" ftm_status ftm_moe_layer_forward_noalloc(const ftm_layer_desc* L, const ftm_layer_weights* W,
                                                    const void* x, int32_t T, void* out, void* stream) {
  const size_t need = ftm_workspace_bytes(L, T);
  if (need == 0)  // invalid descriptor or T: let the regular entry point report it
    return ftm_moe_layer_forward(L, W, nullptr, x, T, out, nullptr, 0, stream, nullptr);
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "ftm_moe_layer_forward_noalloc: T=%d needs %zu bytes of scratch, above the static limit of %zu bytes", T,
             need, kNoAllocScratchBytes);
    return ftm::report_error(FTM_ERR_INVALID_ARG, msg);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return ftm::report_error(FTM_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return ftm::report_error(FTM_ERR_UNSUPPORTED, "device index above 63");
  void* ptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    ptr = g_scratch_ptr[dev];
    if (!ptr) {
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess || !ptr) {
        char msg[200];
        snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
        return ftm::report_error(FTM_ERR_CUDA, msg);
      }
      g_scratch_ptr[dev] = ptr;
    }
  }
  // Every call shares this scratch.  Every byte of it that the layer reads is
  // written earlier in the same call, so nothing needs clearing between calls.
  return ftm_moe_layer_forward(L, W, nullptr, x, T, out, ptr, kNoAllocScratchBytes, stream, nullptr);
}
