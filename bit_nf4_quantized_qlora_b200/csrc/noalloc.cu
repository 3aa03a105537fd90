// Forward entry point that needs no caller workspace and allocates nothing.
//
// qlora_linear_fwd needs scratch for the rank-r intermediate T = bf16(s X A^T)
// and takes it from a caller workspace.  Some callers cannot provide one: code
// that must not allocate device memory after start-up (an inference engine
// plugin whose host owns every device allocation, a real-time or
// certification-bound deployment that forbids allocation on its serving
// path, a C caller with no device allocator of its own).  For them this file
// holds the scratch in a fixed device array that lives as long as the library
// is loaded, and the entry point below passes it to the existing forward.
#include <cstdint>
#include <mutex>

#include "../../include/qlora.h"
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr size_t kNoallocScratchBytes = QLORA_NOALLOC_SCRATCH_BYTES;

// Every device that loads the library holds this array until process exit.
static __device__ __align__(256) unsigned char g_fwd_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// The array's device address for the current device.  In host code the
// symbol itself is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaFree(nullptr);   // a context current on this thread before the lookup
    if (e != cudaSuccess) return e;
    e = cudaGetSymbolAddress(&p, g_fwd_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace qlora

extern "C" int qlora_linear_fwd_noalloc(const uint16_t *X, int64_t m, const qlora_nf4_weight *w,
                                        const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                                        uint16_t *Y, qlora_stream_t stream) {
  if (!w) return QLORA_ERR_NULL;
  void *scratch = nullptr;
  size_t cap = 0;
  const bool lora = r > 0 && (A != nullptr || B != nullptr);
  // Only a well-formed adapter call needs the scratch; everything else is
  // validated (and rejected) by qlora_linear_fwd exactly as for any caller.
  if (lora && m > 0 && (r % 16) == 0 && r <= 256 && w->n > 0 && w->k > 0) {
    const size_t need = qlora_workspace_bytes(QLORA_OP_FWD, m, w->n, w->k, r);
    if (need > qlora::kNoallocScratchBytes) return QLORA_ERR_WORKSPACE;
    const cudaError_t e = qlora::scratch_address(&scratch);
    if (e != cudaSuccess) return qlora::status_from_cuda(e);
    cap = qlora::kNoallocScratchBytes;
  }
  return qlora_linear_fwd(X, m, w, A, B, r, scale, Y, scratch, cap, stream);
}
