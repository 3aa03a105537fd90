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

// The driver context current on this thread (null if none, or if the driver
// entry point is unavailable), fetched through the runtime so that the
// library does not link libcuda.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);

CUcontext current_context() {
  static CtxGetCurrentFn fn = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(f);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// The array's device address as seen from the context that is current now.
// In host code the symbol itself is only a host-side stand-in, so the address
// is looked up with the device current (cudaGetSymbolAddress) the first time a
// device is used, and again whenever a different driver context is current on
// that device (each context loads its own copy of the library's module).
struct ScratchSlot {
  CUcontext ctx = nullptr;
  void *ptr = nullptr;
};
std::mutex g_scratch_mutex;
ScratchSlot g_scratch[kMaxDevicesPerProcess];

cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevicesPerProcess) return cudaErrorInvalidDevice;
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot &s = g_scratch[dev];
  if (s.ptr == nullptr || s.ctx != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fwd_scratch);
    if (e != cudaSuccess) return e;
    s.ptr = p;
    s.ctx = ctx;
  }
  *out = s.ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace qlora

extern "C" int qlora_linear_fwd_noalloc(const uint16_t *X, int64_t m, const qlora_nf4_weight *w,
                                        const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                                        uint16_t *Y, qlora_stream_t stream) {
  // The same checks, in the same order, as qlora_linear_fwd; the built-in
  // scratch then stands where the caller's workspace would be checked.
  bool lora = false;
  int st = qlora::validate_fwd(X, m, w, A, B, r, Y, &lora);
  if (st != QLORA_OK || m == 0) return st;
  void *scratch = nullptr;
  if (lora && qlora_workspace_bytes(QLORA_OP_FWD, m, w->n, w->k, r) > qlora::kNoallocScratchBytes)
    return QLORA_ERR_WORKSPACE;
  st = qlora::check_device();
  if (st != QLORA_OK) return st;
  if (lora) {
    const cudaError_t e = qlora::scratch_address(&scratch);
    if (e != cudaSuccess) return qlora::status_from_cuda(e);
  }
  return qlora::launch_fwd(X, X, m, w, A, B, r, scale, Y, static_cast<uint16_t *>(scratch),
                           reinterpret_cast<cudaStream_t>(stream));
}
