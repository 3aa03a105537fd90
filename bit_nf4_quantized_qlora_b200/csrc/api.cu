// C ABI of libqlora (declared in include/qlora.h): argument validation on the
// host, workspace carving, dispatch by M, and status reporting.  Every check
// runs before the first launch of a call, so a call that returns an error has
// launched nothing.
#include <atomic>
#include <climits>
#include <cstdint>
#include <cmath>
#include <cstring>

#include "../../include/qlora.h"
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

__device__ unsigned g_device_error = 0u;

thread_local int t_last_cuda_error = 0;
thread_local cudaEvent_t t_prof_start = nullptr;
thread_local cudaEvent_t t_prof_stop = nullptr;
std::atomic<uint64_t> g_launches{0};

// Record the caller's profiling event (if any) on the call's stream.
cudaError_t prof_mark(cudaEvent_t ev, cudaStream_t s) { return ev ? cudaEventRecord(ev, s) : cudaSuccess; }

constexpr int64_t kSmallM = 16;       // m <= 16: weight-streaming forward
constexpr size_t kWsAlign = 256;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QLORA_OK;
  t_last_cuda_error = static_cast<int>(e);
  return QLORA_ERR_CUDA;
}

size_t round_up(size_t v) { return (v + kWsAlign - 1) / kWsAlign * kWsAlign; }

// The linear operations also need n % 8 == 0 (16-byte rows of Y and dY).
int check_weight(const qlora_nf4_weight *w, bool linear = true) {
  if (!w || !w->codes || !w->absmax_q || !w->group_scale) return QLORA_ERR_NULL;
  if (w->n <= 0 || w->k <= 0 || (w->k % 64) != 0) return QLORA_ERR_SHAPE;
  if (linear && (w->n % 8) != 0) return QLORA_ERR_SHAPE;
  if (w->block != 64 || w->group != 256) return QLORA_ERR_SHAPE;
  if (w->codebook < 0 || w->codebook >= kCodebookCount) return QLORA_ERR_CODEBOOK;
  if (w->dq_format < 0 || w->dq_format >= kDqFormatCount) return QLORA_ERR_FORMAT;
  if (w->n > (int64_t(1) << 31) || w->k > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (!aligned16(w->codes) || !aligned16(w->absmax_q) || !aligned16(w->group_scale)) return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

// r == 0 or A == B == NULL: no adapter.  Otherwise both pointers, r % 16 == 0.
int check_adapter(const uint16_t *A, const uint16_t *B, int32_t r, bool *use) {
  *use = false;
  if (r < 0 || r > 256 || (r % 16) != 0) return QLORA_ERR_SHAPE;
  if (r == 0 || (A == nullptr && B == nullptr)) return QLORA_OK;
  if (A == nullptr || B == nullptr) return QLORA_ERR_NULL;
  if (!aligned16(A) || !aligned16(B)) return QLORA_ERR_ALIGN;
  *use = true;
  return QLORA_OK;
}

WeightView view(const qlora_nf4_weight *w) {
  return WeightView{w->codes, w->absmax_q, w->group_scale, w->n, w->k, &codebook_tables(w->codebook),
                    mean_ptr(w->group_scale, w->n * w->k / 64, w->dq_format)};
}

constexpr int kMaxDevices = kMaxDevicesPerProcess;

// The dropout constants of probability p: threshold = round_half_even(fp32(p)
// . 65536) for the 16-bit keep test, keep_scale = fp32(1 / fp32(1 - p)).
// False unless 0 <= p < 1.
bool dropout_params(float p, uint64_t seed, uint64_t offset, DropoutParams *d) {
  if (!(p >= 0.0f && p < 1.0f)) return false;
  d->seed = seed;
  d->offset = offset;
  d->threshold = static_cast<uint32_t>(std::nearbyint(static_cast<double>(p) * 65536.0));
  const float one = 1.0f;
  const volatile float q = one - p;   // rounded to fp32 before the division
  d->keep_scale = one / q;
  return true;
}

}  // namespace

// The device the calls run on must be sm_100.  The first call on a host
// thread also makes sure the runtime has a context current on that thread
// (a thread that never touched CUDA, such as a framework's worker thread, may
// have none yet; kernel configuration calls made before it is bound have
// failed with cudaErrorInvalidValue).  cudaSetDevice binds the device's
// primary context to the calling thread and allocates nothing.
int check_device() {
  thread_local int t_ready_dev = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (t_ready_dev != dev) {
    e = cudaSetDevice(dev);
    if (e != cudaSuccess) return cuda_status(e);
    t_ready_dev = dev;
  }
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_status(e);
  return major == 10 ? QLORA_OK : QLORA_ERR_DEVICE;
}

int status_from_cuda(cudaError_t e) { return cuda_status(e); }

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

// The error word's device address, looked up once per device.  Two threads
// on a fresh device may both look it up; they store the same value, and the
// slots are atomics, so the race is harmless.
unsigned *device_error_word() {
  static std::atomic<unsigned *> cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot) {
    unsigned *p = cache[dev].load(std::memory_order_acquire);
    if (p) return p;
  }
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_device_error) != cudaSuccess) return nullptr;
  if (slot) cache[dev].store(static_cast<unsigned *>(ptr), std::memory_order_release);
  return static_cast<unsigned *>(ptr);
}

cudaError_t set_smem_once(const void *kernel, int smem_bytes, std::atomic<bool> *done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e == cudaSuccess && slot) done[dev].store(true, std::memory_order_release);
  return e;
}

int validate_fwd(const uint16_t *X, int64_t m, const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B,
                 int32_t r, uint16_t *Y, bool *use_adapter) {
  int st = check_weight(w);
  if (st != QLORA_OK) return st;
  st = check_adapter(A, B, r, use_adapter);
  if (st != QLORA_OK) return st;
  if (m < 0 || m > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (m == 0) return QLORA_OK;
  if (!X || !Y) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(Y)) return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

int launch_fwd(const uint16_t *X, const uint16_t *Xa, int64_t m, const qlora_nf4_weight *w, const uint16_t *A,
               const uint16_t *B, int32_t r, float scale, uint16_t *Y, uint16_t *T, cudaStream_t s) {
  const bool lora = T != nullptr;
  cudaError_t e = cudaSuccess;
  // The main kernel overlaps the adapter projection (programmatic dependent
  // launch) unless the caller is timing the main kernel alone.
  const bool pdl = lora && t_prof_start == nullptr;
  if (m <= kSmallM) {
    if (lora) e = launch_lora_proj_small(Xa, m, w->k, A, r, scale, T, s);
    if (e == cudaSuccess) e = prof_mark(t_prof_start, s);
    if (e == cudaSuccess) {
      // Decode sizes take the per-warp streaming kernel; the rest (m > 4,
      // or K beyond one cluster's warps) the CTA-ring kernel.
      e = gemv_stream_supported(m, w->n, w->k)
              ? launch_gemv_stream(X, m, w->codes, w->absmax_q, w->group_scale, view(w).mu, w->n, w->k, T,
                                   lora ? B : nullptr, lora ? r : 0, Y, codebook_tables(w->codebook), s, pdl)
              : launch_gemv_fwd(X, m, w->codes, w->absmax_q, w->group_scale, view(w).mu, w->n, w->k, T,
                                lora ? B : nullptr, lora ? r : 0, Y, codebook_tables(w->codebook), s, pdl);
    }
  } else {
    if (lora) e = tc_proj_kmajor(Xa, m, w->k, A, r, scale, T, s);
    if (e == cudaSuccess) e = prof_mark(t_prof_start, s);
    if (e == cudaSuccess) e = tc_fwd(X, m, view(w), T, lora ? B : nullptr, lora ? r : 0, Y, s, pdl);
  }
  if (e == cudaSuccess) e = prof_mark(t_prof_stop, s);
  return cuda_status(e);
}

}  // namespace qlora

using namespace qlora;

extern "C" {

int qlora_version(void) { return (1 << 16) | 1; }

int qlora_last_cuda_error(void) { return t_last_cuda_error; }

int qlora_set_profile_events(void *start, void *stop) {
  if ((start == nullptr) != (stop == nullptr)) return QLORA_ERR_NULL;
  t_prof_start = static_cast<cudaEvent_t>(start);
  t_prof_stop = static_cast<cudaEvent_t>(stop);
  return QLORA_OK;
}

uint64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *qlora_status_string(int status) {
  switch (status) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_NULL: return "QLORA_ERR_NULL: a required pointer is NULL";
    case QLORA_ERR_SHAPE: return "QLORA_ERR_SHAPE: a size breaks the shape rules";
    case QLORA_ERR_ALIGN: return "QLORA_ERR_ALIGN: a pointer is not 16-byte aligned";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE: workspace missing or too small";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA: a CUDA call failed";
    case QLORA_ERR_DEVICE: return "QLORA_ERR_DEVICE: the current device is not sm_100";
    case QLORA_ERR_CODEBOOK: return "QLORA_ERR_CODEBOOK: unknown codebook";
    case QLORA_ERR_FORMAT: return "QLORA_ERR_FORMAT: unknown absmax storage format";
    default: return "unknown qlora status";
  }
}

void qlora_nf4_levels(float *levels) {
  if (!levels) return;
  std::memcpy(levels, nf4_tables().level, sizeof(float) * 16);
}

int qlora_codebook_levels(int32_t codebook, float *levels) {
  if (!levels) return QLORA_ERR_NULL;
  if (codebook < 0 || codebook >= kCodebookCount) return QLORA_ERR_CODEBOOK;
  std::memcpy(levels, codebook_tables(codebook).level, sizeof(float) * 16);
  return QLORA_OK;
}

size_t qlora_workspace_bytes(int op, int64_t m, int64_t n, int64_t k, int32_t r) {
  if (m < 0 || n <= 0 || k <= 0 || r < 0) return SIZE_MAX;
  const size_t mr = round_up(static_cast<size_t>(m) * static_cast<size_t>(r) * 2u);
  switch (op) {
    case QLORA_OP_FWD: return r > 0 ? mr : 0;
    case QLORA_OP_BWD_DX: return r > 0 ? mr : 0;
    case QLORA_OP_LORA_BWD: return 2 * mr + round_up(m > 0 ? dy_pass_workspace_bytes(m, n, r) : 0);
    default: return SIZE_MAX;
  }
}

int qlora_quantize_nf4_dq(const float *W, int64_t n, int64_t k, uint8_t *codes, uint8_t *absmax_q,
                          float *group_scale, float *absmax_fp32, qlora_stream_t stream) {
  return qlora_quantize_4bit_dq(W, n, k, QLORA_CODEBOOK_NF4, codes, absmax_q, group_scale, absmax_fp32, stream);
}

int qlora_quantize_4bit_dq(const float *W, int64_t n, int64_t k, int32_t codebook, uint8_t *codes,
                           uint8_t *absmax_q, float *group_scale, float *absmax_fp32, qlora_stream_t stream) {
  return qlora_quantize_4bit_dq_format(W, n, k, codebook, QLORA_DQ_LINEAR8, codes, absmax_q, group_scale,
                                       absmax_fp32, stream);
}

int qlora_quantize_4bit_dq_format(const float *W, int64_t n, int64_t k, int32_t codebook, int32_t dq_format,
                                  uint8_t *codes, uint8_t *absmax_q, float *group_scale, float *absmax_fp32,
                                  qlora_stream_t stream) {
  if (!W || !codes || !absmax_q || !group_scale) return QLORA_ERR_NULL;
  if (codebook < 0 || codebook >= kCodebookCount) return QLORA_ERR_CODEBOOK;
  if (dq_format < 0 || dq_format >= kDqFormatCount) return QLORA_ERR_FORMAT;
  if (n <= 0 || k <= 0 || (k % 64) != 0) return QLORA_ERR_SHAPE;
  if (n > (int64_t(1) << 40) / k) return QLORA_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(absmax_q) || !aligned16(group_scale) ||
      (absmax_fp32 && !aligned16(absmax_fp32)))
    return QLORA_ERR_ALIGN;
  int st = check_device();
  if (st != QLORA_OK) return st;
  return cuda_status(launch_quantize(W, n * k, codes, absmax_q, group_scale, absmax_fp32, codebook_tables(codebook),
                                     codebook_buckets(codebook), dq_format, reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_merge_adapter(const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                        uint16_t *W_bf16, float *W_f32, qlora_stream_t stream) {
  int st = check_weight(w, false);
  if (st != QLORA_OK) return st;
  if (!W_bf16 && !W_f32) return QLORA_ERR_NULL;
  if ((W_bf16 && !aligned16(W_bf16)) || (W_f32 && !aligned16(W_f32))) return QLORA_ERR_ALIGN;
  bool lora = false;
  st = check_adapter(A, B, r, &lora);
  if (st != QLORA_OK) return st;
  st = check_device();
  if (st != QLORA_OK) return st;
  return cuda_status(launch_merge(view(w), lora ? A : nullptr, lora ? B : nullptr, lora ? r : 0, scale, W_bf16,
                                  W_f32, reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_dequant(const qlora_nf4_weight *w, uint16_t *W_bf16, qlora_stream_t stream) {
  int st = check_weight(w, false);
  if (st != QLORA_OK) return st;
  if (!W_bf16) return QLORA_ERR_NULL;
  if (!aligned16(W_bf16)) return QLORA_ERR_ALIGN;
  st = check_device();
  if (st != QLORA_OK) return st;
  return cuda_status(launch_dequant(w->codes, w->absmax_q, w->group_scale, w->n * w->k, W_bf16,
                                    codebook_tables(w->codebook), w->dq_format,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_linear_fwd(const uint16_t *X, int64_t m, const qlora_nf4_weight *w, const uint16_t *A,
                     const uint16_t *B, int32_t r, float scale, uint16_t *Y, void *ws, size_t ws_bytes,
                     qlora_stream_t stream) {
  bool lora = false;
  int st = validate_fwd(X, m, w, A, B, r, Y, &lora);
  if (st != QLORA_OK || m == 0) return st;
  const size_t need = lora ? qlora_workspace_bytes(QLORA_OP_FWD, m, w->n, w->k, r) : 0;
  if (need > 0 && (ws == nullptr || ws_bytes < need)) return QLORA_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return QLORA_ERR_ALIGN;
  st = check_device();
  if (st != QLORA_OK) return st;
  return launch_fwd(X, X, m, w, A, B, r, scale, Y, lora ? static_cast<uint16_t *>(ws) : nullptr,
                    reinterpret_cast<cudaStream_t>(stream));
}

int qlora_linear_bwd_dx(const uint16_t *dY, int64_t m, const qlora_nf4_weight *w, const uint16_t *A,
                        const uint16_t *B, int32_t r, float scale, uint16_t *dX, void *ws, size_t ws_bytes,
                        qlora_stream_t stream) {
  int st = check_weight(w);
  if (st != QLORA_OK) return st;
  bool lora = false;
  st = check_adapter(A, B, r, &lora);
  if (st != QLORA_OK) return st;
  if (m < 0 || m > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (m == 0) return QLORA_OK;
  if (!dY || !dX) return QLORA_ERR_NULL;
  if (!aligned16(dY) || !aligned16(dX)) return QLORA_ERR_ALIGN;
  const size_t need = lora ? qlora_workspace_bytes(QLORA_OP_BWD_DX, m, w->n, w->k, r) : 0;
  if (need > 0 && (ws == nullptr || ws_bytes < need)) return QLORA_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return QLORA_ERR_ALIGN;
  st = check_device();
  if (st != QLORA_OK) return st;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint16_t *U = lora ? static_cast<uint16_t *>(ws) : nullptr;
  cudaError_t e = cudaSuccess;
  const bool pdl = lora && t_prof_start == nullptr;
  if (lora) e = tc_proj_mnmajor(dY, m, w->n, B, r, scale, U, s);
  if (e == cudaSuccess) e = prof_mark(t_prof_start, s);
  if (e == cudaSuccess) e = tc_bwd_dx(dY, m, view(w), U, lora ? A : nullptr, lora ? r : 0, dX, s, pdl);
  if (e == cudaSuccess) e = prof_mark(t_prof_stop, s);
  return cuda_status(e);
}

int qlora_lora_bwd(const uint16_t *X, const uint16_t *dY, int64_t m, int64_t n, int64_t k, const uint16_t *A,
                   const uint16_t *B, int32_t r, float scale, uint16_t *dA, uint16_t *dB, void *ws,
                   size_t ws_bytes, qlora_stream_t stream) {
  if (!A || !B || !dA || !dB) return QLORA_ERR_NULL;
  if (n <= 0 || k <= 0 || (k % 64) != 0 || (n % 8) != 0) return QLORA_ERR_SHAPE;
  if (r <= 0 || r > 256 || (r % 16) != 0) return QLORA_ERR_SHAPE;
  if (m < 0 || m > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (!aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB)) return QLORA_ERR_ALIGN;
  if (m > 0) {
    if (!X || !dY) return QLORA_ERR_NULL;
    if (!aligned16(X) || !aligned16(dY)) return QLORA_ERR_ALIGN;
    const size_t need = qlora_workspace_bytes(QLORA_OP_LORA_BWD, m, n, k, r);
    if (ws == nullptr || ws_bytes < need) return QLORA_ERR_WORKSPACE;
    if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  }
  int st = check_device();
  if (st != QLORA_OK) return st;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (m == 0) {
    cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * static_cast<size_t>(k) * 2u, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(n) * static_cast<size_t>(r) * 2u, s);
    return cuda_status(e);
  }
  const size_t mr = round_up(static_cast<size_t>(m) * static_cast<size_t>(r) * 2u);
  uint16_t *T = static_cast<uint16_t *>(ws);
  uint16_t *U = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(ws) + mr);
  void *scratch = static_cast<uint8_t *>(ws) + 2 * mr;
  const bool one_pass = plan_dy_pass(m, n, r).ok;                         // U and dB in one pass over dY
  cudaError_t e = tc_proj_kmajor(X, m, k, A, r, scale, T, s);             // T = bf16(s X A^T)
  if (e == cudaSuccess)
    e = one_pass ? launch_dy_pass(dY, m, n, B, T, r, scale, U, dB, scratch, ws_bytes - 2 * mr, s, true)
                 : tc_proj_mnmajor(dY, m, n, B, r, scale, U, s);          // U = bf16(s dY B)
  if (e == cudaSuccess) e = tc_tn_skinny(X, m, k, U, r, dA, true, s);      // dA = U^T X
  if (e == cudaSuccess && !one_pass) e = tc_tn_skinny(dY, m, n, T, r, dB, false, s);   // dB = dY^T T
  return cuda_status(e);
}

int qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const uint16_t *T, int64_t m, const qlora_nf4_weight *w,
                     const uint16_t *A, const uint16_t *B, int32_t r, float scale, uint16_t *dX, uint16_t *dA,
                     uint16_t *dB, void *ws, size_t ws_bytes, qlora_stream_t stream) {
  int st = check_weight(w);
  if (st != QLORA_OK) return st;
  if (!A || !B || !dA || !dB) return QLORA_ERR_NULL;
  if (r <= 0 || r > 256 || (r % 16) != 0) return QLORA_ERR_SHAPE;
  if (m < 0 || m > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (!aligned16(A) || !aligned16(B) || !aligned16(dA) || !aligned16(dB)) return QLORA_ERR_ALIGN;
  if ((dX && !aligned16(dX)) || (T && !aligned16(T))) return QLORA_ERR_ALIGN;
  if (m > 0) {
    if (!X || !dY) return QLORA_ERR_NULL;
    if (!aligned16(X) || !aligned16(dY)) return QLORA_ERR_ALIGN;
    const size_t need = qlora_workspace_bytes(QLORA_OP_LORA_BWD, m, w->n, w->k, r);
    if (ws == nullptr || ws_bytes < need) return QLORA_ERR_WORKSPACE;
    if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  }
  st = check_device();
  if (st != QLORA_OK) return st;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = w->n, k = w->k;
  if (m == 0) {
    cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * static_cast<size_t>(k) * 2u, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(n) * static_cast<size_t>(r) * 2u, s);
    return cuda_status(e);
  }
  const size_t mr = round_up(static_cast<size_t>(m) * static_cast<size_t>(r) * 2u);
  uint16_t *U = static_cast<uint16_t *>(ws);
  uint16_t *Tw = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(ws) + mr);
  void *scratch = static_cast<uint8_t *>(ws) + 2 * mr;
  const size_t scratch_bytes = ws_bytes - 2 * mr;
  // U once, for the input gradient and for dA; T from the forward when given.
  // With r <= 64, U and dB come from one pass over dY.
  const bool one_pass = plan_dy_pass(m, n, r).ok;
  cudaError_t e = cudaSuccess;
  if (T == nullptr) e = tc_proj_kmajor(X, m, k, A, r, scale, Tw, s);                   // T = bf16(s X A^T)
  if (e == cudaSuccess)
    e = one_pass ? launch_dy_pass(dY, m, n, B, T ? T : Tw, r, scale, U, dB, scratch, scratch_bytes, s,
                                  t_prof_start == nullptr)                             // U and dB = dY^T T
                 : tc_proj_mnmajor(dY, m, n, B, r, scale, U, s);                       // U = bf16(s dY B)
  // The input-gradient kernel needs U only for its adapter k-steps: it is
  // launched as a programmatic dependent of the kernel that writes U, which
  // directly precedes it (unless the caller times the main kernel alone).
  const bool pdl = t_prof_start == nullptr;
  if (e == cudaSuccess) e = prof_mark(t_prof_start, s);
  if (e == cudaSuccess && dX) e = tc_bwd_dx(dY, m, view(w), U, A, r, dX, s, pdl);      // dX = dY W^ + U A
  if (e == cudaSuccess) e = prof_mark(t_prof_stop, s);
  if (e == cudaSuccess) e = tc_tn_skinny(X, m, k, U, r, dA, true, s);                  // dA = U^T X
  if (e == cudaSuccess && !one_pass) e = tc_tn_skinny(dY, m, n, T ? T : Tw, r, dB, false, s);   // dB = dY^T T
  return cuda_status(e);
}

int qlora_lora_dropout(const uint16_t *X, int64_t m, int64_t k, float p, uint64_t seed, uint64_t offset,
                       uint16_t *Xd, qlora_stream_t stream) {
  DropoutParams d{};
  if (!dropout_params(p, seed, offset, &d)) return QLORA_ERR_SHAPE;
  if (m < 0 || k <= 0 || (k % 64) != 0 || m > (int64_t(1) << 31) || k > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (m == 0) return QLORA_OK;
  if (!X || !Xd) return QLORA_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xd)) return QLORA_ERR_ALIGN;
  int st = check_device();
  if (st != QLORA_OK) return st;
  return cuda_status(launch_dropout_apply(X, m * k, d, Xd, reinterpret_cast<cudaStream_t>(stream)));
}

int qlora_linear_fwd_dropout(const uint16_t *X, int64_t m, const qlora_nf4_weight *w, const uint16_t *A,
                             const uint16_t *B, int32_t r, float scale, float p, uint64_t seed, uint64_t offset,
                             uint16_t *Xd, uint16_t *Y, void *ws, size_t ws_bytes, qlora_stream_t stream) {
  bool lora = false;
  int st = validate_fwd(X, m, w, A, B, r, Y, &lora);
  if (st != QLORA_OK) return st;
  if (!lora) return A == nullptr || B == nullptr ? QLORA_ERR_NULL : QLORA_ERR_SHAPE;
  DropoutParams d{};
  if (!dropout_params(p, seed, offset, &d)) return QLORA_ERR_SHAPE;
  if (m == 0) return QLORA_OK;
  if (!Xd) return QLORA_ERR_NULL;
  if (!aligned16(Xd)) return QLORA_ERR_ALIGN;
  const size_t need = qlora_workspace_bytes(QLORA_OP_FWD, m, w->n, w->k, r);
  if (ws == nullptr || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  st = check_device();
  if (st != QLORA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = cuda_status(launch_dropout_apply(X, m * w->k, d, Xd, s));
  if (st != QLORA_OK) return st;
  return launch_fwd(X, Xd, m, w, A, B, r, scale, Y, static_cast<uint16_t *>(ws), s);
}

int qlora_linear_bwd_dx_dropout(const uint16_t *dY, int64_t m, const qlora_nf4_weight *w, const uint16_t *A,
                                const uint16_t *B, int32_t r, float scale, float p, uint64_t seed, uint64_t offset,
                                uint16_t *dX, void *ws, size_t ws_bytes, qlora_stream_t stream) {
  int st = check_weight(w);
  if (st != QLORA_OK) return st;
  bool lora = false;
  st = check_adapter(A, B, r, &lora);
  if (st != QLORA_OK) return st;
  if (!lora) return A == nullptr || B == nullptr ? QLORA_ERR_NULL : QLORA_ERR_SHAPE;
  DropoutParams d{};
  if (!dropout_params(p, seed, offset, &d)) return QLORA_ERR_SHAPE;
  if (m < 0 || m > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (m == 0) return QLORA_OK;
  if (!dY || !dX) return QLORA_ERR_NULL;
  if (!aligned16(dY) || !aligned16(dX)) return QLORA_ERR_ALIGN;
  const size_t need = qlora_workspace_bytes(QLORA_OP_BWD_DX, m, w->n, w->k, r);
  if (ws == nullptr || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  st = check_device();
  if (st != QLORA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint16_t *U = static_cast<uint16_t *>(ws);
  // dX = bf16(dY . W^) first, then the masked adapter term is added to it.
  cudaError_t e = tc_proj_mnmajor(dY, m, w->n, B, r, scale, U, s);       // U = bf16(s dY B)
  if (e == cudaSuccess) e = tc_bwd_dx(dY, m, view(w), nullptr, nullptr, 0, dX, s, false);
  if (e == cudaSuccess) e = tc_dropout_add(U, m, r, A, w->k, d, dX, s);
  return cuda_status(e);
}

int qlora_poll_device_error(qlora_stream_t stream, unsigned *flags) {
  if (!flags) return QLORA_ERR_NULL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  unsigned *word = device_error_word();
  if (!word) return cuda_status(cudaErrorInvalidSymbol);
  e = cudaMemcpy(flags, word, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e);
  const unsigned zero = 0u;
  e = cudaMemcpy(word, &zero, sizeof(unsigned), cudaMemcpyHostToDevice);
  return cuda_status(e);
}

}  // extern "C"
