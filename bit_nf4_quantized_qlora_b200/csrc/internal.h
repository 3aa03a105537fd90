// Host-side declarations shared by the translation units of libqlora.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/qlora.h"
#include "types.h"

namespace qlora {

// Per-device tables of the library (attribute flags, cached addresses).
constexpr int kMaxDevicesPerProcess = 64;

// The library's codebooks and their midpoints (derived once at load time):
// codebook_tables(kCodebookNF4 | kCodebookFP4 | kCodebookINT4).
const Nf4Tables &codebook_tables(int codebook);
const QuantBuckets &codebook_buckets(int codebook);
const Nf4Tables &nf4_tables();

// Device error word (bounded waits that gave up); one per device.
unsigned *device_error_word();

// Process-wide count of kernel launches (see qlora_launch_count).
void count_launches(int n);

// QLORA_OK for cudaSuccess; otherwise records the error for
// qlora_last_cuda_error() and returns QLORA_ERR_CUDA.
int status_from_cuda(cudaError_t e);

// QLORA_OK when the current device is an sm_100 part (binding the device's
// primary context to this thread on its first call); QLORA_ERR_DEVICE or
// QLORA_ERR_CUDA otherwise.
int check_device();

// Raises a kernel's dynamic shared-memory limit once per device (`done`
// holds one flag per device; the attribute call is idempotent, so two threads
// that race on a fresh device both set the same value).
cudaError_t set_smem_once(const void *kernel, int smem_bytes, std::atomic<bool> *done);

// Host-side checks of a forward call (weight, adapter, m, X, Y), in the order
// every forward entry point reports them; *use_adapter tells whether the call
// has an adapter.  No CUDA call is made.
int validate_fwd(const uint16_t *X, int64_t m, const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B,
                 int32_t r, uint16_t *Y, bool *use_adapter);

// Launches a validated forward (m > 0) with T as the rank-r scratch (null:
// no adapter); Xa is the adapter's input (X itself, or its dropout); returns
// a qlora status.
int launch_fwd(const uint16_t *X, const uint16_t *Xa, int64_t m, const qlora_nf4_weight *w, const uint16_t *A,
               const uint16_t *B, int32_t r, float scale, uint16_t *Y, uint16_t *T, cudaStream_t s);

// LoRA dropout on the adapter input: keep an element when its 16-bit draw is
// >= threshold = round(fp32(p) . 65536); a kept element is scaled by
// keep_scale = fp32(1 / fp32(1 - p)).  The draws come from the counter-based
// generator of philox.cuh keyed by (seed, offset).
struct DropoutParams {
  uint64_t seed, offset;
  uint32_t threshold;
  float keep_scale;
};

// Xd = bf16(D . X . keep_scale), +0 where dropped; numel % 16 == 0.
cudaError_t launch_dropout_apply(const uint16_t *X, int64_t numel, const DropoutParams &d, uint16_t *Xd,
                                 cudaStream_t stream);

// TMA tensor maps (2D, row-major).  bf16: 128-byte swizzle.  codes: uint8
// rows of packed codes, optional 128-byte swizzle.  False if encoding failed.
bool encode_bf16_map(CUtensorMap *m, const uint16_t *ptr, int64_t rows, int64_t cols, uint32_t box_cols,
                     uint32_t box_rows);
// 3D map over `slabs` row-major fp32 [rows x cols] matrices; 128-byte
// swizzled boxes of {box_cols (<= 32), box_rows, 1}.  Stores clip at the
// slab's rows and columns.
bool encode_f32_slab_map(CUtensorMap *m, const float *ptr, int64_t slabs, int64_t rows, int64_t cols,
                         uint32_t box_cols, uint32_t box_rows);
// fp32 row-major [rows x cols], box {box_cols, box_rows}, 128-byte swizzle
// (box_cols * 4 <= 128).
bool encode_f32_map(CUtensorMap *m, const float *ptr, int64_t rows, int64_t cols, uint32_t box_cols,
                    uint32_t box_rows);
bool encode_codes_map(CUtensorMap *m, const uint8_t *ptr, int64_t rows, int64_t row_bytes, uint32_t box_bytes,
                      uint32_t box_rows, bool swizzle128);

// The tensor mean of the absmax for the E4M3 + mean format (the entry after
// the ceil(nb / 256) group scales), null for linear 8-bit.
inline const float *mean_ptr(const float *group_scale, int64_t nblocks, int dq_format) {
  return dq_format == kDqFp8Mean ? group_scale + (nblocks + 255) / 256 : nullptr;
}

// --- launchers (all asynchronous on `stream`; return cudaError_t) --------

// dq_format is a kDq* value (types.h); for kDqFp8Mean group_scale holds
// ceil(numel / 16384) + 1 entries, the last the tensor mean of the absmax.
cudaError_t launch_quantize(const float *W, int64_t numel, uint8_t *codes, uint8_t *absmax_q,
                            float *group_scale, float *absmax_fp32, const Nf4Tables &tab, const QuantBuckets &bk,
                            int dq_format, cudaStream_t stream);

cudaError_t launch_dequant(const uint8_t *codes, const uint8_t *absmax_q, const float *group_scale,
                           int64_t numel, uint16_t *out, const Nf4Tables &tab, int dq_format,
                           cudaStream_t stream);

// T[m x r] = bf16(scale * X[m x k] . A[r x k]^T) for small m (m <= 16).
cudaError_t launch_lora_proj_small(const uint16_t *X, int64_t m, int64_t k, const uint16_t *A,
                                   int32_t r, float scale, uint16_t *T, cudaStream_t stream);

// Y[m x n] = bf16(X . W^T + T . B^T) for m <= 16 (CTA-ring weight-streaming
// kernel); with pdl it overlaps the preceding T projection.
cudaError_t launch_gemv_fwd(const uint16_t *X, int64_t m, const uint8_t *codes,
                            const uint8_t *absmax_q, const float *group_scale, const float *mu, int64_t n,
                            int64_t k, const uint16_t *T, const uint16_t *B, int32_t r, uint16_t *Y,
                            const Nf4Tables &tab, cudaStream_t stream, bool pdl);

// Decode-sized forward (m <= 4, k/64 <= 512): per-warp TMA streams of the
// codes, K split over a cluster.  Same contract as launch_gemv_fwd.
bool gemv_stream_supported(int64_t m, int64_t n, int64_t k);
cudaError_t launch_gemv_stream(const uint16_t *X, int64_t m, const uint8_t *codes,
                               const uint8_t *absmax_q, const float *group_scale, const float *mu,
                               int64_t n, int64_t k, const uint16_t *T, const uint16_t *B, int32_t r, uint16_t *Y,
                               const Nf4Tables &tab, cudaStream_t stream, bool pdl);

// tcgen05 paths -------------------------------------------------------------

struct WeightView {
  const uint8_t *codes;
  const uint8_t *absmax_q;
  const float *group_scale;
  int64_t n, k;
  const Nf4Tables *tab;   // the weight's codebook
  const float *mu;        // E4M3 + mean format: the tensor mean; null for linear 8-bit
};

// Y = bf16(X . W^T + T . B^T); T may be null (no adapter).
// With pdl, the kernel is launched as a programmatic dependent of the
// preceding kernel (the adapter projection) and waits for it only before its
// adapter k-steps.
cudaError_t tc_fwd(const uint16_t *X, int64_t m, const WeightView &w, const uint16_t *T,
                   const uint16_t *B, int32_t r, uint16_t *Y, cudaStream_t stream, bool pdl);

// The same for m > 128: 512 x 256 tiles on CTA pairs (fused_pair.cu).
cudaError_t fused_fwd_large(const uint16_t *X, int64_t m, const WeightView &w, const uint16_t *T,
                            const uint16_t *B, int32_t r, uint16_t *Y, cudaStream_t stream, bool pdl);

// The same for m > 128 on CTA pairs (fused_pair.cu).
cudaError_t fused_bwd_dx_large(const uint16_t *dY, int64_t m, const WeightView &w, const uint16_t *U,
                               const uint16_t *A, int32_t r, uint16_t *dX, cudaStream_t stream, bool pdl);

// dX = bf16(dY . W^ + U . A); U may be null.
cudaError_t tc_bwd_dx(const uint16_t *dY, int64_t m, const WeightView &w, const uint16_t *U,
                      const uint16_t *A, int32_t r, uint16_t *dX, cudaStream_t stream, bool pdl);

// dX = bf16(dX + D . (U . A) . keep_scale) for U [m x r], A [r x k], k % 64 == 0.
cudaError_t tc_dropout_add(const uint16_t *U, int64_t m, int32_t r, const uint16_t *A, int64_t k,
                           const DropoutParams &d, uint16_t *dX, cudaStream_t stream);

// One pass over dY for U = bf16(s dY B) [m x r] and dB = bf16(dY^T T) [n x r]
// (r <= 64, r % 16 == 0), with fp32 partials in a scratch of
// dy_pass_workspace_bytes (dy_pass.cu); the split depends on the shape only.
struct DyPassPlan {
  bool ok;
  int nslices;           // m-slices (grid x)
  int nranges;           // n-ranges (grid y)
  uint32_t tmem_cols;
  size_t upart_bytes, dpart_bytes;
};
DyPassPlan plan_dy_pass(int64_t m, int64_t n, int32_t r);
size_t dy_pass_workspace_bytes(int64_t m, int64_t n, int32_t r);
cudaError_t launch_dy_pass(const uint16_t *dY, int64_t m, int64_t n, const uint16_t *B, const uint16_t *T, int32_t r,
                           float scale, uint16_t *U, uint16_t *dB, void *scratch, size_t scratch_bytes,
                           cudaStream_t stream, bool pdl_reduce);

// Adapter merge W' = W^ + scale * B . A (B [n x r], A [r x k], r % 16 == 0,
// r <= 256; r == 0 gives W^), written as bf16 and/or fp32 [n x k].
cudaError_t launch_merge(const WeightView &w, const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                         uint16_t *out_bf16, float *out_f32, cudaStream_t stream);

// out[m x r] = bf16(scale * L[m x kc] . R^T) with R given as [r x kc] (k-major).
cudaError_t tc_proj_kmajor(const uint16_t *L, int64_t m, int64_t kc, const uint16_t *R, int32_t r,
                           float scale, uint16_t *out, cudaStream_t stream);

// out[m x r] = bf16(scale * L[m x kc] . R) with R given as [kc x r] (r contiguous).
cudaError_t tc_proj_mnmajor(const uint16_t *L, int64_t m, int64_t kc, const uint16_t *R, int32_t r,
                            float scale, uint16_t *out, cudaStream_t stream);

// out = bf16(Lt^T . R): Lt [mc x p] (p contiguous), R [mc x r] (r contiguous),
// contraction over mc; result [p x r] stored row-major (transposed == false)
// or as [r x p] (transposed == true).
cudaError_t tc_tn_skinny(const uint16_t *Lt, int64_t mc, int64_t p, const uint16_t *R, int32_t r,
                         uint16_t *out, bool transposed, cudaStream_t stream);

}  // namespace qlora
