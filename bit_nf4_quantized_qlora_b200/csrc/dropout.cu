// LoRA dropout on the adapter input: Xd = bf16(D . X . fp32(1 / fp32(1 - p))).
//
// "QLoRA and Quantized Training", In code: the adapters are trained with
// LoraConfig(..., lora_dropout=0.05).  The pages say nothing more; the reading
// taken is inverted dropout on the adapter's input only, as in the LoRA
// configuration they use: the frozen product keeps X, the adapter multiplies
// Xd, and a dropped element is +0.  The keep mask D comes from a counter-based
// generator (philox.cuh), so the backward pass regenerates it from the same
// (seed, offset) instead of storing it.
//
// One thread per block of 16 elements (one generator call): 32 bytes of X in,
// 32 bytes of Xd out, consecutive threads on consecutive blocks.  Bound by HBM.
#include "common.cuh"
#include "internal.h"
#include "philox.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) dropout_apply_kernel(const uint16_t *__restrict__ X, int64_t nblocks,
                                                                 uint64_t seed, uint64_t offset, uint32_t threshold,
                                                                 float keep_scale, uint16_t *__restrict__ Xd) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; b < nblocks; b += stride) {
    const uint4 *src = reinterpret_cast<const uint4 *>(X) + 2 * b;
    const uint4 v[2] = {__ldg(src), __ldg(src + 1)};
    const uint32_t keep = dropout_keep_bits(static_cast<uint64_t>(b), seed, offset, threshold);
    uint4 o[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t in[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
      uint32_t out[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = 8 * h + 2 * j;
        const float lo = __fmul_rn(bf16lo_to_f32(in[j]), keep_scale);
        const float hi = __fmul_rn(bf16hi_to_f32(in[j]), keep_scale);
        const uint32_t packed = pack_bf16x2(lo, hi);
        const uint32_t mask = ((keep >> e) & 1u ? 0x0000FFFFu : 0u) | ((keep >> (e + 1)) & 1u ? 0xFFFF0000u : 0u);
        out[j] = packed & mask;
      }
      o[h] = make_uint4(out[0], out[1], out[2], out[3]);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(Xd) + 2 * b;
    dst[0] = o[0];
    dst[1] = o[1];
  }
}

}  // namespace

cudaError_t launch_dropout_apply(const uint16_t *X, int64_t numel, const DropoutParams &d, uint16_t *Xd,
                                 cudaStream_t stream) {
  const int64_t nblocks = numel / 16;
  if (nblocks == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (nblocks + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  dropout_apply_kernel<<<grid, kThreads, 0, stream>>>(X, nblocks, d.seed, d.offset, d.threshold, d.keep_scale, Xd);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
