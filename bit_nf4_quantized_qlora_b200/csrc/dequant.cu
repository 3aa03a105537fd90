// Standalone NF4 dequantization to bf16 (HBM-bound).
//
// "QLoRA", Storage precision is not calculation precision: the 4-bit stored
// weight is dequantized to a higher-precision compute type; "A 65B fine-tune
// on the GPU you already have", figure 2: block by block to bf16.
//
// Each thread expands half a block (32 weights): one 16-byte load of packed
// codes, the absmax code and group constant of its block, a per-block bf16
// table (see common.cuh) and four 16-byte stores.  A grid-stride loop over
// half-blocks keeps every SM busy for any size.
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint8_t *__restrict__ codes,
                                                           const uint8_t *__restrict__ absmax_q,
                                                           const float *__restrict__ group_scale,
                                                           int64_t n_half_blocks,
                                                           uint16_t *__restrict__ out,
                                                           const Nf4Tables tab, const float *mu_ptr) {
  const bool fp8 = mu_ptr != nullptr;
  const float mu = load_mu(mu_ptr);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t h = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; h < n_half_blocks;
       h += stride) {
    const int64_t blk = h >> 1;
    const uint4 cw = __ldcs(reinterpret_cast<const uint4 *>(codes) + h);
    const uint32_t q = absmax_q[blk];
    const float S = __ldg(group_scale + (blk >> 8));
    Bf16Table t;
    make_table(tab, block_constant(q, group_constant(S, fp8), fp8, mu), t);
    uint32_t o[16];
    decode8(cw.x, t, o + 0);
    decode8(cw.y, t, o + 4);
    decode8(cw.z, t, o + 8);
    decode8(cw.w, t, o + 12);
    uint4 *dst = reinterpret_cast<uint4 *>(out + h * 32);
    __stcs(dst + 0, make_uint4(o[0], o[1], o[2], o[3]));
    __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
    __stcs(dst + 2, make_uint4(o[8], o[9], o[10], o[11]));
    __stcs(dst + 3, make_uint4(o[12], o[13], o[14], o[15]));
  }
}

}  // namespace

cudaError_t launch_dequant(const uint8_t *codes, const uint8_t *absmax_q, const float *group_scale,
                           int64_t numel, uint16_t *out, const Nf4Tables &tab, int dq_format,
                           cudaStream_t stream) {
  const int64_t nh = numel / 32;
  if (nh == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (nh + kThreads - 1) / kThreads;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  dequant_kernel<<<grid, kThreads, 0, stream>>>(codes, absmax_q, group_scale, nh, out, tab,
                                                mean_ptr(group_scale, numel / 64, dq_format));
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
