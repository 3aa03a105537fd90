// Blockwise NF4 quantization with double-quantized absmax (HBM-bound).
//
// "QLoRA and Quantized Training", The idea / Worked example: weights are
// stored in blocks of 64, one fp32 scale per block, 0.5 byte per weight.
// "A 65B fine-tune on the GPU you already have", figure 4: the per-block
// constants are themselves quantized to 8 bits in blocks of 256.
//
// One CTA of 256 threads per group of 256 blocks (16384 weights, 64 KB of
// fp32).  Each warp owns 32 blocks and reads them as 16 coalesced 512-byte
// rows (two blocks per row, 16 lanes per block, one float4 per lane); the
// block absmax is a 16-lane shuffle reduction, the codes are counted against
// the 15 fp32 midpoints after an IEEE division by the absmax, and each lane
// stores its 4 codes as one 16-bit word.  The group maximum is then reduced
// through shared memory and every thread emits one absmax code.
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;
constexpr int kBlocksPerGroup = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint32_t nf4_code(float x, const Nf4Tables &tab) {
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) c += (x > tab.mid[i]) ? 1u : 0u;
  return c;
}

__global__ void __launch_bounds__(kThreads) quantize_kernel(const float *__restrict__ W, int64_t nb,
                                                            uint8_t *__restrict__ codes,
                                                            uint8_t *__restrict__ absmax_q,
                                                            float *__restrict__ group_scale,
                                                            float *__restrict__ absmax_out,
                                                            const Nf4Tables tab) {
  __shared__ float s_c[kBlocksPerGroup];
  __shared__ float s_red[kThreads / 32];

  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kBlocksPerGroup;
  const int nblk = static_cast<int>(nb - b0 < kBlocksPerGroup ? nb - b0 : kBlocksPerGroup);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;   // which of the two blocks of a 512-byte row
  const int sub = lane & 15;    // float4 index inside the block

  // Warp w owns blocks [32w, 32w + 32) of the group: 16 rows of 2 blocks.
#pragma unroll 1
  for (int j0 = 0; j0 < 16; j0 += kUnroll) {
    float4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int blk = warp * 32 + 2 * (j0 + u) + half;
      if (blk < nblk) {
        v[u] = __ldcs(reinterpret_cast<const float4 *>(W + (b0 + blk) * 64) + sub);
      } else {
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int blk = warp * 32 + 2 * (j0 + u) + half;
      float m = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (blk < nblk) {
        uint32_t c0 = 7, c1 = 7, c2 = 7, c3 = 7;
        if (m > 0.0f) {
          c0 = nf4_code(__fdiv_rn(v[u].x, m), tab);
          c1 = nf4_code(__fdiv_rn(v[u].y, m), tab);
          c2 = nf4_code(__fdiv_rn(v[u].z, m), tab);
          c3 = nf4_code(__fdiv_rn(v[u].w, m), tab);
        }
        const uint32_t packed = ((c0 << 4) | c1) | (((c2 << 4) | c3) << 8);
        reinterpret_cast<uint16_t *>(codes + (b0 + blk) * 32)[sub] = static_cast<uint16_t>(packed);
        if (sub == 0) {
          s_c[blk] = m;
          if (absmax_out) absmax_out[b0 + blk] = m;
        }
      }
    }
  }
  __syncthreads();

  // Double quantization of this group's absmax values.
  const int t = threadIdx.x;
  const float c = (t < nblk) ? s_c[t] : 0.0f;
  float gm = c;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
  if (lane == 0) s_red[warp] = gm;
  __syncthreads();
  float S = s_red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) S = fmaxf(S, s_red[i]);
  if (t < nblk) {
    uint32_t q = 0;
    if (S > 0.0f) q = static_cast<uint32_t>(rintf(__fmul_rn(__fdiv_rn(c, S), 255.0f)));
    absmax_q[b0 + t] = static_cast<uint8_t>(q);
  }
  if (t == 0) group_scale[g] = S;
}

}  // namespace

cudaError_t launch_quantize(const float *W, int64_t numel, uint8_t *codes, uint8_t *absmax_q,
                            float *group_scale, float *absmax_fp32, cudaStream_t stream) {
  const int64_t nb = numel / 64;
  const int64_t ng = (nb + kBlocksPerGroup - 1) / kBlocksPerGroup;
  if (ng == 0) return cudaSuccess;
  quantize_kernel<<<static_cast<unsigned>(ng), kThreads, 0, stream>>>(W, nb, codes, absmax_q, group_scale,
                                                                      absmax_fp32, nf4_tables());
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
