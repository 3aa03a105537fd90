// Blockwise NF4 quantization with double-quantized absmax (HBM-bound).
//
// "QLoRA and Quantized Training", The idea / Worked example: weights are
// stored in blocks of 64, one fp32 scale per block, 0.5 byte per weight.
// "A 65B fine-tune on the GPU you already have", figure 4: the per-block
// constants are themselves quantized to 8 bits in blocks of 256.
//
// One CTA of 256 threads per group of 256 blocks (16384 weights, 64 KB of
// fp32).  Each warp owns 32 blocks; four lanes share a block and each holds 16
// of its weights, so a lane has 16 independent division + search chains in
// flight.  The block absmax is a 4-lane shuffle reduction; each weight is
// divided by it (correctly rounded, see div_by_absmax) and located among the
// 15 fp32 midpoints by a branchless binary search; codes are stored as 16-bit
// words (4 weights).  The group maximum is then reduced
// through shared memory and every thread emits one absmax code.
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;
constexpr int kBlocksPerGroup = 256;
// Absmax values below this take the IEEE division path.  The reciprocal
// step below needs the residual w - m * q0 to be exact: its lowest bit,
// 2^(e_m + e_q0 - 46), must not fall under the smallest subnormal 2^-149.
// A code can only change where x = w / m is near a midpoint, |x| >= 1/24
// (FP4's smallest nonzero one; NF4's and INT4's are larger), so e_q0 >= -5
// there and m >= 2^-98 suffices; the guard keeps a margin.  (Quotients under
// the normal range, where only x = 0 against x > 0 matters, are redone
// separately in div_by_absmax.)
constexpr float kMinFastAbsmax = 0x1p-90f;

template <bool TINY>
__device__ __forceinline__ float div_by_absmax(float w, float m, float y) {
  const float q0 = __fmul_rn(w, y);
  const float rho = __fmaf_rn(-q0, m, w);
  float x = __fmaf_rn(rho, y, q0);
  // Below the normal range the residual can underflow and the result may be
  // off by an ulp.  Only zero against nonzero (and the sign) can decide a
  // code there, and only in a codebook with a midpoint at 0 (TINY, FP4:
  // -0 | +0): IEEE division settles those rare quotients.
  if (TINY && fabsf(x) < 0x1p-125f) x = __fdiv_rn(w, m);
  return x;
}

// #{i : x > T_i} over the 15 sorted midpoints, as a branchless binary search:
// code >= 8 iff x > T7; then code >= base + 4 iff x > T[base + 3], and so on.
__device__ __forceinline__ uint32_t nf4_code(float x, const Nf4Tables &t) {
  const bool b3 = x > t.mid[7];
  const bool b2 = x > (b3 ? t.mid[11] : t.mid[3]);
  const float m1 = b2 ? (b3 ? t.mid[13] : t.mid[5]) : (b3 ? t.mid[9] : t.mid[1]);
  const bool b1 = x > m1;
  const float lo = b1 ? (b3 ? t.mid[10] : t.mid[2]) : (b3 ? t.mid[8] : t.mid[0]);
  const float hi = b1 ? (b3 ? t.mid[14] : t.mid[6]) : (b3 ? t.mid[12] : t.mid[4]);
  const bool b0 = x > (b2 ? hi : lo);
  return (b3 ? 8u : 0u) | (b2 ? 4u : 0u) | (b1 ? 2u : 0u) | (b0 ? 1u : 0u);
}

// The same count by bucket (QuantBuckets): one FMA, two shuffles from the
// lane-held tables (lane b holds code[b] and thr[b]) and one compare.  All
// lanes of the warp take part.
__device__ __forceinline__ uint32_t bucket_code(float x, uint32_t lane_code, float lane_thr) {
  // u = 1.5 * 2^23 + rn(15.4 x + 16): the bucket is the low five bits of u,
  // which is all a shuffle takes of its source lane.
  const int u = __float_as_int(__fmaf_rn(x, 15.4f, 12582928.0f));
  const uint32_t c = __shfl_sync(0xffffffffu, lane_code, u);
  const float t = __shfl_sync(0xffffffffu, lane_thr, u);
  return c + (x > t ? 1u : 0u);
}

// Where the fp64 sum of group g's absmax values waits for the mean kernel
// (E4M3 + mean format): in the group's own absmax-code bytes, which the final
// pass overwrites; a partial last group (which may have fewer than 8 bytes)
// uses bytes 8..15 of group 0 instead.  Only when there are at least two
// groups, so group 0 is whole.
__device__ __forceinline__ double *group_sum_slot(uint8_t *absmax_q, int64_t g, int64_t ng, bool last_partial) {
  return reinterpret_cast<double *>(absmax_q + ((last_partial && g == ng - 1) ? 8 : 256 * g));
}

// fp64 sum of s_c[0..len) by pairwise halving (adjacent pairs, an odd last
// element carried), the order the format fixes; every thread gets the sum.
__device__ double group_pairwise_sum(const float *s_c, int len, double *b0, double *b1) {
  const int t = threadIdx.x;
  b0[t] = t < len ? static_cast<double>(s_c[t]) : 0.0;
  __syncthreads();
  while (len > 1) {
    const int half = len / 2;
    if (t < half) b1[t] = b0[2 * t] + b0[2 * t + 1];
    if ((len & 1) && t == half) b1[half] = b0[len - 1];
    __syncthreads();
    double *tmp = b0;
    b0 = b1;
    b1 = tmp;
    len = (len + 1) / 2;
  }
  const double r = b0[0];
  __syncthreads();
  return r;
}

// BUCKET: codes by bucket_code (codebooks whose buckets allow it), else by
// the binary search.  TINY: the codebook has a midpoint at 0.
template <bool BUCKET, bool TINY>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const float *__restrict__ W, int64_t nb,
                                                            uint8_t *__restrict__ codes,
                                                            uint8_t *__restrict__ absmax_q,
                                                            float *__restrict__ group_scale,
                                                            float *__restrict__ absmax_out,
                                                            const Nf4Tables tab, const QuantBuckets bk,
                                                            int dq_format) {
  __shared__ float s_c[kBlocksPerGroup];
  __shared__ float s_red[kThreads / 32];
  __shared__ double s_sum[2][kBlocksPerGroup];

  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kBlocksPerGroup;
  const int nblk = static_cast<int>(nb - b0 < kBlocksPerGroup ? nb - b0 : kBlocksPerGroup);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;      // 4 lanes per block, 16 weights each
  const int bl = lane >> 2;      // 8 blocks per warp iteration
  const uint32_t lane_code = BUCKET ? bk.code[lane] : 0u;
  const float lane_thr = BUCKET ? bk.thr[lane] : 0.f;

  // Warp w owns blocks [32w, 32w + 32): 4 iterations of 8 blocks.  Lane
  // (bl, sub) holds weights 16j + 4sub .. +3 (j = 0..3) of its block, so each
  // load instruction reads 8 blocks x 64 contiguous bytes.
  float4 v[4], nv[4];
  auto load = [&](int it, float4 (&dst)[4]) {
    const int blk = warp * 32 + it * 8 + bl;
    if (blk < nblk) {
      const float4 *src = reinterpret_cast<const float4 *>(W + (b0 + blk) * 64) + sub;
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = __ldcs(src + 4 * j);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  load(0, v);
#pragma unroll 1
  for (int it = 0; it < 4; ++it) {
    if (it + 1 < 4) load(it + 1, nv);
    const int blk = warp * 32 + it * 8 + bl;
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[j].x), fabsf(v[j].y)), fmaxf(fabsf(v[j].z), fabsf(v[j].w))));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    // Quotients x = fp32(w / m) (per-lane branches, no shuffles inside).
    float x[16];
    if (m >= kMinFastAbsmax) {
      // Correctly rounded w / m without a divide per weight (Markstein's
      // theorem): with y = RN(1/m) and q0 = RN(w*y) within one ulp of w/m,
      // the residual w - m*q0 is exact in one FMA and RN(q0 + residual*y)
      // is RN(w/m).  |w/m| <= 1 cannot overflow; results below the normal
      // range are redone by IEEE division (div_by_absmax).
      const float y = __frcp_rn(m);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[4 * j + 0] = div_by_absmax<TINY>(v[j].x, m, y);
        x[4 * j + 1] = div_by_absmax<TINY>(v[j].y, m, y);
        x[4 * j + 2] = div_by_absmax<TINY>(v[j].z, m, y);
        x[4 * j + 3] = div_by_absmax<TINY>(v[j].w, m, y);
      }
    } else if (m > 0.0f) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[4 * j + 0] = __fdiv_rn(v[j].x, m);
        x[4 * j + 1] = __fdiv_rn(v[j].y, m);
        x[4 * j + 2] = __fdiv_rn(v[j].z, m);
        x[4 * j + 3] = __fdiv_rn(v[j].w, m);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = 0.f;
    }
    // Codes (the warp converged again: bucket_code shuffles).  A zero block
    // takes code 7.
    uint32_t c[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) c[e] = BUCKET ? bucket_code(x[e], lane_code, lane_thr) : nf4_code(x[e], tab);
    if (blk < nblk) {
      uint16_t *dst = reinterpret_cast<uint16_t *>(codes + (b0 + blk) * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t packed = ((c[4 * j] << 4) | c[4 * j + 1]) | (((c[4 * j + 2] << 4) | c[4 * j + 3]) << 8);
        dst[4 * j + sub] = static_cast<uint16_t>(m > 0.0f ? packed : 0x7777u);   // bytes 8j + 2sub, +1
      }
      if (sub == 0) {
        s_c[blk] = m;
        if (absmax_out) absmax_out[b0 + blk] = m;
      }
    }
    if (it + 1 < 4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = nv[j];
    }
  }
  __syncthreads();

  if (dq_format == kDqFp8Mean) {
    // E4M3 + mean: only the group's fp64 absmax sum here; the codes of the
    // absmax values follow once the tensor's mean is known.
    const double sum = group_pairwise_sum(s_c, nblk, s_sum[0], s_sum[1]);
    if (threadIdx.x == 0) {
      const int64_t ng = gridDim.x;
      if (ng == 1)
        group_scale[1] = static_cast<float>(sum / static_cast<double>(nb));   // the mean itself
      else
        *group_sum_slot(absmax_q, g, ng, (nb % kBlocksPerGroup) != 0) = sum;
    }
    return;
  }

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

// mu = fp32(T / nb), T the pairwise sum of the ng group sums: strides 1, 2,
// 4, ... in place (slot i += slot i + s for i a multiple of 2s), the same
// additions as halving adjacent pairs level by level with an odd last one
// carried.  One CTA; ng >= 2.
__global__ void __launch_bounds__(1024) dq_mean_kernel(uint8_t *absmax_q, int64_t ng, int64_t nb,
                                                       float *group_scale) {
  const bool last_partial = (nb % kBlocksPerGroup) != 0;
  for (int64_t s = 1; s < ng; s *= 2) {
    for (int64_t i = 2 * s * threadIdx.x; i + s < ng; i += 2 * s * blockDim.x)
      *group_sum_slot(absmax_q, i, ng, last_partial) += *group_sum_slot(absmax_q, i + s, ng, last_partial);
    __syncthreads();
  }
  if (threadIdx.x == 0)
    group_scale[ng] = static_cast<float>(*group_sum_slot(absmax_q, 0, ng, last_partial) / static_cast<double>(nb));
}

// E4M3 codes of the offsets from the mean, one CTA per group (the block
// absmax values are recomputed from W, as in quantize_kernel):
//   d = fp32(c - mu), S = max |d|, q = E4M3_rn(fp32(fp32(d / S) * 448)),
//   group_scale[g] = fp32(S / 448).
__global__ void __launch_bounds__(kThreads) dq_fp8_kernel(const float *__restrict__ W, int64_t nb,
                                                          uint8_t *__restrict__ absmax_q,
                                                          float *__restrict__ group_scale) {
  __shared__ float s_red[kThreads / 32];
  __shared__ float s_c[kBlocksPerGroup];
  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kBlocksPerGroup;
  const int nblk = static_cast<int>(nb - b0 < kBlocksPerGroup ? nb - b0 : kBlocksPerGroup);
  const int64_t ng = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane & 3, bl = lane >> 2;
  // Block maxima with the load pattern of quantize_kernel: 4 lanes per
  // block, each load instruction covering 8 blocks x 64 contiguous bytes.
  float4 v[4][4];
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int blk = warp * 32 + it * 8 + bl;
    const float4 *src = reinterpret_cast<const float4 *>(W + (b0 + blk) * 64) + sub;
#pragma unroll
    for (int j = 0; j < 4; ++j) v[it][j] = blk < nblk ? __ldcs(src + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float mu = __ldg(group_scale + ng);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[it][j].x), fabsf(v[it][j].y)), fmaxf(fabsf(v[it][j].z), fabsf(v[it][j].w))));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    if (sub == 0) s_c[warp * 32 + it * 8 + bl] = m;
  }
  __syncthreads();
  const int t = threadIdx.x;
  const float d = t < nblk ? __fsub_rn(s_c[t], mu) : 0.f;
  float m = fabsf(d);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  float S = s_red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) S = fmaxf(S, s_red[i]);
  if (t < nblk) {
    uint32_t q = 0;
    if (S > 0.0f) {
      const float x = __fmul_rn(__fdiv_rn(d, S), 448.0f);
      uint16_t pair;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(pair) : "f"(x));
      q = pair & 0xFFu;
    }
    absmax_q[b0 + t] = static_cast<uint8_t>(q);
  }
  if (t == 0) group_scale[g] = __fdiv_rn(S, 448.0f);
}

}  // namespace

cudaError_t launch_quantize(const float *W, int64_t numel, uint8_t *codes, uint8_t *absmax_q,
                            float *group_scale, float *absmax_fp32, const Nf4Tables &tab, const QuantBuckets &bk,
                            int dq_format, cudaStream_t stream) {
  const int64_t nb = numel / 64;
  const int64_t ng = (nb + kBlocksPerGroup - 1) / kBlocksPerGroup;
  if (ng == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(ng));
  if (bk.ok && !bk.zero_mid)
    quantize_kernel<true, false><<<grid, kThreads, 0, stream>>>(W, nb, codes, absmax_q, group_scale, absmax_fp32, tab,
                                                               bk, dq_format);
  else if (bk.ok)
    quantize_kernel<true, true><<<grid, kThreads, 0, stream>>>(W, nb, codes, absmax_q, group_scale, absmax_fp32, tab,
                                                              bk, dq_format);
  else
    quantize_kernel<false, true><<<grid, kThreads, 0, stream>>>(W, nb, codes, absmax_q, group_scale, absmax_fp32, tab,
                                                               bk, dq_format);
  count_launches(1);
  if (dq_format != kDqFp8Mean) return cudaGetLastError();
  if (ng > 1) {
    dq_mean_kernel<<<1, 1024, 0, stream>>>(absmax_q, ng, nb, group_scale);
    count_launches(1);
  }
  dq_fp8_kernel<<<static_cast<unsigned>(ng), kThreads, 0, stream>>>(W, nb, absmax_q, group_scale);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
