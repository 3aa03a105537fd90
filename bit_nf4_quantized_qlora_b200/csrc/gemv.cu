// Small-M forward (M <= 16): Y = bf16(X . W^T + T . B^T), weight-streaming.
//
// At decode-sized M the layer is bound by reading the packed weights from HBM
// ("QLoRA and Quantized Training", The idea: dequantize each block, multiply,
// discard).  Each warp owns 16 weight rows and walks K in chunks of 256 (four
// NF4 blocks per row); lane (g = lane/4, q = lane%4) streams the 32 bytes of
// block q of rows g and g+8 with 16-byte loads, expands them to exact bf16 W^
// in registers (per-block table, common.cuh) and feeds m16n8k16 tensor-core
// MMAs whose A operand is X.  The MMA's k order inside a step is permuted to
// match what each lane holds, and X is read with the same permutation.
//
// A CTA is 8 warps = 2 row groups x 4 K parts (32 rows).  A thread-block
// cluster of 1..8 CTAs splits K further; partial sums meet in shared memory
// and are reduced across the cluster through distributed shared memory, after
// which the adapter term T . B^T is added and Y is written once in bf16.
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kThreads = 256;
constexpr int kNT = 2;                         // n8 tiles per warp
constexpr int kRowsPerWarp = 8 * kNT;          // 16
constexpr int kKParts = 4;
constexpr int kRowGroups = (kThreads / 32) / kKParts;  // 2
constexpr int kRows = kRowGroups * kRowsPerWarp;       // 32 rows per CTA
constexpr int kMaxM = 16;

struct GemvParams {
  const uint16_t *X;
  const uint8_t *codes;
  const uint8_t *absmax_q;
  const float *group_scale;
  const uint16_t *T;
  const uint16_t *B;
  uint16_t *Y;
  int64_t n, k;
  int m, r;
  int nchunks;
  Nf4Tables tab;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(const float *local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads) gemv_fwd_kernel(const __grid_constant__ GemvParams p) {
  __shared__ float red[kKParts][kMaxM][kRows];

  const uint32_t crank = cluster_rank();
  const uint32_t csize = cluster_size();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int rg = warp / kKParts, kp = warp % kKParts;
  const int64_t n_cta = static_cast<int64_t>(blockIdx.x) * kRows;
  const int64_t kblocks = p.k / 64;
  const int c_lo = static_cast<int>((static_cast<int64_t>(p.nchunks) * crank) / csize);
  const int c_hi = static_cast<int>((static_cast<int64_t>(p.nchunks) * (crank + 1)) / csize);

  float acc[kNT][4];
#pragma unroll
  for (int t = 0; t < kNT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  const bool row_lo_x = g < p.m;
  const bool row_hi_x = g + 8 < p.m;

#pragma unroll 1
  for (int c = c_lo + kp; c < c_hi; c += kKParts) {
    const int64_t kb = static_cast<int64_t>(c) * 4 + q;
    const bool kvalid = kb < kblocks;
    uint4 cw[kNT][2];
    Bf16Table tb[kNT];
#pragma unroll
    for (int t = 0; t < kNT; ++t) {
      const int64_t row = n_cta + rg * kRowsPerWarp + 8 * t + g;
      if (kvalid && row < p.n) {
        const int64_t blk = row * kblocks + kb;
        const uint4 *src = reinterpret_cast<const uint4 *>(p.codes + blk * 32);
        cw[t][0] = __ldcs(src);
        cw[t][1] = __ldcs(src + 1);
        const uint32_t qv = __ldg(p.absmax_q + blk);
        const float S = __ldg(p.group_scale + (blk >> 8));
        make_table(p.tab, absmax_dequant(qv, S), tb[t]);
      } else {
        cw[t][0] = cw[t][1] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < 4; ++j) tb[t].lo[j] = tb[t].hi[j] = 0u;
      }
    }
    const uint16_t *xg = p.X + static_cast<int64_t>(g) * p.k + kb * 64;
    const uint16_t *x8 = p.X + static_cast<int64_t>(g + 8) * p.k + kb * 64;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t P[kNT][4];
#pragma unroll
      for (int t = 0; t < kNT; ++t) {
        const uint4 &v = cw[t][w >> 2];
        const uint32_t word = (w & 3) == 0 ? v.x : (w & 3) == 1 ? v.y : (w & 3) == 2 ? v.z : v.w;
        decode8(word, tb[t], P[t]);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int ss = 2 * w + h;
        uint2 xa = make_uint2(0u, 0u), xb = make_uint2(0u, 0u);
        if (kvalid && row_lo_x) xa = __ldg(reinterpret_cast<const uint2 *>(xg + 4 * ss));
        if (kvalid && row_hi_x) xb = __ldg(reinterpret_cast<const uint2 *>(x8 + 4 * ss));
        const uint32_t a[4] = {xa.x, xb.x, xa.y, xb.y};
#pragma unroll
        for (int t = 0; t < kNT; ++t) mma_bf16_16816(acc[t], a, P[t][2 * h], P[t][2 * h + 1]);
      }
    }
  }

  // Partial sums of this warp: D[m][n] with m = g, g+8 and n = 2q, 2q+1.
#pragma unroll
  for (int t = 0; t < kNT; ++t) {
    const int nl = rg * kRowsPerWarp + 8 * t + 2 * q;
    red[kp][g][nl] = acc[t][0];
    red[kp][g][nl + 1] = acc[t][1];
    red[kp][g + 8][nl] = acc[t][2];
    red[kp][g + 8][nl + 1] = acc[t][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kMaxM * kRows; i += kThreads) {
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kKParts; ++j) s += (&red[j][0][0])[i];
    (&red[0][0][0])[i] = s;
  }
  cluster_sync_all();

  // Each CTA of the cluster finishes a slice of the 32 rows.
  const int rpr = kRows / static_cast<int>(csize);
  for (int i = threadIdx.x; i < p.m * rpr; i += kThreads) {
    const int mi = i / rpr;
    const int nl = static_cast<int>(crank) * rpr + (i % rpr);
    const int64_t n = n_cta + nl;
    if (n >= p.n) continue;
    float s = 0.f;
    for (uint32_t peer = 0; peer < csize; ++peer) s += ld_dsmem_f32(&red[0][mi][nl], peer);
    if (p.r > 0) {
      const uint16_t *trow = p.T + static_cast<int64_t>(mi) * p.r;
      const uint16_t *brow = p.B + n * p.r;
      for (int j = 0; j < p.r; j += 8) {
        const uint4 tv = *reinterpret_cast<const uint4 *>(trow + j);
        const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(brow + j));
        const uint32_t ta[4] = {tv.x, tv.y, tv.z, tv.w};
        const uint32_t ba[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s = fmaf(bf16lo_to_f32(ta[e]), bf16lo_to_f32(ba[e]), s);
          s = fmaf(bf16hi_to_f32(ta[e]), bf16hi_to_f32(ba[e]), s);
        }
      }
    }
    const uint32_t packed = pack_bf16x2(s, 0.f);
    p.Y[static_cast<int64_t>(mi) * p.n + n] = static_cast<uint16_t>(packed & 0xFFFFu);
  }
  cluster_sync_all();
}

// T[m x r] = bf16(scale * X . A^T): one CTA per adapter row j.
__global__ void __launch_bounds__(256) lora_proj_small_kernel(const uint16_t *__restrict__ X, int m,
                                                              int64_t k, const uint16_t *__restrict__ A,
                                                              int r, float scale,
                                                              uint16_t *__restrict__ T) {
  __shared__ float red[8][kMaxM];
  const int j = blockIdx.x;
  const uint16_t *arow = A + static_cast<int64_t>(j) * k;
  float acc[kMaxM];
#pragma unroll
  for (int i = 0; i < kMaxM; ++i) acc[i] = 0.f;
  for (int64_t kk = static_cast<int64_t>(threadIdx.x) * 8; kk < k; kk += 256 * 8) {
    const uint4 av = __ldg(reinterpret_cast<const uint4 *>(arow + kk));
    const uint32_t aa[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int i = 0; i < kMaxM; ++i) {
      if (i < m) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<int64_t>(i) * k + kk));
        const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
        float s = acc[i];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s = fmaf(bf16lo_to_f32(xx[e]), bf16lo_to_f32(aa[e]), s);
          s = fmaf(bf16hi_to_f32(xx[e]), bf16hi_to_f32(aa[e]), s);
        }
        acc[i] = s;
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < kMaxM; ++i) {
    float v = acc[i];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][i] = v;
  }
  __syncthreads();
  if (threadIdx.x < m) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w][threadIdx.x];
    T[static_cast<int64_t>(threadIdx.x) * r + j] = static_cast<uint16_t>(pack_bf16x2(s * scale, 0.f) & 0xFFFFu);
  }
}

}  // namespace

cudaError_t launch_lora_proj_small(const uint16_t *X, int64_t m, int64_t k, const uint16_t *A,
                                   int32_t r, float scale, uint16_t *T, cudaStream_t stream) {
  if (m <= 0 || r <= 0) return cudaSuccess;
  lora_proj_small_kernel<<<r, 256, 0, stream>>>(X, static_cast<int>(m), k, A, r, scale, T);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_gemv_fwd(const uint16_t *X, int64_t m, const uint8_t *codes, const uint8_t *absmax_q,
                            const float *group_scale, int64_t n, int64_t k, const uint16_t *T,
                            const uint16_t *B, int32_t r, uint16_t *Y, cudaStream_t stream) {
  if (m <= 0) return cudaSuccess;
  GemvParams p{};
  p.X = X;
  p.codes = codes;
  p.absmax_q = absmax_q;
  p.group_scale = group_scale;
  p.T = T;
  p.B = B;
  p.Y = Y;
  p.n = n;
  p.k = k;
  p.m = static_cast<int>(m);
  p.r = (T != nullptr && B != nullptr) ? r : 0;
  p.nchunks = static_cast<int>((k + 255) / 256);
  p.tab = nf4_tables();

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t row_ctas = (n + kRows - 1) / kRows;
  // Split K over a cluster until there are about three CTAs per SM, keeping
  // at least one chunk of K per warp and never more than 8 CTAs per cluster.
  int cs = 1;
  while (cs < 8 && row_ctas * cs < 3LL * sms && p.nchunks / (cs * 2) >= kKParts) cs *= 2;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(row_ctas), static_cast<unsigned>(cs), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_fwd_kernel, p);
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace qlora
