// One pass over dY for both adapter products of the backward:
//
//   U  = bf16(s . dY . B)    [m x r]   the adapter operand of the input
//                                      gradient, and dA = U^T X
//   dB = bf16(dY^T . T)      [n x r]   T = bf16(s X A^T) from the forward
//
// ("QLoRA", Follow one QLoRA training step, step 4: the gradient reaches the
// adapters through the quantized layer; "QLoRA and Quantized Training", The
// idea: only the adapters receive weight gradients.)
//
// dY [m x n] is the large operand (m x n x 2 bytes; r is 16..64), so the two
// products are HBM-bound and each would stream dY on its own.  Here every
// byte of dY is read once:
//
//   * A CTA owns a rectangle of dY: an m-slice (a run of 128-row blocks) by an
//     n-range (a run of 128-column blocks).  A producer warp streams its
//     [128 x 128] stages by TMA (two 128-byte-swizzled 64-column boxes) into a
//     4-slot ring, each stage with the matching [128 x 64] tile of B.
//   * One thread issues two tcgen05 MMA chains on every stage, reading the same
//     shared-memory tile two ways: as a K-major A operand (M = m rows, K = n)
//     for U += dY . B, and as an MN-major A operand (M = n, K = m) for
//     dB += dY^T . T.  N is 64 (columns past r are zeros from the TMA fill).
//   * U of one m-block is complete over the CTA's n-range after the range's
//     stages: four epilogue warps read it from tensor memory (double-buffered,
//     so the next m-block's MMAs proceed) and store it as an fp32 partial of
//     that n-range.  dB of every n-block of the range stays in tensor memory
//     until the m-slice is done, then goes out as an fp32 partial of that
//     m-slice.
//   * A second kernel adds the partials in a fixed order (n-ranges for U,
//     m-slices for dB) and rounds once to bf16: results are deterministic and
//     do not depend on the device, since the split depends on the shape only.
//     The split (m-slices x n-ranges, about one CTA per SM of a B200) is
//     chosen to minimise the stages of the busiest CTA, then the partials'
//     bytes.
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 192;                       // producer, MMA, 4 epilogue warps
constexpr int kStages = 4;
constexpr uint32_t kBox = 128u * 128u;              // one [128 rows x 64 bf16] box, 16 KB
constexpr uint32_t kStageBytes = 3u * kBox;         // dY (two boxes) + B
constexpr uint32_t kTOff = kStages * kStageBytes;   // two T buffers
constexpr uint32_t kBarOff = kTOff + 2u * kBox;
constexpr uint32_t kSmemBytes = kBarOff + 256u + 1024u;   // + barriers, + base alignment slack
constexpr int kAccCols = 64;                        // accumulator columns per block (MMA N)
constexpr int kMaxRangeBlocks = 6;                  // (2 + 6) x 64 = 512 tensor-memory columns
constexpr int64_t kTargetCtas = 148;                // one wave on a B200 (the split depends on the shape only)
static_assert(kSmemBytes <= 227u * 1024u, "shared memory");

struct __align__(64) PassParams {
  CUtensorMap tmDY;    // dY [m x n], box {64, 128}
  CUtensorMap tmB;     // B  [n x r], box {64, 128}
  CUtensorMap tmT;     // T  [m x r], box {64, 128}
  CUtensorMap tmD;     // dB partials [S][n][r] fp32, box {32, 128, 1}
  float *upart;        // [R x m x r] fp32: U of each n-range
  float *dpart;        // [S x n x r] fp32: dB of each m-slice (written through tmD)
  unsigned *err;
  int m, n, r;
  int mblocks, nblocks;
  int nslices, nranges;   // S, R
  uint32_t tmem_cols;
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z), "r"(src)
               : "memory");
}

// Balanced split of `total` items into `parts`: the first item of part i.
__device__ __forceinline__ int split_at(int total, int parts, int i) {
  return static_cast<int>((static_cast<int64_t>(total) * i) / parts);
}

__global__ void __launch_bounds__(kThreads, 1) dy_pass_kernel(const __grid_constant__ PassParams p) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  uint8_t *gbase = dsmem + (base - smem_u32(dsmem));
  uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + kBarOff);
  uint64_t *full = bars;                 // [kStages]  stage landed (TMA)
  uint64_t *empty = bars + kStages;      // [kStages]  stage consumed (MMA commit)
  uint64_t *tfull = bars + 2 * kStages;  // [2]        T buffer landed
  uint64_t *tempty = tfull + 2;          // [2]        T buffer consumed
  uint64_t *ufull = tfull + 4;           // [2]        U accumulator of an m-block complete
  uint64_t *uempty = tfull + 6;          // [2]        U accumulator read out
  uint64_t *dbfull = tfull + 8;          // every MMA complete
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tfull + 9);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = static_cast<int>(blockIdx.x), range = static_cast<int>(blockIdx.y);
  const int mb0 = split_at(p.mblocks, p.nslices, slice);
  const int nmb = split_at(p.mblocks, p.nslices, slice + 1) - mb0;
  const int nb0 = split_at(p.nblocks, p.nranges, range);
  const int nnb = split_at(p.nblocks, p.nranges, range + 1) - nb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 1);
      mbar_init(&ufull[b], 1);
      mbar_init(&uempty[b], 4);
    }
    mbar_init(dbfull, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmDY);
    tma_prefetch_desc(&p.tmB);
    tma_prefetch_desc(&p.tmT);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int li = 0, ti = 0;
      for (int i = 0; i < nmb && ok; ++i) {
        const int mb = mb0 + i, tb = i & 1;
        ok = mbar_wait_bounded(&tempty[tb], ((i >> 1) & 1) ^ 1u, p.err, kErrTimeoutEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(&tfull[tb], kBox);
        tma_load_2d(base + kTOff + tb * kBox, &p.tmT, &tfull[tb], 0, mb * 128);
        ++ti;
        for (int j = 0; j < nnb; ++j, ++li) {
          const int s = li % kStages;
          ok = mbar_wait_bounded(&empty[s], ((li / kStages) & 1) ^ 1u, p.err, kErrTimeoutEmpty);
          if (!ok) break;
          const uint32_t st = base + s * kStageBytes;
          const int n0 = (nb0 + j) * 128;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(st, &p.tmDY, &full[s], n0, mb * 128);
          tma_load_2d(st + kBox, &p.tmDY, &full[s], n0 + 64, mb * 128);
          tma_load_2d(st + 2 * kBox, &p.tmB, &full[s], 0, n0);
        }
      }
      // Copies still in flight land before the CTA's memory is reused (they
      // all have, unless a wait above gave up).
      for (int jj = li - kStages < 0 ? 0 : li - kStages; jj < li; ++jj)
        mbar_wait_bounded(&full[jj % kStages], (jj / kStages) & 1u, p.err, kErrTimeoutDrain);
      for (int i = ti - 2 < 0 ? 0 : ti - 2; i < ti; ++i)
        mbar_wait_bounded(&tfull[i & 1], (i >> 1) & 1u, p.err, kErrTimeoutDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_u = make_idesc(kAccCols, false, true);   // A = dY (K-major), B = B (MN-major)
      constexpr uint32_t idesc_db = make_idesc(kAccCols, true, true);   // A = dY^T (MN-major), B = T (MN-major)
      int li = 0;
      for (int i = 0; i < nmb && ok; ++i) {
        const int tb = i & 1, ub = i & 1;
        ok = mbar_wait_bounded(&tfull[tb], (i >> 1) & 1u, p.err, kErrTimeoutFullB) &&
             mbar_wait_bounded(&uempty[ub], ((i >> 1) & 1) ^ 1u, p.err, kErrTimeoutAcc);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tbuf = base + kTOff + tb * kBox;
        for (int j = 0; j < nnb; ++j, ++li) {
          const int s = li % kStages;
          ok = mbar_wait_bounded(&full[s], (li / kStages) & 1u, p.err, kErrTimeoutFullA);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = base + s * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = smem_desc(st + (kk >> 2) * kBox + (kk & 3) * 32u, 16u, 1024u);
            const uint64_t b = smem_desc(st + 2 * kBox + kk * 2048u, kBox, 1024u);
            umma_f16(tmem + ub * kAccCols, a, b, idesc_u, (j > 0 || kk > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = smem_desc(st + kk * 2048u, kBox, 1024u);
            const uint64_t b = smem_desc(tbuf + kk * 2048u, kBox, 1024u);
            umma_f16(tmem + (2 + j) * kAccCols, a, b, idesc_db, (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&ufull[ub]);
        umma_commit(&tempty[tb]);
      }
      umma_commit(dbfull);
    }
  } else {
    // ------------------------------------------------------------ U partials
    const int q = warp & 3;                       // tensor-memory lanes 32q .. 32q + 31
    const int row = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    for (int i = 0; i < nmb; ++i) {
      const int ub = i & 1;
      if (!mbar_wait_bounded(&ufull[ub], (i >> 1) & 1u, p.err, kErrTimeoutAcc)) break;
      tc_fence_after();
      const int grow = (mb0 + i) * 128 + row;
      float *dst = p.upart + (static_cast<int64_t>(range) * p.m + grow) * p.r;
      for (int c = 0; c < p.r; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_addr + static_cast<uint32_t>(ub * kAccCols + c), v);
        if (grow < p.m) {
          float4 *d4 = reinterpret_cast<float4 *>(dst + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[ub]);
    }
  }

  // ------------------------------------------------------------ dB partials
  // Each n-block's [128 x r] fp32 partial goes through shared memory (the
  // ring is free once every MMA has completed) as 128-byte-swizzled boxes of
  // 32 columns, written out by TMA stores (rows past n are clipped).
  const int nbox = (p.r + 31) / 32;
  if (warp >= 2) {
    const bool acc_ok = nmb == 0 || mbar_wait_bounded(dbfull, 0u, p.err, kErrTimeoutAcc, 20000000000ull);
    tc_fence_after();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    for (int j = 0; j < nnb; ++j) {
      for (int c = 0; c < p.r; c += 16) {
        uint32_t v[16];
        if (nmb > 0 && acc_ok) {
          tmem_ld16(tmem + lane_addr + static_cast<uint32_t>((2 + j) * kAccCols + c), v);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0u;
        }
        const uint32_t box = base + static_cast<uint32_t>(j * 2 + c / 32) * kBox;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t chunk = static_cast<uint32_t>((c % 32) / 4 + e);
          const uint32_t w[4] = {v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]};
          sts128(box + row * 128u + ((chunk ^ static_cast<uint32_t>(row & 7)) << 4), w);
        }
      }
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (warp == 2 && lane == 0) {
    for (int j = 0; j < nnb; ++j)
      for (int b = 0; b < nbox; ++b)
        tma_store_3d(&p.tmD, base + static_cast<uint32_t>(j * 2 + b) * kBox, 32 * b, (nb0 + j) * 128, slice);
    tma_store_drain();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols) : "memory");
}

// out[i] = bf16(scale * sum over parts of part[p][i]), parts in order.
__device__ __forceinline__ uint2 sum_parts(const float4 *__restrict__ part, int parts, int64_t stride, int64_t i,
                                           float scale) {
  float4 acc = __ldcs(part + i);
  int pi = 1;
  // Eight partials' loads in flight at once; the additions stay in order.
  for (; pi + 8 <= parts; pi += 8) {
    float4 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __ldcs(part + (pi + e) * stride + i);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc.x += v[e].x;
      acc.y += v[e].y;
      acc.z += v[e].z;
      acc.w += v[e].w;
    }
  }
  for (; pi < parts; ++pi) {
    const float4 v = __ldcs(part + pi * stride + i);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  return make_uint2(pack_bf16x2(scale * acc.x, scale * acc.y), pack_bf16x2(scale * acc.z, scale * acc.w));
}

// U = bf16(s * sum of the n-ranges' partials) [m x r] and dB = bf16(sum of the
// m-slices' partials) [n x r], four elements per thread.
__global__ void __launch_bounds__(256) pass_reduce_kernel(const float4 *__restrict__ upart, int nranges, int64_t u4,
                                                           float scale, uint2 *__restrict__ U,
                                                           const float4 *__restrict__ dpart, int nslices,
                                                           int64_t d4, uint2 *__restrict__ dB) {
  // The input-gradient kernel that consumes U may launch now; it waits for
  // this grid before it reads U.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < u4 + d4; i += stride) {
    if (i < u4)
      U[i] = sum_parts(upart, nranges, u4, i, scale);
    else
      dB[i - u4] = sum_parts(dpart, nslices, d4, i - u4, 1.0f);
  }
}

}  // namespace

DyPassPlan plan_dy_pass(int64_t m, int64_t n, int32_t r) {
  DyPassPlan pl{};
  if (m <= 0 || n <= 0 || r <= 0 || r > 64 || (r % 16) != 0) return pl;
  if (m > (int64_t(1) << 31) || n > (int64_t(1) << 31)) return pl;
  const int64_t mblocks = (m + 127) / 128, nblocks = (n + 127) / 128;
  const int64_t rmin = (nblocks + kMaxRangeBlocks - 1) / kMaxRangeBlocks;
  const int64_t rmax = std::max(rmin, std::min<int64_t>(nblocks, kTargetCtas));
  int64_t best_w = INT64_MAX, best_p = INT64_MAX;
  for (int64_t R = rmin; R <= rmax; ++R) {
    const int64_t S = std::min<int64_t>(mblocks, std::max<int64_t>(1, kTargetCtas / R));
    const int64_t w = ((mblocks + S - 1) / S) * ((nblocks + R - 1) / R);    // stages of the busiest CTA
    const int64_t parts = R * m + S * n;                                     // partial rows of r floats
    if (w < best_w || (w == best_w && parts < best_p)) {
      best_w = w;
      best_p = parts;
      pl.nslices = static_cast<int>(S);
      pl.nranges = static_cast<int>(R);
    }
  }
  if (pl.nranges > 65535) return DyPassPlan{};
  const int64_t nb = (nblocks + pl.nranges - 1) / pl.nranges;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>((2 + nb) * kAccCols)) cols *= 2;
  pl.tmem_cols = cols;
  pl.upart_bytes = static_cast<size_t>(pl.nranges) * static_cast<size_t>(m) * static_cast<size_t>(r) * 4u;
  pl.dpart_bytes = static_cast<size_t>(pl.nslices) * static_cast<size_t>(n) * static_cast<size_t>(r) * 4u;
  pl.ok = true;
  return pl;
}

size_t dy_pass_workspace_bytes(int64_t m, int64_t n, int32_t r) {
  const DyPassPlan pl = plan_dy_pass(m, n, r);
  if (!pl.ok) return 0;
  return (pl.upart_bytes + 255u) / 256u * 256u + pl.dpart_bytes;
}

cudaError_t launch_dy_pass(const uint16_t *dY, int64_t m, int64_t n, const uint16_t *B, const uint16_t *T, int32_t r,
                           float scale, uint16_t *U, uint16_t *dB, void *scratch, size_t scratch_bytes,
                           cudaStream_t stream, bool pdl_reduce) {
  if (m <= 0) return cudaSuccess;
  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(dy_pass_kernel), static_cast<int>(kSmemBytes),
                                configured);
  if (e != cudaSuccess) return e;
  const DyPassPlan pl = plan_dy_pass(m, n, r);
  if (!pl.ok || dy_pass_workspace_bytes(m, n, r) > scratch_bytes) return cudaErrorInvalidValue;
  float *upart = static_cast<float *>(scratch);
  float *dpart = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + (pl.upart_bytes + 255u) / 256u * 256u);

  PassParams p{};
  if (!encode_bf16_map(&p.tmDY, dY, m, n, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_bf16_map(&p.tmB, B, n, r, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_bf16_map(&p.tmT, T, m, r, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_f32_slab_map(&p.tmD, dpart, pl.nslices, n, r, 32, 128)) return cudaErrorInvalidValue;
  p.upart = upart;
  p.dpart = dpart;
  p.err = device_error_word();
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.r = r;
  p.mblocks = static_cast<int>((m + 127) / 128);
  p.nblocks = static_cast<int>((n + 127) / 128);
  p.nslices = pl.nslices;
  p.nranges = pl.nranges;
  p.tmem_cols = pl.tmem_cols;
  dy_pass_kernel<<<dim3(static_cast<unsigned>(pl.nslices), static_cast<unsigned>(pl.nranges), 1), kThreads,
                   kSmemBytes, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launches(1);

  const int64_t u4 = m * r / 4, d4 = n * r / 4;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (u4 + d4 + 255) / 256;
  cudaLaunchConfig_t rc{};
  rc.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 4)), 1, 1);
  rc.blockDim = dim3(256, 1, 1);
  rc.stream = stream;
  cudaLaunchAttribute rattr[1];
  rattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  rattr[0].val.programmaticStreamSerializationAllowed = 1;
  rc.attrs = rattr;
  rc.numAttrs = pdl_reduce ? 1 : 0;
  e = cudaLaunchKernelEx(&rc, pass_reduce_kernel, reinterpret_cast<const float4 *>(upart), pl.nranges, u4, scale,
                         reinterpret_cast<uint2 *>(U), reinterpret_cast<const float4 *>(dpart), pl.nslices, d4,
                         reinterpret_cast<uint2 *>(dB));
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace qlora
