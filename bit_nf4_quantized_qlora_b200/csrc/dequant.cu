// Standalone NF4 dequantization to bf16 (HBM-bound).
//
// "QLoRA", Storage precision is not calculation precision: the 4-bit stored
// weight is dequantized to a higher-precision compute type; "A 65B fine-tune
// on the GPU you already have", figure 2: block by block to bf16.
//
// The output (2 bytes per weight) is four fifths of the traffic, so it leaves
// through TMA stores: a CTA expands a chunk of 128 blocks (8192 weights) into
// a 16 KB shared-memory tile laid out as the TMA box [128 blocks x 64
// weights] with the 128-byte swizzle (a quarter-warp's 16-byte stores land in
// eight distinct bank groups), and one thread writes the tile with a single
// TMA store while the CTA expands the next chunk into the other half of a
// double buffer.  Each thread expands half a block (32 weights): one 16-byte
// load of packed codes (issued a chunk ahead), the absmax code and group
// constant of its block, a per-block bf16 table (see common.cuh) and four
// 16-byte shared-memory stores.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 256;                   // two threads per block
constexpr int kChunkBlocks = kThreads / 2;      // 128 blocks per chunk
constexpr uint32_t kTileBytes = kChunkBlocks * 128u;

__global__ void __launch_bounds__(kThreads) dequant_kernel(const __grid_constant__ CUtensorMap tmOut,
                                                           const uint8_t *__restrict__ codes,
                                                           const uint8_t *__restrict__ absmax_q,
                                                           const float *__restrict__ group_scale,
                                                           int64_t nblocks, const Nf4Tables tab,
                                                           const float *mu_ptr) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const bool fp8 = mu_ptr != nullptr;
  const float mu = load_mu(mu_ptr);
  const int t = threadIdx.x;
  const int bl = t >> 1, h = t & 1;             // block of the chunk, half of the block
  const int64_t nchunks = (nblocks + kChunkBlocks - 1) / kChunkBlocks;

  int64_t chunk = blockIdx.x;
  uint4 cw = make_uint4(0u, 0u, 0u, 0u);
  auto load_codes = [&](int64_t ch) {
    const int64_t blk = ch * kChunkBlocks + bl;
    cw = (ch < nchunks && blk < nblocks) ? __ldcs(reinterpret_cast<const uint4 *>(codes) + blk * 2 + h)
                                         : make_uint4(0u, 0u, 0u, 0u);
  };
  load_codes(chunk);
  for (int it = 0; chunk < nchunks; ++it, chunk += gridDim.x) {
    const int64_t blk = chunk * kChunkBlocks + bl;
    const uint4 cur = cw;
    load_codes(chunk + gridDim.x);
    const uint32_t buf = base + static_cast<uint32_t>(it & 1) * kTileBytes;
    // The store that last read this half of the buffer (two chunks ago) has
    // finished reading shared memory.
    if (t == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
    __syncthreads();
    uint32_t o[16];
    if (blk < nblocks) {
      const float S = __ldg(group_scale + (blk >> 8));
      Bf16Table tb;
      make_table(tab, block_constant(__ldg(absmax_q + blk), group_constant(S, fp8), fp8, mu), tb);
      decode8(cur.x, tb, o + 0);
      decode8(cur.y, tb, o + 4);
      decode8(cur.z, tb, o + 8);
      decode8(cur.w, tb, o + 12);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) o[e] = 0u;
    }
    // Row bl of the tile (128 bytes), 16-byte chunks 4h .. 4h+3, swizzled.
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t c = static_cast<uint32_t>(4 * h + j) ^ static_cast<uint32_t>(bl & 7);
      const uint32_t w[4] = {o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]};
      sts128(buf + static_cast<uint32_t>(bl) * 128u + (c << 4), w);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (t == 0) {
      tma_store_2d(&tmOut, buf, 0, static_cast<int>(chunk * kChunkBlocks));
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
  }
  if (t == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace

cudaError_t launch_dequant(const uint8_t *codes, const uint8_t *absmax_q, const float *group_scale,
                           int64_t numel, uint16_t *out, const Nf4Tables &tab, int dq_format,
                           cudaStream_t stream) {
  const int64_t nblocks = numel / 64;
  if (nblocks == 0) return cudaSuccess;
  if (nblocks > (int64_t(1) << 31) - kChunkBlocks) return cudaErrorInvalidValue;
  CUtensorMap tm;
  // The output as [nblocks rows x 64 weights] bf16; stores clip past the last block.
  if (!encode_bf16_map(&tm, out, nblocks, 64, 64, kChunkBlocks)) return cudaErrorInvalidValue;
  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  constexpr int smem = static_cast<int>(2 * kTileBytes + 1024);
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(dequant_kernel), smem, configured);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nchunks = (nblocks + kChunkBlocks - 1) / kChunkBlocks;
  const int64_t cap = static_cast<int64_t>(sms) * 4;
  const unsigned grid = static_cast<unsigned>(nchunks < cap ? nchunks : cap);
  dequant_kernel<<<grid, kThreads, smem, stream>>>(tm, codes, absmax_q, group_scale, nblocks, tab,
                                                   mean_ptr(group_scale, nblocks, dq_format));
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
