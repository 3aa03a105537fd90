// Small-M forward (M <= 16): Y = bf16(X . W^T + T . B^T), weight-streaming.
// Decode sizes (M <= 4, K up to 32768) take the per-warp streaming kernel of
// gemv_stream.cu; this CTA-ring kernel serves M = 5..16 and longer K.
//
// At decode-sized M the layer is bound by reading the packed weights from HBM
// ("QLoRA and Quantized Training", The idea: dequantize each block, multiply,
// discard), so the kernel is a streaming pipeline whose decode costs two
// integer ops (the table address) and one shared-memory load per two weights:
//
//   * one producer warp streams each stage into a shared-memory ring with TMA:
//     a 16 KB tile of packed codes (128 weight rows x 4 NF4 blocks) and the
//     matching 16-token x 4-block slice of X, both 128-byte swizzled, on one
//     mbarrier, so the consumers never wait on a global load of X;
//   * a 32 KB shared table maps every code byte (two weights) to the bf16 pair
//     {NF4[hi nibble], NF4[lo nibble]}, with 32 lane-private copies in each
//     128-byte row so 32 lookups always hit 32 banks;
//   * eight consumer warps (16 rows each) feed the pairs as the A operand of
//     m16n8k16 tensor-core MMAs with X as the B operand; the four MMAs of an
//     NF4 block accumulate into a fresh tile that is scaled by the block's
//     reconstructed absmax c' = q * fp32(S/255) and added to the running sum;
//   * when the 128-row tiles alone leave SMs empty, a cluster of CTAs splits
//     K; partial tiles are reduced through distributed shared memory (in the
//     ring's memory, free by then) and the adapter term T . B^T is added before
//     Y is written once in bf16.  T comes from the preceding projection
//     kernel, which this kernel overlaps (programmatic dependent launch) and
//     waits for only before its epilogue.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kConsumers = 8;
constexpr int kThreads = 32 * (kConsumers + 1);       // + one producer warp
constexpr int kRows = 16 * kConsumers;                 // 128 weight rows per CTA
constexpr int kStageBlocks = 4;                        // NF4 blocks of K per stage
constexpr uint32_t kStageBytes = kRows * kStageBlocks * 32u;   // 16 KB
constexpr int kStages = 3;                             // x 2 CTAs per SM
constexpr int kMaxM = 16;
constexpr uint32_t kXBlockBytes = 16u * 128u;          // X slice of one NF4 block: 16 tokens x 64 bf16
constexpr uint32_t kSlotBytes = kStageBytes + kStageBlocks * kXBlockBytes;   // codes tile, then X
constexpr uint32_t kLutBytes = 256u * 128u;            // one 128-byte row per code byte
constexpr uint32_t kRedBytes = kMaxM * kRows * 4u;     // partial sums, aliased onto the ring
static_assert(kRedBytes <= kStages * kSlotBytes, "partial sums fit in the ring");
constexpr uint32_t kSmemBytes = kLutBytes + 1024u + kStages * kSlotBytes;

struct __align__(64) GemvParams {
  CUtensorMap tmCodes;          // codes as [n rows x k/2 bytes], box {128, 128}, 128B swizzle
  CUtensorMap tmX;              // X as [m rows x k] bf16, box {64, 8 or 16}, 128B swizzle
  const uint16_t *X;
  const uint8_t *absmax_q;
  const float *group_scale;
  const float *mu;              // E4M3 + mean absmax format: the tensor mean; else null
  const uint16_t *T;
  const uint16_t *B;
  uint16_t *Y;
  unsigned *err;
  int64_t n, k;
  int m, r;
  uint32_t x_box_bytes;         // bytes of one X box (64 columns x 8 or 16 token rows)
  Nf4Tables tab;
};

// The byte-pair table: row b (128 bytes) holds 32 copies of the bf16 pair
// {NF4[b >> 4], NF4[b & 15]}, one per lane.
__device__ __forceinline__ void build_lut(uint8_t *lut, const Nf4Tables &tab, int tid, int nthreads) {
  uint4 *lw = reinterpret_cast<uint4 *>(lut);
  for (int i = tid; i < 256 * 8; i += nthreads) {
    const int b = i >> 3;
    const uint32_t v = pack_bf16x2(tab.level[b >> 4], tab.level[b & 15]);
    lw[i] = make_uint4(v, v, v, v);
  }
}
// Table offset of byte J (0..3) of `word` for the lane whose lane*4 is lane4.
template <int J>
__device__ __forceinline__ uint32_t lut_off(uint32_t word, uint32_t lane4) {
  const uint32_t sh = J == 0 ? (word << 7) : (word >> (8 * J - 7));
  return (sh & 0x7F80u) | lane4;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// One NF4 block (4 MMA k-steps) of this lane's two rows: returns the block's
// raw products (before its absmax scale) in bacc.
template <int TOK_TILES>
__device__ __forceinline__ void block_mma(float (&bacc)[TOK_TILES][4], uint2 c0, uint2 c1, const uint4 (&xa)[TOK_TILES],
                                          const uint4 (&xb)[TOK_TILES], const uint8_t *lut, uint32_t lane4) {
#pragma unroll
  for (int t = 0; t < TOK_TILES; ++t) bacc[t][0] = bacc[t][1] = bacc[t][2] = bacc[t][3] = 0.f;
#pragma unroll
  for (int ss = 0; ss < 4; ++ss) {
    const uint32_t w0 = ss < 2 ? c0.x : c0.y;
    const uint32_t w1 = ss < 2 ? c1.x : c1.y;
    uint32_t a[4];
    if ((ss & 1) == 0) {
      a[0] = *reinterpret_cast<const uint32_t *>(lut + lut_off<0>(w0, lane4));
      a[1] = *reinterpret_cast<const uint32_t *>(lut + lut_off<0>(w1, lane4));
      a[2] = *reinterpret_cast<const uint32_t *>(lut + lut_off<1>(w0, lane4));
      a[3] = *reinterpret_cast<const uint32_t *>(lut + lut_off<1>(w1, lane4));
    } else {
      a[0] = *reinterpret_cast<const uint32_t *>(lut + lut_off<2>(w0, lane4));
      a[1] = *reinterpret_cast<const uint32_t *>(lut + lut_off<2>(w1, lane4));
      a[2] = *reinterpret_cast<const uint32_t *>(lut + lut_off<3>(w0, lane4));
      a[3] = *reinterpret_cast<const uint32_t *>(lut + lut_off<3>(w1, lane4));
    }
#pragma unroll
    for (int t = 0; t < TOK_TILES; ++t) {
      const uint4 &xv = ss < 2 ? xa[t] : xb[t];
      mma_bf16_16816(bacc[t], a[0], a[1], a[2], a[3], (ss & 1) ? xv.z : xv.x, (ss & 1) ? xv.w : xv.y);
    }
  }
}

template <int TOK_TILES>
__global__ void __launch_bounds__(kThreads, 2) gemv_fwd_kernel(const __grid_constant__ GemvParams p) {
  extern __shared__ __align__(16) uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];

  // The byte-pair table sits at the start of dynamic shared memory (a
  // link-time constant address); the TMA ring is 1024-aligned after it.
  const uint8_t *lut = dsmem;
  const uint32_t ring = (smem_u32(dsmem) + kLutBytes + 1023u) & ~1023u;
  // The partial sums reuse the ring once every stage has been consumed.
  const uint32_t red_addr = ring;
  float *red = reinterpret_cast<float *>(dsmem + (red_addr - smem_u32(dsmem)));

  const uint32_t crank = cluster_rank();
  const uint32_t csize = cluster_size();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n_cta = static_cast<int64_t>(blockIdx.x) * kRows;
  const int kblocks = static_cast<int>(p.k / 64);
  // This CTA's share of K in whole stages of 4 blocks (the last may be ragged).
  const int nst_all = (kblocks + kStageBlocks - 1) / kStageBlocks;
  const int st_lo = static_cast<int>((static_cast<int64_t>(nst_all) * crank) / csize);
  const int st_hi = static_cast<int>((static_cast<int64_t>(nst_all) * (crank + 1)) / csize);
  const int nst = st_hi - st_lo;
  const int kb_lo = st_lo * kStageBlocks;
  // CTAs walk their stages from different starting points (rotated by the
  // row tile's index), so that at any moment the CTAs read different slices
  // of X rather than all hitting the same few L2 lines.
  const int rot = nst > 0 ? static_cast<int>(blockIdx.x % static_cast<unsigned>(nst)) : 0;
  const auto phys = [&](int st) { return st + rot < nst ? st + rot : st + rot - nst; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumers);
    }
    fence_mbar_init();
  }
  build_lut(dsmem, p.tab, threadIdx.x, kThreads);
  __syncthreads();

  const int g = lane >> 2, q = lane & 3;
  const int lr0 = warp * 16 + g, lr1 = lr0 + 8;          // rows of the tile (rows past n are
  float acc[TOK_TILES][4];                                // computed but never stored)
#pragma unroll
  for (int t = 0; t < TOK_TILES; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int st = 0; st < nst; ++st) {
        const int s = st % kStages;
        const uint32_t ph = static_cast<uint32_t>(st / kStages) & 1u;
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, p.err, kErrTimeoutEmpty)) break;
        const int kb_st = kb_lo + phys(st) * kStageBlocks;
        const int nb = kblocks - kb_st < kStageBlocks ? kblocks - kb_st : kStageBlocks;   // blocks of X inside K
        mbar_arrive_expect_tx(&full_bar[s], kStageBytes + static_cast<uint32_t>(nb) * p.x_box_bytes);
        const uint32_t slot = ring + s * kSlotBytes;
        tma_load_2d(slot, &p.tmCodes, &full_bar[s], kb_st * 32, static_cast<int>(n_cta));
        for (int b = 0; b < nb; ++b)
          tma_load_2d(slot + kStageBytes + b * kXBlockBytes, &p.tmX, &full_bar[s], (kb_st + b) * 64, 0);
        ++issued;
      }
      for (int st = issued - kStages < 0 ? 0 : issued - kStages; st < issued; ++st)
        mbar_wait_bounded(&full_bar[st % kStages], static_cast<uint32_t>(st / kStages) & 1u, p.err,
                          kErrTimeoutDrain);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int64_t gr0 = n_cta + lr0 < p.n ? n_cta + lr0 : p.n - 1;   // computed but never stored)
    const int64_t gr1 = n_cta + lr1 < p.n ? n_cta + lr1 : p.n - 1;
    const int64_t b0 = gr0 * kblocks, b1 = gr1 * kblocks;
    const uint8_t *q0p = p.absmax_q + b0 + kb_lo;
    const uint8_t *q1p = p.absmax_q + b1 + kb_lo;
    // Word loads of 4 absmax codes need 4-aligned block indices.
    const bool qwords = (kblocks & 3) == 0;
    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    // Swizzled offsets (inside a stage tile) of this lane's 8 bytes of block b.
    uint32_t off0[kStageBlocks], off1[kStageBlocks];
#pragma unroll
    for (int b = 0; b < kStageBlocks; ++b) {
      const uint32_t chunk = ((2u * b + (q >> 1)) ^ static_cast<uint32_t>(g)) << 4;
      off0[b] = static_cast<uint32_t>(lr0) * 128u + chunk + 8u * (q & 1);
      off1[b] = static_cast<uint32_t>(lr1) * 128u + chunk + 8u * (q & 1);
    }

    // t (the group constant, fp32(S / 255) for linear 8-bit codes) of each
    // row's current group and the block where the next group starts.
    const bool fp8 = p.mu != nullptr;
    const float mu = load_mu(p.mu);
    float t0 = 0.f, t1 = 0.f;
    int next0 = kb_lo, next1 = kb_lo;

    // Swizzled offsets of this lane's two 16-byte pieces of X (columns 16q ..
    // 16q + 15 of token g + 8t) inside a block's X slice.
    uint32_t xoff[TOK_TILES][2];
#pragma unroll
    for (int t = 0; t < TOK_TILES; ++t) {
      const uint32_t row = static_cast<uint32_t>(g + 8 * t) * 128u;
      xoff[t][0] = row + ((static_cast<uint32_t>(2 * q) ^ static_cast<uint32_t>(g)) << 4);
      xoff[t][1] = row + ((static_cast<uint32_t>(2 * q + 1) ^ static_cast<uint32_t>(g)) << 4);
    }

    bool ok = true;
    // Absmax code words of a whole stage (4-aligned blocks, stage inside K),
    // loaded one stage ahead so that their latency hides under a stage.
    const auto stage_words = [&](int st_, uint32_t &w0, uint32_t &w1) {
      const int sp_ = phys(st_);
      if (qwords && kb_lo + (sp_ + 1) * kStageBlocks <= kblocks) {
        w0 = __ldg(reinterpret_cast<const uint32_t *>(q0p + sp_ * kStageBlocks));
        w1 = __ldg(reinterpret_cast<const uint32_t *>(q1p + sp_ * kStageBlocks));
      }
    };
    uint32_t wn0 = 0, wn1 = 0;
    if (nst > 0) stage_words(0, wn0, wn1);
    for (int st = 0; st < nst && ok; ++st) {
      const int s = st % kStages;
      const uint32_t ph = static_cast<uint32_t>(st / kStages) & 1u;
      const uint32_t wc0 = wn0, wc1 = wn1;
      if (st + 1 < nst) stage_words(st + 1, wn0, wn1);
      const int sp = phys(st);
      const int kb_st = kb_lo + sp * kStageBlocks;
      // Back at the start of the CTA's K range: the group constants are
      // looked up afresh.
      if (sp == 0 && st > 0) next0 = next1 = kb_lo;
      const bool full = kb_st + kStageBlocks <= kblocks;
      // Absmax codes of this stage (prefetched on the word path).
      float qf0[kStageBlocks], qf1[kStageBlocks];
      bool qv[kStageBlocks];
      if (full && qwords) {
        const uint32_t w0 = wc0, w1 = wc1;
        if (fp8) {
#pragma unroll
          for (int b = 0; b < kStageBlocks; ++b) {
            qf0[b] = e4m3_to_f32((w0 >> (8 * b)) & 0xFFu);
            qf1[b] = e4m3_to_f32((w1 >> (8 * b)) & 0xFFu);
          }
        } else {
          qf0[0] = byte_to_f32<0>(w0); qf0[1] = byte_to_f32<1>(w0); qf0[2] = byte_to_f32<2>(w0); qf0[3] = byte_to_f32<3>(w0);
          qf1[0] = byte_to_f32<0>(w1); qf1[1] = byte_to_f32<1>(w1); qf1[2] = byte_to_f32<2>(w1); qf1[3] = byte_to_f32<3>(w1);
        }
#pragma unroll
        for (int b = 0; b < kStageBlocks; ++b) qv[b] = true;
      } else {
#pragma unroll
        for (int b = 0; b < kStageBlocks; ++b) {
          qv[b] = kb_st + b < kblocks;
          qf0[b] = qv[b] ? code_value(__ldg(q0p + sp * kStageBlocks + b), fp8) : 0.f;
          qf1[b] = qv[b] ? code_value(__ldg(q1p + sp * kStageBlocks + b), fp8) : 0.f;
        }
      }
      // Group constants: with 4-aligned blocks a group boundary falls on a
      // stage start; otherwise the slow path below takes it block by block.
      if (kb_st >= next0) {
        t0 = group_constant(__ldg(p.group_scale + ((b0 + kb_st) >> 8)), fp8);
        next0 = kb_st + 256 - static_cast<int>((b0 + kb_st) & 255);
      }
      if (kb_st >= next1) {
        t1 = group_constant(__ldg(p.group_scale + ((b1 + kb_st) >> 8)), fp8);
        next1 = kb_st + 256 - static_cast<int>((b1 + kb_st) & 255);
      }
      // A wait that gives up (it never should) ends the warp's loop on every
      // lane together, so the warp-collective MMAs below always see 32 lanes.
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full_bar[s], ph, p.err, kErrTimeoutFullA));
      if (!ok) break;
      const uint32_t tile = ring + s * kSlotBytes;
      const uint32_t xtile = tile + kStageBytes;
      // A whole stage inside K and inside one group per row needs no
      // per-block checks (the checks are scalar; every lane runs the same
      // MMAs either way).
      const bool fast = full && next0 >= kb_st + kStageBlocks && next1 >= kb_st + kStageBlocks;
#pragma unroll
      for (int b = 0; b < kStageBlocks; ++b) {
        const uint2 c0 = lds64(tile + off0[b]);
        const uint2 c1 = lds64(tile + off1[b]);
        // X of the block (zero past K, where its slice was not loaded).
        uint4 xa[TOK_TILES], xb[TOK_TILES];
#pragma unroll
        for (int t = 0; t < TOK_TILES; ++t) {
          xa[t] = qv[b] ? lds128(xtile + b * kXBlockBytes + xoff[t][0]) : make_uint4(0u, 0u, 0u, 0u);
          xb[t] = qv[b] ? lds128(xtile + b * kXBlockBytes + xoff[t][1]) : make_uint4(0u, 0u, 0u, 0u);
        }
        float bacc[TOK_TILES][4];
        block_mma<TOK_TILES>(bacc, c0, c1, xa, xb, lut, lane4);
        if (!fast) {
          const int kb = kb_st + b;
          if (kb == next0 && kb < kblocks) {
            t0 = group_constant(__ldg(p.group_scale + ((b0 + kb) >> 8)), fp8);
            next0 += 256;
          }
          if (kb == next1 && kb < kblocks) {
            t1 = group_constant(__ldg(p.group_scale + ((b1 + kb) >> 8)), fp8);
            next1 += 256;
          }
        }
        // c' of the block (zero past K, where the block adds nothing).
        const float s0 = qv[b] ? __fadd_rn(__fmul_rn(qf0[b], t0), mu) : 0.f;
        const float s1 = qv[b] ? __fadd_rn(__fmul_rn(qf1[b], t1), mu) : 0.f;
#pragma unroll
        for (int t = 0; t < TOK_TILES; ++t) {
          acc[t][0] = fmaf(s0, bacc[t][0], acc[t][0]);
          acc[t][1] = fmaf(s0, bacc[t][1], acc[t][1]);
          acc[t][2] = fmaf(s1, bacc[t][2], acc[t][2]);
          acc[t][3] = fmaf(s1, bacc[t][3], acc[t][3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }
  }
  // Every stage is consumed and every copy has landed (the producer drained
  // its ring): the partial sums may now overwrite it.
  __syncthreads();
  if (warp < kConsumers) {
    // Partial sums: rows lr0/lr1, tokens 2q, 2q+1 (+8t); red is [token][row].
#pragma unroll
    for (int t = 0; t < TOK_TILES; ++t) {
      const int tok = 8 * t + 2 * q;
      red[tok * kRows + lr0] = acc[t][0];
      red[(tok + 1) * kRows + lr0] = acc[t][1];
      red[tok * kRows + lr1] = acc[t][2];
      red[(tok + 1) * kRows + lr1] = acc[t][3];
    }
  }
  __syncthreads();
  cluster_sync_all();

  // Adapter intermediate T is written by the preceding kernel (a no-op when
  // this grid was not launched as its programmatic dependent).
  if (p.r > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  // CTA `crank` of the cluster finishes rows [r_lo, r_hi) of the tile.
  const int r_lo = static_cast<int>((static_cast<uint32_t>(kRows) * crank) / csize);
  const int r_hi = static_cast<int>((static_cast<uint32_t>(kRows) * (crank + 1)) / csize);
  const int rpr = r_hi - r_lo;
  for (int i = threadIdx.x; i < p.m * rpr; i += kThreads) {
    const int mi = i / rpr;
    const int nl = r_lo + (i % rpr);
    const int64_t n = n_cta + nl;
    if (n >= p.n) continue;
    const uint32_t off = red_addr + static_cast<uint32_t>(mi * kRows + nl) * 4u;
    // Every peer's partial is requested before the first add (a cluster has
    // at most 8 CTAs); the adds run in peer order.
    float part[8];
#pragma unroll
    for (uint32_t peer = 0; peer < 8; ++peer) part[peer] = peer < csize ? ld_dsmem_f32(off, peer) : 0.f;
    float sum = 0.f;
#pragma unroll
    for (uint32_t peer = 0; peer < 8; ++peer)
      if (peer < csize) sum += part[peer];
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
          sum = fmaf(bf16lo_to_f32(ta[e]), bf16lo_to_f32(ba[e]), sum);
          sum = fmaf(bf16hi_to_f32(ta[e]), bf16hi_to_f32(ba[e]), sum);
        }
      }
    }
    p.Y[static_cast<int64_t>(mi) * p.n + n] = static_cast<uint16_t>(pack_bf16x2(sum, 0.f) & 0xFFFFu);
  }
  cluster_sync_all();
}

// T[m x r] = bf16(scale * X . A^T): one CTA per adapter row j, 1024 threads
// so that K up to 8192 is one pass (the kernel sits on the critical path of a
// decode call: the main kernel's CTAs cannot share an SM with it).
constexpr int kProjThreads = 1024;
__global__ void __launch_bounds__(kProjThreads) lora_proj_small_kernel(const uint16_t *__restrict__ X, int m,
                                                              int64_t k, const uint16_t *__restrict__ A,
                                                              int r, float scale,
                                                              uint16_t *__restrict__ T) {
  __shared__ float red[kProjThreads / 32][kMaxM];
  // The weight-streaming kernel that consumes T may start now; it waits for
  // this grid's completion before its epilogue reads T.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int j = blockIdx.x;
  const uint16_t *arow = A + static_cast<int64_t>(j) * k;
  float acc[kMaxM];
#pragma unroll
  for (int i = 0; i < kMaxM; ++i) acc[i] = 0.f;
  for (int64_t kk = static_cast<int64_t>(threadIdx.x) * 8; kk < k; kk += kProjThreads * 8) {
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
    for (int w = 0; w < kProjThreads / 32; ++w) s += red[w][threadIdx.x];
    T[static_cast<int64_t>(threadIdx.x) * r + j] = static_cast<uint16_t>(pack_bf16x2(s * scale, 0.f) & 0xFFFFu);
  }
}

}  // namespace

cudaError_t launch_lora_proj_small(const uint16_t *X, int64_t m, int64_t k, const uint16_t *A,
                                   int32_t r, float scale, uint16_t *T, cudaStream_t stream) {
  if (m <= 0 || r <= 0) return cudaSuccess;
  lora_proj_small_kernel<<<r, kProjThreads, 0, stream>>>(X, static_cast<int>(m), k, A, r, scale, T);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_gemv_fwd(const uint16_t *X, int64_t m, const uint8_t *codes, const uint8_t *absmax_q,
                            const float *group_scale, const float *mu, int64_t n, int64_t k, const uint16_t *T,
                            const uint16_t *B, int32_t r, uint16_t *Y, const Nf4Tables &tab,
                            cudaStream_t stream, bool pdl) {
  if (m <= 0) return cudaSuccess;
  GemvParams p{};
  if (!encode_codes_map(&p.tmCodes, codes, n, k / 2, 128, kRows, true)) return cudaErrorInvalidValue;
  // X boxes of 64 columns and 8 (m <= 8) or 16 token rows; rows past m read
  // as zero.
  const uint32_t x_rows = m <= 8 ? 8u : 16u;
  if (!encode_bf16_map(&p.tmX, X, m, k, 64, x_rows)) return cudaErrorInvalidValue;
  p.x_box_bytes = 128u * x_rows;
  p.X = X;
  p.absmax_q = absmax_q;
  p.group_scale = group_scale;
  p.mu = mu;
  p.T = T;
  p.B = B;
  p.Y = Y;
  p.err = device_error_word();
  p.n = n;
  p.k = k;
  p.m = static_cast<int>(m);
  p.r = (T != nullptr && B != nullptr) ? r : 0;
  p.tab = tab;

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<bool> configured1[kMaxDevicesPerProcess] = {}, configured2[kMaxDevicesPerProcess] = {};
  const int variant = m <= 8 ? 0 : 1;
  {
    const cudaError_t e =
        variant == 0 ? set_smem_once(reinterpret_cast<const void *>(gemv_fwd_kernel<1>), static_cast<int>(kSmemBytes),
                                     configured1)
                     : set_smem_once(reinterpret_cast<const void *>(gemv_fwd_kernel<2>), static_cast<int>(kSmemBytes),
                                     configured2);
    if (e != cudaSuccess) return e;
  }
  // Split K over a cluster of cs CTAs: the smallest cs in 1..8 that puts a
  // CTA on every SM, keeping at least two stages of K per CTA.  Each CTA
  // pays for its table, its ring fill and a cluster reduction, so splitting
  // further (to fill both CTA slots of every SM, or whole waves) costs more
  // than the idle slots do.
  const int64_t row_ctas = (n + kRows - 1) / kRows;
  const int64_t kblocks = k / 64;
  int cs = 1;
  while (cs < 8 && row_ctas * cs < sms && (kblocks / kStageBlocks) / (cs + 1) >= 2) ++cs;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(row_ctas), static_cast<unsigned>(cs), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (p.r > 0 && pdl) ? 2 : 1;
  const cudaError_t e = variant == 0 ? cudaLaunchKernelEx(&cfg, gemv_fwd_kernel<1>, p)
                                     : cudaLaunchKernelEx(&cfg, gemv_fwd_kernel<2>, p);
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace qlora
