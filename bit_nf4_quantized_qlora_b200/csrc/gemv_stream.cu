// Decode-sized forward (M <= 4): Y = bf16(X . W^T + T . B^T), streaming the
// packed weights from HBM at close to copy bandwidth.
//
// At decode M the layer reads each packed weight once and does a couple of
// FLOPs with it ("QLoRA and Quantized Training", The idea: dequantize each
// block, multiply, discard), so the kernel is built around the load-store
// unit, which every byte of codes passes through twice (once arriving, once
// as a table lookup):
//
//   * Memory side.  A CTA owns a run of 16-row tiles; its 16 warps split K in
//     chunks of 4 NF4 blocks (128 bytes of a row), so at any moment a CTA
//     reads 16 rows x 2 KB of contiguous bytes.  Each warp streams its own
//     chunk of successive tiles through a private 3-slot ring: one lane issues
//     a TMA copy of the 16 x 128-byte box (plus the 16 x 16-byte box of absmax
//     codes around it) on the slot's mbarrier.  No CTA-wide barriers, no
//     producer warp; TMA writes bypass the load-store pipe, and the 128-byte
//     swizzle with a row order that pairs rows r and r+4 in each quarter-warp
//     makes the 16-byte reads conflict-free.
//   * Expansion.  A 64 KB shared table maps every code byte (two weights) to
//     the bf16 pair {NF4[hi], NF4[lo]} (32 lane-private copies, so lookups
//     never conflict); the pairs are the A operand of m16n8k16 tensor-core
//     MMAs whose B operand is X, kept in registers for the whole kernel.
//   * Absmax scaling after the MMA.  A lane's 16 bytes are half of one NF4
//     block, so the four lanes of an MMA row group cover two blocks.  The
//     block is carried in the MMA's N dimension: column 2t holds token t on
//     the lanes holding the first block of the pair, column 2t+1 token t on
//     the lanes holding the second.  One MMA chain gives both blocks' raw sums
//     side by side and each is scaled by its own c' = q * fp32(S/255) in fp32
//     (fp32(S/255) is tabulated per group once per CTA, and applied once per
//     row and chunk when the chunk lies in one group).  Columns are spare at
//     M <= 4.
//   * K split.  Chunks beyond one CTA's 16 warps go to the other CTAs of a
//     thread-block cluster; warps add their per-tile partial sums into a
//     shared buffer, the cluster reduces it through distributed shared memory,
//     and the adapter term T . B^T is added before Y is written once in bf16.
//     T comes from the preceding projection kernel, which this kernel
//     overlaps (programmatic dependent launch) and waits for only before its
//     epilogue.
#include <cuda.h>

#include <type_traits>
#include <utility>

#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxM = 4;                 // two N columns per token in one n8 MMA
constexpr int kTileRows = 32;            // weight rows per tile: two m16n8k16 row tiles
constexpr int kSub = kTileRows / 16;
constexpr int kMaxTiles = 16;            // tiles per CTA held in the reduction buffer
constexpr int kMaxCluster = 8;
constexpr int kMaxKBlocks = kMaxCluster * kWarps * 4;
constexpr int kStages = 2;                // ring slots per warp (one in flight while one is read)
constexpr uint32_t kCodeSlot = kTileRows * 128u;   // tile rows x 4 blocks of codes
constexpr uint32_t kQSlot = kTileRows * 16u;       // tile rows x 16 absmax codes
constexpr uint32_t kRedBytes = kMaxTiles * kTileRows * kMaxM * 4u;
constexpr uint32_t kMaxGroups = (kMaxTiles * kTileRows * kMaxKBlocks) / 256u + 2u;
constexpr uint32_t kTabBytes = (kMaxGroups * 4u + 1023u) & ~1023u;
constexpr uint32_t kRingOff = kPairLutBytes + kRedBytes + kTabBytes;          // 1024-aligned
constexpr uint32_t kQRingOff = kRingOff + kWarps * kStages * kCodeSlot;
constexpr uint32_t kBarOff = kQRingOff + kWarps * kStages * kQSlot;
constexpr uint32_t kSmemBytes = kBarOff + kWarps * kStages * 8u + 1024u;   // + base alignment slack
static_assert(kRingOff % 1024u == 0, "128-byte swizzled boxes need 1024-byte alignment");
static_assert(kSmemBytes <= 227u * 1024u, "shared memory");

// MODE 2: k/64 % 16 == 0 (absmax codes by TMA, one group per chunk);
// MODE 1: k/64 % 4 == 0 (absmax codes as words, one group per chunk);
// MODE 0: any k/64 (byte loads, a group may change inside a chunk).
struct __align__(64) StreamParams {
  CUtensorMap tmCodes;           // codes [n x k/2] bytes, box {128, tile rows}, 128B swizzle
  CUtensorMap tmQ;               // absmax codes [n x k/64] bytes, box {16, tile rows} (MODE 2)
  const uint8_t *absmax_q;       // [n x k/64]
  const float *group_scale;      // [ceil(n k / 16384)] (+ the tensor mean, E4M3 + mean format)
  const float *mu;               // E4M3 + mean format: the tensor mean; else null
  const uint16_t *X;             // [m x k] bf16
  const uint16_t *T;             // [m x r] bf16 (adapter intermediate) or null
  const uint16_t *B;             // [n x r] bf16
  uint16_t *Y;                   // [m x n] bf16
  unsigned *err;
  int64_t n, k;
  int m, r;
  int ntiles;                    // ceil(n / tile rows)
  int chunks;                    // ceil((k / 64) / 4)
  int chunks_per_cta;            // chunks owned by one CTA of a cluster (<= 16)
  Nf4Tables tab;
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// On lanes with `pred` set: expect `bytes` on the slot's mbarrier and start
// the TMA copy of the codes box (and, if qmap is non-zero, of the absmax-code
// box) into the slot.  Predicated rather than branched: every lane runs it.
__device__ __forceinline__ void issue_unit(uint32_t pred, uint32_t bar, uint32_t bytes, uint32_t dst, uint64_t map,
                                           int x, uint32_t qdst, uint64_t qmap, int qx, int y) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %0, 0;\n\t"
      "@p fence.proxy.async.shared::cta;\n\t"
      "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %2;\n\t"
      "@p cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%3], [%4, {%5, %9}], [%1];\n\t"
      "}" ::"r"(pred), "r"(bar), "r"(bytes), "r"(dst), "l"(map), "r"(x), "r"(qdst), "l"(qmap), "r"(qx), "r"(y)
      : "memory");
  if (qmap != 0)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.u32 p, %0, 0;\n\t"
        "@p cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%2], [%3, {%4, %5}], [%1];\n\t"
        "}" ::"r"(pred), "r"(bar), "r"(qdst), "l"(qmap), "r"(qx), "r"(y)
        : "memory");
}

__device__ __forceinline__ uint32_t try_wait_u32(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok;
}

// Adds a and b at addr and addr + 32 bytes when pred is set.
__device__ __forceinline__ void red_pair(uint32_t pred, uint32_t addr, float a, float b) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %0, 0;\n\t"
      "@p red.shared.add.f32 [%1], %2;\n\t"
      "@p red.shared.add.f32 [%1+32], %3;\n\t}" ::"r"(pred), "r"(addr), "f"(a), "f"(b)
      : "memory");
}

// Two k-steps from one 32-bit word of each of the rows g and g+8 (8 weights
// each): byte 0 -> a0/a1, byte 1 -> a2/a3, then bytes 2 and 3.  xv holds the
// matching 8 activations of this lane's column.  FIRST starts the chain from
// a zero accumulator.
template <bool FIRST>
__device__ __forceinline__ void word_mma(float (&d)[4], uint32_t w_g, uint32_t w_g8, const uint8_t *lut, uint32_t lane4,
                                         const uint4 &xv) {
  const auto L = [&](uint32_t off) { return *reinterpret_cast<const uint32_t *>(lut + off); };
  const uint32_t a0 = L(pair_lut_off<0>(w_g, lane4)), a1 = L(pair_lut_off<0>(w_g8, lane4));
  const uint32_t a2 = L(pair_lut_off<1>(w_g, lane4)), a3 = L(pair_lut_off<1>(w_g8, lane4));
  if (FIRST)
    mma_bf16_16816_zero(d, a0, a1, a2, a3, xv.x, xv.y);
  else
    mma_bf16_16816(d, a0, a1, a2, a3, xv.x, xv.y);
  mma_bf16_16816(d, L(pair_lut_off<2>(w_g, lane4)), L(pair_lut_off<2>(w_g8, lane4)), L(pair_lut_off<3>(w_g, lane4)),
                 L(pair_lut_off<3>(w_g8, lane4)), xv.z, xv.w);
}

template <class F, int... S>
__device__ __forceinline__ bool slot_pass(const F &f, uint32_t ph, std::integer_sequence<int, S...>) {
  return f(ph, std::integral_constant<int, S>{}...);
}

// FP8: the absmax codes are E4M3 offsets from the tensor mean (p.mu).
template <int MODE, bool FP8>
__global__ void __launch_bounds__(kThreads, 1) gemv_stream_kernel(const __grid_constant__ StreamParams p) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  const uint8_t *lut = dsmem;
  float *red = reinterpret_cast<float *>(dsmem + kPairLutBytes);
  float *ttab = reinterpret_cast<float *>(dsmem + kPairLutBytes + kRedBytes);
  // Ring offsets are taken from a 1024-aligned base (the 128-byte swizzle
  // pattern is defined on 1024-byte atoms of shared memory).
  const uint32_t sbase = smem_u32(dsmem);
  const uint32_t abase = (sbase + 1023u) & ~1023u;
  const uint32_t ring = abase + kRingOff;
  const uint32_t qring = abase + kQRingOff;
  const uint32_t bars = abase + kBarOff;

  const uint32_t crank = cluster_rank();
  const uint32_t csize = cluster_size();
  // The warp index read through a shuffle is known to be warp-uniform, so
  // everything derived from it (ring, barrier and TMA operands) can live in
  // uniform registers.
  const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int ncl = static_cast<int>(gridDim.y);
  const int cl = static_cast<int>(blockIdx.y);
  const int t_lo = static_cast<int>((static_cast<int64_t>(p.ntiles) * cl) / ncl);
  const int t_hi = static_cast<int>((static_cast<int64_t>(p.ntiles) * (cl + 1)) / ncl);
  const int nt = t_hi - t_lo;
  const int kblocks = static_cast<int>(p.k >> 6);

  // Warp -> (chunk, tile phase): with fewer chunks than warps, several warps
  // take the same chunk on interleaved tiles.
  const int cpc = p.chunks_per_cta;
  const int phases = kWarps / cpc;
  const int phase = warp / cpc;
  const int chunk = static_cast<int>(crank) * cpc + warp % cpc;
  const bool active = phase < phases && chunk < p.chunks;
  const int kb0 = chunk * 4;
  const int nvalid = min(4, kblocks - kb0);
  const int nunits = active && nt > phase ? (nt - phase + phases - 1) / phases : 0;
  const uint32_t tx_bytes = kCodeSlot + (MODE == 2 ? kQSlot : 0u);
  const uint64_t map_codes = reinterpret_cast<uint64_t>(&p.tmCodes);
  const uint64_t map_q = MODE == 2 ? reinterpret_cast<uint64_t>(&p.tmQ) : 0ull;
  const uint32_t bar_w = bars + warp * kStages * 8u;                     // slot s: + 8 s
  const uint32_t ring_w = ring + warp * kStages * kCodeSlot;              // slot s: + s kCodeSlot
  const uint32_t qring_w = qring + warp * kStages * kQSlot;               // slot s: + s kQSlot
  const int y_step = kTileRows * phases;
  // Each warp's ring starts filling before the tables are built.
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_w + s * 8u));
    fence_mbar_init();
  }
  __syncwarp();
  for (int s = 0; s < kStages && s < nunits; ++s)
    issue_unit(lane == 0, bar_w + s * 8u, tx_bytes, ring_w + s * kCodeSlot, map_codes, kb0 * 32,
               qring_w + s * kQSlot, map_q, kb0 & ~15, (t_lo + phase) * kTileRows + s * y_step);

  // B operand (X): column g = 2 * token + block parity; lanes whose piece is
  // in the other block of the pair, and tokens >= m, hold zeros.  Loaded
  // before the tables are built so that the load latency overlaps them.
  const int tok = g >> 1;
  const bool live = active && (g & 1) == (q >> 1) && tok < p.m;
  uint4 xf[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool v = live && (MODE != 0 || 2 * i + (q >> 1) < nvalid);
    const uint4 *xp = reinterpret_cast<const uint4 *>(p.X + static_cast<int64_t>(v ? tok : 0) * p.k +
                                                      (v ? kb0 * 64 + 64 * (2 * i + (q >> 1)) + 32 * (q & 1) : 0));
#pragma unroll
    for (int j = 0; j < 4; ++j) xf[i][j] = v ? __ldg(xp + j) : make_uint4(0u, 0u, 0u, 0u);
  }

  // The group constant t (fp32(S / 255) for linear codes) of every group
  // the CTA's rows touch.  Rows of the last
  // tile past n (codes and absmax codes read as zero) index the table too;
  // their entries repeat the last group.  Row * k/64 fits in 32 bits
  // (checked on the host).  The first group scale of each thread is loaded
  // before the pair table is built.
  const int gbase = (t_lo * kTileRows * kblocks) >> 8;
  const int ngroups = ((t_hi * kTileRows * kblocks - 1) >> 8) - gbase + 1;
  const int glast = static_cast<int>((p.n * kblocks - 1) >> 8);
  const float s_first = static_cast<int>(threadIdx.x) < ngroups
                            ? __ldg(p.group_scale + min(gbase + static_cast<int>(threadIdx.x), glast))
                            : 0.f;
  build_pair_lut(dsmem, p.tab, threadIdx.x, kThreads);
  for (int i = threadIdx.x; i < nt * kTileRows * kMaxM; i += kThreads) red[i] = 0.f;
  const auto gconst = [](float stored) { return FP8 ? stored : div255_rn(stored); };
  if (static_cast<int>(threadIdx.x) < ngroups) ttab[threadIdx.x] = gconst(s_first);
  for (int i = threadIdx.x + kThreads; i < ngroups; i += kThreads)
    ttab[i] = gconst(__ldg(p.group_scale + min(gbase + i, glast)));
  const float mu = FP8 ? __ldg(p.mu) : 0.f;
  __syncthreads();

  if (active) {
    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    // MMA row group g reads physical rows pr and pr + 8 of the tile, with pr
    // pairing rows r and r + 4 in each quarter-warp: the two rows' swizzle
    // phases then differ in the chunk index's top bit.
    const int pr = (g >> 1) + 4 * (g & 1);
    const uint32_t off_r0_p0 = static_cast<uint32_t>(pr) * 128u + ((static_cast<uint32_t>(q) ^ pr) << 4);
    const uint32_t off_r0_p1 = static_cast<uint32_t>(pr) * 128u + ((static_cast<uint32_t>(4 + q) ^ pr) << 4);
    const uint32_t off_r1_p0 = off_r0_p0 + 8u * 128u;
    const uint32_t off_r1_p1 = off_r0_p1 + 8u * 128u;

    const uint32_t tab_w = smem_u32(ttab) - 4u * static_cast<uint32_t>(gbase);
    const uint32_t qoff = static_cast<uint32_t>(pr) * 16u + (kb0 & 15);
    const uint32_t red_pred = q < p.m ? 1u : 0u;
    // Loop state: rk = row * k/64 + kb0 for row pr of the current tile;
    // y_refill is the first row of the unit kStages ahead.
    int rk0 = ((t_lo + phase) * kTileRows + pr) * kblocks + kb0;
    const int rk_step = kTileRows * phases * kblocks, rk_8 = 8 * kblocks;
    int y_refill = (t_lo + phase) * kTileRows + kStages * y_step;
    const int y_end = t_hi * kTileRows;
    uint32_t red_addr = smem_u32(red) + 4u * static_cast<uint32_t>((phase * kMaxM + q) * kTileRows + pr);
    const uint32_t red_step = 4u * static_cast<uint32_t>(phases * kMaxM * kTileRows);
    const int nm1 = static_cast<int>(p.n) - 1;
    int u = phase;

    // One unit (this warp's chunk of one tile) from ring slot S; false when
    // the warp is done or a wait gave up.  Row pair j of the lane is rows
    // pr + 8j of the tile (j = 0 .. 2 kSub - 1); sub-tile st holds pairs
    // 2st and 2st + 1 and is one m16n8k16 row tile.
    const auto unit = [&](auto s_const, uint32_t ph) -> bool {
      constexpr int S = decltype(s_const)::value;
      if (u >= nt) return false;
      uint32_t qw[2 * kSub];
      float tlo[2 * kSub], thi[2 * kSub];
      int split[2 * kSub];
#pragma unroll
      for (int j = 0; j < 2 * kSub; ++j) {
        const int rk = rk0 + j * rk_8;
        tlo[j] = __uint_as_float(lds32(tab_w + 4u * static_cast<uint32_t>(rk >> 8)));
        thi[j] = tlo[j];
        split[j] = 4;   // blocks of the chunk before the row's next group
        qw[j] = 0;
        if (MODE != 2) {
          // Absmax codes by plain loads, from rows clamped to the matrix.
          const int64_t bq = static_cast<int64_t>(min((t_lo + u) * kTileRows + pr + 8 * j, nm1)) * kblocks + kb0;
          if (MODE == 1) {
            qw[j] = __ldg(reinterpret_cast<const uint32_t *>(p.absmax_q + bq));
          } else {
            for (int b = 0; b < nvalid; ++b) qw[j] |= static_cast<uint32_t>(__ldg(p.absmax_q + bq + b)) << (8 * b);
            thi[j] = __uint_as_float(lds32(tab_w + 4u * static_cast<uint32_t>((rk + nvalid - 1) >> 8)));
            split[j] = 256 - (rk & 255);
          }
        }
      }
      // A wait that gives up (it never should) ends the warp's loop on every
      // lane together.
      const uint32_t bar = bar_w + S * 8u;
      if (__any_sync(0xffffffffu, try_wait_u32(bar, ph) == 0u)) {
        uint64_t *barp = reinterpret_cast<uint64_t *>(dsmem + (bar - sbase));
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(barp, ph, p.err, kErrTimeoutFullA))) return false;
      }
      const uint32_t slot = ring_w + S * kCodeSlot;
      uint4 c[kSub][4];   // [sub-tile][row g piece 0, row g piece 1, row g+8 piece 0, row g+8 piece 1]
#pragma unroll
      for (int st = 0; st < kSub; ++st) {
        c[st][0] = lds128(slot + st * 2048u + off_r0_p0);
        c[st][1] = lds128(slot + st * 2048u + off_r0_p1);
        c[st][2] = lds128(slot + st * 2048u + off_r1_p0);
        c[st][3] = lds128(slot + st * 2048u + off_r1_p1);
      }
      if (MODE == 2) {
#pragma unroll
        for (int j = 0; j < 2 * kSub; ++j) qw[j] = lds32(qring_w + S * kQSlot + qoff + 128u * j);
      }
      float acc[2 * kSub], dsum[2 * kSub];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float d[kSub][4];
#pragma unroll
        for (int st = 0; st < kSub; ++st) {
          const uint4 cg = c[st][i], cg8 = c[st][2 + i];
          word_mma<true>(d[st], cg.x, cg8.x, lut, lane4, xf[i][0]);
          word_mma<false>(d[st], cg.y, cg8.y, lut, lane4, xf[i][1]);
          word_mma<false>(d[st], cg.z, cg8.z, lut, lane4, xf[i][2]);
          word_mma<false>(d[st], cg.w, cg8.w, lut, lane4, xf[i][3]);
        }
        // d[st][0], d[st][1]: row pair 2st (row pr + 16 st), token q, blocks
        // 2i and 2i+1; d[st][2], d[st][3]: row pair 2st + 1 (8 rows below).
#pragma unroll
        for (int j = 0; j < 2 * kSub; ++j) {
          const float da = d[j >> 1][2 * (j & 1)], db = d[j >> 1][2 * (j & 1) + 1];
          float qa, qb;
          if (FP8) {
            qa = e4m3_to_f32((qw[j] >> (16 * i)) & 0xFFu);
            qb = e4m3_to_f32((qw[j] >> (16 * i + 8)) & 0xFFu);
          } else {
            qa = i == 0 ? byte_to_f32<0>(qw[j]) : byte_to_f32<2>(qw[j]);
            qb = i == 0 ? byte_to_f32<1>(qw[j]) : byte_to_f32<3>(qw[j]);
          }
          if (MODE != 0) {
            // One group per chunk: t is common to the four blocks and is
            // applied once per row below, the mean term (E4M3 + mean) as
            // mu times the sum of the raw block products.
            acc[j] = i == 0 ? qa * da : fmaf(qa, da, acc[j]);
            acc[j] = fmaf(qb, db, acc[j]);
            if (FP8) dsum[j] = i == 0 ? da + db : dsum[j] + da + db;
          } else {
            const float ta = 2 * i < split[j] ? tlo[j] : thi[j], tb = 2 * i + 1 < split[j] ? tlo[j] : thi[j];
            const float ca = FP8 ? __fadd_rn(__fmul_rn(qa, ta), mu) : __fmul_rn(qa, ta);
            const float cb = FP8 ? __fadd_rn(__fmul_rn(qb, tb), mu) : __fmul_rn(qb, tb);
            acc[j] = i == 0 ? ca * da : fmaf(ca, da, acc[j]);
            acc[j] = fmaf(cb, db, acc[j]);
          }
        }
      }
      if (MODE != 0) {
#pragma unroll
        for (int j = 0; j < 2 * kSub; ++j) acc[j] = FP8 ? fmaf(dsum[j], mu, acc[j] * tlo[j]) : acc[j] * tlo[j];
      }
      // The slot's bytes are consumed: refill it with the unit kStages ahead.
      __syncwarp();
      issue_unit(lane == 0 && y_refill < y_end, bar, tx_bytes, slot, map_codes, kb0 * 32, qring_w + S * kQSlot,
                 map_q, kb0 & ~15, y_refill);
#pragma unroll
      for (int st = 0; st < kSub; ++st) red_pair(red_pred, red_addr + 64u * st, acc[2 * st], acc[2 * st + 1]);
      y_refill += y_step;
      red_addr += red_step;
      rk0 += rk_step;
      u += phases;
      return true;
    };

    // The ring is walked slot by slot with compile-time slot indices; the
    // mbarrier phase flips after every pass over the ring.
    int j = 0;
    const auto pass = [&](uint32_t ph, auto... s) { return ((unit(s, ph) && (++j, true)) && ...); };
    for (uint32_t ph = 0;; ph ^= 1u)
      if (!slot_pass(pass, ph, std::make_integer_sequence<int, kStages>{})) break;
    const bool ok = u >= nt;
    if (!ok && lane == 0) {
      // A wait gave up: let copies still in flight land before the CTA's
      // memory is released.
      for (int jj = j; jj < j + kStages && jj < nunits; ++jj) {
        uint64_t *b = reinterpret_cast<uint64_t *>(dsmem + (bar_w - sbase) + (jj % kStages) * 8u);
        mbar_wait_bounded(b, static_cast<uint32_t>(jj / kStages) & 1u, p.err, kErrTimeoutDrain);
      }
    }
  }
  __syncthreads();
  cluster_sync_all();

  // The adapter intermediate T is written by the preceding kernel (a no-op
  // when this grid was not launched as its programmatic dependent).
  if (p.r > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
  // CTA `crank` finishes its share of the cluster's (tile, token, row) sums.
  const int total = nt * p.m * kTileRows;
  const int o_lo = static_cast<int>((static_cast<int64_t>(total) * crank) / csize);
  const int o_hi = static_cast<int>((static_cast<int64_t>(total) * (crank + 1)) / csize);
  const uint32_t red_addr = smem_u32(red);
  for (int o = o_lo + static_cast<int>(threadIdx.x); o < o_hi; o += kThreads) {
    const int ut = o / (p.m * kTileRows);
    const int rem = o - ut * p.m * kTileRows;
    const int mi = rem / kTileRows, rl = rem % kTileRows;
    const int64_t n = static_cast<int64_t>(t_lo + ut) * kTileRows + rl;
    if (n >= p.n) continue;
    const uint32_t off = red_addr + static_cast<uint32_t>((ut * kMaxM + mi) * kTileRows + rl) * 4u;
    // Every peer's partial is requested before the first add; the adds run
    // in peer order.
    float part[kMaxCluster];
#pragma unroll
    for (uint32_t peer = 0; peer < kMaxCluster; ++peer) part[peer] = peer < csize ? ld_dsmem_f32(off, peer) : 0.f;
    float sum = 0.f;
#pragma unroll
    for (uint32_t peer = 0; peer < kMaxCluster; ++peer)
      if (peer < csize) sum += part[peer];
    if (p.r > 0) {
      const uint16_t *trow = p.T + static_cast<int64_t>(mi) * p.r;
      const uint16_t *brow = p.B + n * p.r;
      for (int jr = 0; jr < p.r; jr += 8) {
        const uint4 tv = *reinterpret_cast<const uint4 *>(trow + jr);
        const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(brow + jr));
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

template <int MODE, bool FP8>
cudaError_t configure(int dev) {
  static std::atomic<bool> done[kMaxDevicesPerProcess] = {};
  if (dev < 0 || dev >= kMaxDevicesPerProcess) return cudaErrorInvalidDevice;
  return set_smem_once(reinterpret_cast<const void *>(gemv_stream_kernel<MODE, FP8>), static_cast<int>(kSmemBytes),
                       &done[dev]);
}

template <int MODE, bool FP8>
cudaError_t launch_mode(const StreamParams &p, int dev, int sms, int cs, cudaStream_t stream, bool pdl) {
  cudaError_t e = configure<MODE, FP8>(dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(cs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // One CTA per SM: as many clusters as can be resident at once (the GPC
  // layout may hold fewer than sms / cs), each with a contiguous run of at
  // most kMaxTiles tiles.
  static std::atomic<int> resident[kMaxDevicesPerProcess][2][kMaxCluster + 1] = {};
  if (dev >= kMaxDevicesPerProcess) return cudaErrorInvalidDevice;
  int res = resident[dev][FP8 ? 1 : 0][cs].load(std::memory_order_relaxed);
  if (res == 0) {
    int v = 0;
    e = cudaOccupancyMaxActiveClusters(&v, gemv_stream_kernel<MODE, FP8>, &cfg);
    if (e != cudaSuccess) return e;
    res = v > 0 ? v : (sms / cs > 0 ? sms / cs : 1);
    resident[dev][FP8 ? 1 : 0][cs].store(res, std::memory_order_relaxed);
  }
  int ncl = res < p.ntiles ? res : p.ntiles;
  const int min_ncl = (p.ntiles + kMaxTiles - 1) / kMaxTiles;
  if (ncl < min_ncl) ncl = min_ncl;
  cfg.gridDim = dim3(static_cast<unsigned>(cs), static_cast<unsigned>(ncl), 1);
  cfg.numAttrs = (p.r > 0 && pdl) ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemv_stream_kernel<MODE, FP8>, p);
}

}  // namespace

bool gemv_stream_supported(int64_t m, int64_t n, int64_t k) {
  // Row * k/64 indices (rows padded to whole tiles) are kept in 32 bits.
  return m >= 1 && m <= kMaxM && k / 64 <= kMaxKBlocks && (n + kTileRows) * (k / 64) < (int64_t(1) << 31);
}

cudaError_t launch_gemv_stream(const uint16_t *X, int64_t m, const uint8_t *codes, const uint8_t *absmax_q,
                               const float *group_scale, const float *mu, int64_t n, int64_t k, const uint16_t *T,
                               const uint16_t *B, int32_t r, uint16_t *Y, const Nf4Tables &tab,
                               cudaStream_t stream, bool pdl) {
  if (m <= 0) return cudaSuccess;
  if (!gemv_stream_supported(m, n, k)) return cudaErrorInvalidValue;
  const int64_t kblocks = k / 64;
  const int mode = kblocks % 16 == 0 ? 2 : (kblocks % 4 == 0 ? 1 : 0);
  StreamParams p{};
  if (!encode_codes_map(&p.tmCodes, codes, n, k / 2, 128, kTileRows, true)) return cudaErrorInvalidValue;
  if (mode == 2 && !encode_codes_map(&p.tmQ, absmax_q, n, kblocks, 16, kTileRows, false)) return cudaErrorInvalidValue;
  p.absmax_q = absmax_q;
  p.group_scale = group_scale;
  p.mu = mu;
  p.X = X;
  p.T = T;
  p.B = B;
  p.Y = Y;
  p.err = device_error_word();
  p.n = n;
  p.k = k;
  p.m = static_cast<int>(m);
  p.r = (T != nullptr && B != nullptr) ? r : 0;
  p.ntiles = static_cast<int>((n + kTileRows - 1) / kTileRows);
  p.chunks = static_cast<int>((kblocks + 3) / 4);
  const int cs = (p.chunks + kWarps - 1) / kWarps;
  p.chunks_per_cta = (p.chunks + cs - 1) / cs;
  p.tab = tab;

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool fp8 = mu != nullptr;
  const cudaError_t e =
      mode == 2   ? (fp8 ? launch_mode<2, true>(p, dev, sms, cs, stream, pdl) : launch_mode<2, false>(p, dev, sms, cs, stream, pdl))
      : mode == 1 ? (fp8 ? launch_mode<1, true>(p, dev, sms, cs, stream, pdl) : launch_mode<1, false>(p, dev, sms, cs, stream, pdl))
                  : (fp8 ? launch_mode<0, true>(p, dev, sms, cs, stream, pdl) : launch_mode<0, false>(p, dev, sms, cs, stream, pdl));
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace qlora
