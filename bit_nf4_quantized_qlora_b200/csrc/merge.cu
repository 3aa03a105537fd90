// Adapter merge: W' = W^ + s . B . A, exported as bf16 and/or fp32.
//
// "QLoRA", Training setup versus deployment setup and Common misconception:
// the adapter folds back into the frozen weight; the only base a quantized
// checkpoint has is W^ = bf16(fp32(L[code] * c')).  W' is formed in fp32 with
// one fused multiply-add, W^ + s * acc, acc the fp32 sum of the rank-r
// product, and rounded once to bf16 for the bf16 export.
//
// One CTA per output tile of 128 rows x 256 columns.  One thread stages the
// tile's operands by TMA, 128-byte swizzled: the tile's 128 rows of B (K-major,
// 64 ranks per slab; ranks past r read as zero), the 64 x 256 slice of A
// (MN-major, four 64-column slabs) and the tile's packed codes (128 rows x
// 128 bytes); it issues the tcgen05 MMAs of B . A into a 128 x 256 fp32
// accumulator in tensor memory (r > 64 walks 64-rank slabs through the same
// buffers).  Eight epilogue warps then each own 32 accumulator rows (the
// tensor-memory lane quarter of their warp) and one half of the columns:
// a thread reads its row's accumulator 32 columns at a time with
// tcgen05.ld, decodes the row's NF4 block through one bf16 table of the
// block's 16 scaled levels (byte permutes, no per-element lookups), forms
// W' = fma(s, acc, W^) in fp32 and writes the row into a 128-byte-swizzled
// staging tile, which one thread of the half stores with TMA.  The floor is
// HBM on the output writes (2 or 4 bytes per weight against 0.52 read).
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace qlora {
namespace {

constexpr int kTM = 128, kTN = 256;               // tile rows x columns
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;     // warp 0: TMA + MMA, warp 1: tensor memory, 2..9: epilogue
constexpr int kMaxR = 256;
constexpr uint32_t kBSlab = kTM * 128u;           // 16 KB: 128 rows of B x 64 ranks
constexpr uint32_t kASlab = 4u * 8192u;           // 32 KB: 64 ranks x 256 columns of A (four 64-column slabs)
constexpr uint32_t kCodeTile = kTM * 128u;        // 16 KB: 128 rows x 4 blocks of codes
constexpr uint32_t kStage = kTM * 128u;           // 16 KB: one staged box per half of the epilogue
constexpr uint32_t kOffB = 0, kOffA = kBSlab, kOffCodes = kOffA + kASlab, kOffStage = kOffCodes + kCodeTile;
constexpr uint32_t kTmemCols = kTN;
constexpr uint32_t kIdesc = make_idesc(kTN, false, true);

struct __align__(64) MergeParams {
  CUtensorMap tmB;        // B [n x r] bf16, box {64, 128}
  CUtensorMap tmA;        // A [r x k] bf16, box {64, 64}
  CUtensorMap tmCodes;    // codes [n x k/2] bytes, box {128, 128}
  CUtensorMap tmOutH;     // W' bf16 [n x k], box {64, 128}
  CUtensorMap tmOutF;     // W' fp32 [n x k], box {32, 128}
  const uint8_t *absmax_q;
  const float *group_scale;
  const float *mu;        // E4M3 + mean absmax format: the tensor mean; else null
  unsigned *err;
  int64_t n, k;
  int r;
  int out_h, out_f;       // which exports are written
  float scale;
  Nf4Tables tab;
};

// AND of v over the `count` threads that take barrier `id` (a multiple of 32).
__device__ __forceinline__ bool barrier_and(uint32_t id, uint32_t count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kThreads, 2) merge_kernel(const __grid_constant__ MergeParams p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t codes_bar;   // the codes tile landed (one phase)
  __shared__ __align__(8) uint64_t full_bar;    // a slab of B and A landed (one phase per slab)
  __shared__ __align__(8) uint64_t mma_bar;     // a slab's MMAs finished reading (one phase per slab but the last)
  __shared__ __align__(8) uint64_t acc_bar;     // the accumulator is complete (one phase)
  __shared__ uint32_t tmem_slot;

  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTM;   // first row of the tile
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTN;   // first column
  const int nslabs = (p.r + 63) / 64;

  if (threadIdx.x == 0) {
    mbar_init(&codes_bar, 1);
    mbar_init(&full_bar, 1);
    mbar_init(&mma_bar, 1);
    mbar_init(&acc_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&codes_bar, kCodeTile);
      tma_load_2d(base + kOffCodes, &p.tmCodes, &codes_bar, static_cast<int>(c0 / 2), static_cast<int>(r0));
      for (int j = 0; j < nslabs; ++j) {
        // The buffers are free once the previous slab's MMAs have read them.
        if (j > 0 && !mbar_wait_bounded(&mma_bar, static_cast<uint32_t>(j - 1) & 1u, p.err, kErrTimeoutEmpty)) break;
        mbar_arrive_expect_tx(&full_bar, kBSlab + kASlab);
        tma_load_2d(base + kOffB, &p.tmB, &full_bar, 64 * j, static_cast<int>(r0));
#pragma unroll
        for (int s = 0; s < 4; ++s)
          tma_load_2d(base + kOffA + 8192u * s, &p.tmA, &full_bar, static_cast<int>(c0) + 64 * s, 64 * j);
        if (!mbar_wait_bounded(&full_bar, static_cast<uint32_t>(j) & 1u, p.err, kErrTimeoutFullA)) {
          // Let the copies in flight land before the CTA's memory is released.
          mbar_wait_bounded(&full_bar, static_cast<uint32_t>(j) & 1u, p.err, kErrTimeoutDrain);
          break;
        }
        tc_fence_after();
        const int ksteps = (p.r - 64 * j) / 16 < 4 ? (p.r - 64 * j) / 16 : 4;   // r is a multiple of 16
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint64_t ad = smem_desc(base + kOffB + 32u * kk, 16u, 1024u);
          const uint64_t bd = smem_desc(base + kOffA + 2048u * kk, 8192u, 1024u);
          umma_f16(tmem, ad, bd, kIdesc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(j + 1 < nslabs ? &mma_bar : &acc_bar);
      }
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;                // tensor-memory lanes 32 quad .. 32 quad + 31
    const int half = ew >> 2;                 // blocks 2 half and 2 half + 1 of the tile
    const int row = quad * 32 + lane;         // tile row of this thread
    const int64_t grow = r0 + row;
    const bool leader = (ew & 3) == 0 && lane == 0;
    const uint32_t bar_id = 1u + static_cast<uint32_t>(half);
    const uint32_t stage_h = base + kOffStage + static_cast<uint32_t>(half) * kStage;
    const uint32_t stage_f = base + kOffStage + (p.out_h ? 2u * kStage : 0u) + static_cast<uint32_t>(half) * kStage;
    const uint32_t sw = static_cast<uint32_t>(row & 7);
    const bool fp8 = p.mu != nullptr;
    const float mu = load_mu(p.mu);
    // W' = fma(s, acc, W^).  Without an adapter the sum is -0 and s is 1,
    // which returns W^ exactly (-0 + x = x for every x, FP4's -0 level
    // included).
    const float s_eff = p.r > 0 ? p.scale : 1.f;
    // c' of the thread's two blocks, requested before the waits.
    float cp[2];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
      const int64_t gcol = c0 + 64 * (2 * half + bb);
      cp[bb] = 0.f;
      if (grow < p.n && gcol < p.k) {
        const int64_t blk = (grow * p.k + gcol) / 64;
        const float sg = __ldg(p.group_scale + (blk >> 8));
        cp[bb] = block_constant(__ldg(p.absmax_q + blk), fp8 ? sg : div255_rn(sg), fp8, mu);
      }
    }
    bool ok = mbar_wait_bounded(&codes_bar, 0u, p.err, kErrTimeoutFullB);
    if (ok && p.r > 0) ok = mbar_wait_bounded(&acc_bar, 0u, p.err, kErrTimeoutAcc);
    // Every epilogue thread takes the same path (the halves' barriers and the
    // warp-collective tensor-memory loads below need all of them).
    ok = barrier_and(3u, 32u * kEpiWarps, ok);
    tc_fence_after();
    // A staging buffer of this half is rewritten only after the stores that
    // read it have finished reading, and stored once all 128 rows are in.
    const auto stage_free = [&]() {
      if (leader) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      named_barrier_sync(bar_id, 128);
    };
    const auto stage_store = [&](const CUtensorMap *map, uint32_t src, int64_t x) {
      fence_proxy_async_smem();
      named_barrier_sync(bar_id, 128);
      if (leader) {
        tma_store_2d(map, src, static_cast<int>(x), static_cast<int>(r0));
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    };
    if (ok) {
#pragma unroll 1
      for (int bb = 0; bb < 2; ++bb) {
        const int blk = 2 * half + bb;
        Bf16Table tb;
        make_table(p.tab, cp[bb], tb);
        const uint32_t crow = base + kOffCodes + static_cast<uint32_t>(row) * 128u;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // 32 columns: the accumulator, the codes (16 bytes) and W^.
          uint32_t v[32];
          if (p.r > 0) {
            tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(64 * blk + 32 * hh), v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0x80000000u;   // -0
          }
          const uint4 cw = lds128(crow + ((static_cast<uint32_t>(2 * blk + hh) ^ sw) << 4));
          uint32_t wv[16];
          decode8(cw.x, tb, wv + 0);
          decode8(cw.y, tb, wv + 4);
          decode8(cw.z, tb, wv + 8);
          decode8(cw.w, tb, wv + 12);
          float m[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            m[2 * i] = __fmaf_rn(s_eff, __uint_as_float(v[2 * i]), bf16lo_to_f32(wv[i]));
            m[2 * i + 1] = __fmaf_rn(s_eff, __uint_as_float(v[2 * i + 1]), bf16hi_to_f32(wv[i]));
          }
          if (p.out_h) {
            // The previous block's store must have read the buffer; the wait
            // comes after this block's first 32 columns are computed, so it
            // overlaps them.
            if (hh == 0) stage_free();
            // Row `row` of the [128 x 64] bf16 box: 16-byte chunks 4 hh .. 4 hh + 3.
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint32_t w4[4] = {pack_bf16x2(m[8 * c + 0], m[8 * c + 1]), pack_bf16x2(m[8 * c + 2], m[8 * c + 3]),
                                      pack_bf16x2(m[8 * c + 4], m[8 * c + 5]), pack_bf16x2(m[8 * c + 6], m[8 * c + 7])};
              sts128(stage_h + static_cast<uint32_t>(row) * 128u + ((static_cast<uint32_t>(4 * hh + c) ^ sw) << 4), w4);
            }
          }
          if (p.out_f) {
            // Row `row` of the [128 x 32] fp32 box of these 32 columns.
            stage_free();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t w4[4] = {__float_as_uint(m[4 * c + 0]), __float_as_uint(m[4 * c + 1]),
                                      __float_as_uint(m[4 * c + 2]), __float_as_uint(m[4 * c + 3])};
              sts128(stage_f + static_cast<uint32_t>(row) * 128u + ((static_cast<uint32_t>(c) ^ sw) << 4), w4);
            }
            stage_store(&p.tmOutF, stage_f, c0 + 64 * blk + 32 * hh);
          }
        }
        if (p.out_h) stage_store(&p.tmOutH, stage_h, c0 + 64 * blk);
      }
    }
    if (leader) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t launch_merge(const WeightView &w, const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                         uint16_t *out_bf16, float *out_f32, cudaStream_t stream) {
  if (r < 0 || r > kMaxR || r % 16 != 0) return cudaErrorInvalidValue;
  if (w.n <= 0 || w.k <= 0 || (out_bf16 == nullptr && out_f32 == nullptr)) return cudaSuccess;
  MergeParams p{};
  if (r > 0) {
    if (!encode_bf16_map(&p.tmB, B, w.n, r, 64, kTM)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&p.tmA, A, r, w.k, 64, 64)) return cudaErrorInvalidValue;
  }
  if (!encode_codes_map(&p.tmCodes, w.codes, w.n, w.k / 2, 128, kTM, true)) return cudaErrorInvalidValue;
  if (out_bf16 && !encode_bf16_map(&p.tmOutH, out_bf16, w.n, w.k, 64, kTM)) return cudaErrorInvalidValue;
  if (out_f32 && !encode_f32_map(&p.tmOutF, out_f32, w.n, w.k, 32, kTM)) return cudaErrorInvalidValue;
  p.absmax_q = w.absmax_q;
  p.group_scale = w.group_scale;
  p.mu = w.mu;
  p.err = device_error_word();
  p.n = w.n;
  p.k = w.k;
  p.r = r;
  p.out_h = out_bf16 ? 1 : 0;
  p.out_f = out_f32 ? 1 : 0;
  p.scale = scale;
  p.tab = *w.tab;
  const uint32_t smem = kOffStage + (out_bf16 ? 2u * kStage : 0u) + (out_f32 ? 2u * kStage : 0u) + 1024u;
  // The limit is raised once per device to the most any call uses.
  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(merge_kernel),
                                static_cast<int>(kOffStage + 4u * kStage + 1024u), configured);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((w.k + kTN - 1) / kTN), static_cast<unsigned>((w.n + kTM - 1) / kTM), 1);
  merge_kernel<<<grid, kThreads, smem, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
