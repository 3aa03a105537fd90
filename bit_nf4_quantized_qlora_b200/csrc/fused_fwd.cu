// Fused NF4 forward for large M: Y = bf16(X . W^T + T . B^T), one 256 x 256
// output tile per CTA, tcgen05 MMAs with the fp32 accumulator in TMEM.
//
// "QLoRA and Quantized Training", The idea: each block is dequantized, used in
// the multiply and discarded; "A 65B fine-tune on the GPU you already have",
// figure 2: dequantized to bf16 only long enough to multiply.  The weight
// exists in bf16 only as a 128-byte-swizzled shared-memory tile that dequant
// warps write and the MMA reads.
//
// Rings and roles:
//   stage ring (3 x 64 KB)  X tile [256 x 64] by TMA (the adapter T tile on
//                           the extra k-steps) + the bf16 weight tile [256 x 64]
//                           written by the dequant warps (the adapter's B tile,
//                           on the extra k-steps, by plain loads)
//   code rings (2 x 2 x 8 KB) packed codes [256 rows x 32 B] of a k-step, one
//                           ring per dequant group
//   warp 0 producer (X and code copies), warp 1 TMEM allocation + MMA issuer,
//   warps 2..17 two groups of 8 dequant warps taking k-steps in turn (thread =
//   one weight row = one NF4 block per k-step), then the epilogue.
// The producer issues a k-step's codes only after the stage that step will use
// has been released by the MMAs, so a group that sees its codes arrive knows
// its weight slot is free.  Every barrier is waited on by its consumers use
// after use (each group waits only on its own code ring), so a parity wait
// can never be satisfied by an older phase.  Every wait is bounded in time (a
// flag in the device error word on expiry); no kernel traps.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace qlora {
namespace {

constexpr int kBM = 256, kBN = 256, kBK = 64;
constexpr int kStages = 3;
constexpr int kGroups = 2, kGroupWarps = 8, kCodeSlots = 2;   // per group
constexpr uint32_t kASub = 128u * kBK * 2u;          // one 128-row A sub-tile (16 KB)
constexpr uint32_t kABytes = 2u * kASub;
constexpr uint32_t kBBytes = static_cast<uint32_t>(kBN) * kBK * 2u;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kCBytes = static_cast<uint32_t>(kBN) * 32u;
constexpr uint32_t kCOff = kStages * kStageBytes;
constexpr uint32_t kSmemBytes = kCOff + kGroups * kCodeSlots * kCBytes + 1024u;
constexpr int kThreads = 32 * (2 + kGroups * kGroupWarps);
constexpr uint32_t kTmemCols = 512;                   // two 128 x 256 fp32 accumulators
constexpr uint32_t kIdesc = make_idesc(kBN, false, false);
static_assert(kSmemBytes <= 227u * 1024u, "shared memory");

struct __align__(64) FwdParams {
  CUtensorMap tmA;       // X [m x k] bf16, box {64, 128}, 128B swizzle
  CUtensorMap tmCodes;   // codes [n x k/2] bytes, box {32, 256}
  CUtensorMap tmA2;      // T [m x r] bf16, box {64, 128}, 128B swizzle
  const uint16_t *B2;    // adapter B [n x r] bf16
  const uint8_t *absmax_q;
  const float *group_scale;
  uint16_t *out;         // Y [m x n]
  unsigned *err;
  int64_t n, k;
  int m, r;
  int num_main, num_lora;
  int pdl;
  Nf4Tables tab;
};

__global__ void __launch_bounds__(kThreads, 1) fused_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_a[kStages], full_b[kStages], empty[kStages];
  __shared__ __align__(8) uint64_t c_full[kGroups][kCodeSlots], c_empty[kGroups][kCodeSlots];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_slot;

  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y;
  const int total = p.num_main + p.num_lora;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_a[s], 1);
      mbar_init(&full_b[s], kGroupWarps);
      mbar_init(&empty[s], 1);
    }
    for (int g = 0; g < kGroups; ++g)
      for (int c = 0; c < kCodeSlots; ++c) {
        mbar_init(&c_full[g][c], 1);
        mbar_init(&c_empty[g][c], kGroupWarps);
      }
    mbar_init(&acc_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmCodes);
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % kStages;
        if (!mbar_wait_bounded(&empty[s], (static_cast<uint32_t>(it / kStages) & 1u) ^ 1u, p.err, kErrTimeoutEmpty))
          break;
        const uint32_t a_s = base + static_cast<uint32_t>(s) * kStageBytes;
        const bool lora = it >= p.num_main;
        // The adapter operand T comes from the preceding projection kernel.
        if (lora && it == p.num_main && p.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
        mbar_arrive_expect_tx(&full_a[s], kABytes);
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tma_load_2d(a_s + h * kASub, lora ? &p.tmA2 : &p.tmA, &full_a[s], (lora ? it - p.num_main : it) * kBK,
                      m_tile * kBM + h * 128);
        // The step's codes (or, on an adapter step, a bare arrival) go to the
        // group that takes it, now that the step's weight slot is free.
        const int g = it % kGroups, gi = it / kGroups, cs = gi % kCodeSlots;
        if (!mbar_wait_bounded(&c_empty[g][cs], (static_cast<uint32_t>(gi / kCodeSlots) & 1u) ^ 1u, p.err,
                               kErrTimeoutEmpty))
          break;
        if (!lora) {
          mbar_arrive_expect_tx(&c_full[g][cs], kCBytes);
          tma_load_2d(base + kCOff + static_cast<uint32_t>(g * kCodeSlots + cs) * kCBytes, &p.tmCodes, &c_full[g][cs],
                      it * 32, n_tile * kBN);
        } else {
          mbar_arrive(&c_full[g][cs]);
        }
        ++issued;
      }
      // Let the last copies land before the CTA may exit.
      for (int it = issued - kStages < 0 ? 0 : issued - kStages; it < issued; ++it)
        mbar_wait_bounded(&full_a[it % kStages], static_cast<uint32_t>(it / kStages) & 1u, p.err, kErrTimeoutDrain);
      for (int it = issued - kGroups * kCodeSlots < 0 ? 0 : issued - kGroups * kCodeSlots; it < issued; ++it) {
        const int g = it % kGroups, gi = it / kGroups;
        mbar_wait_bounded(&c_full[g][gi % kCodeSlots], static_cast<uint32_t>(gi / kCodeSlots) & 1u, p.err,
                          kErrTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int it = 0; it < total && ok; ++it) {
        const int s = it % kStages;
        const uint32_t ph = static_cast<uint32_t>(it / kStages) & 1u;
        ok = mbar_wait_bounded(&full_a[s], ph, p.err, kErrTimeoutFullA) &&
             mbar_wait_bounded(&full_b[s], ph, p.err, kErrTimeoutFullB);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_s = base + static_cast<uint32_t>(s) * kStageBytes;
        const uint32_t b_s = a_s + kABytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc(a_s + h * kASub + kk * 32u, 16u, 1024u);
            const uint64_t bd = smem_desc(b_s + kk * 32u, 16u, 1024u);
            umma_f16(tmem + static_cast<uint32_t>(h * kBN), ad, bd, kIdesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(&acc_bar);
    }
  } else {
    // ------------------------------------------------------------ dequant
    const int grp = (warp - 2) / kGroupWarps;
    const int dt = (threadIdx.x - 64) & (32 * kGroupWarps - 1);   // weight row of the tile
    const int64_t kblocks = p.k / 64;
    const int64_t gn = static_cast<int64_t>(n_tile) * kBN + dt;
    const bool row_ok = gn < p.n;
    const uint32_t row_off = static_cast<uint32_t>(dt) * 128u;
    const uint32_t sw = static_cast<uint32_t>(dt & 7);
    const uint32_t first_half = ((lane >> 2) & 1u) ? 16u : 0u;
    // Absmax code and group scale of this group's next k-step, fetched one
    // step of the group ahead; t = fp32(S / 255) recomputed only when the
    // group index changes (a thread walks one weight row).
    uint32_t q_nx = (row_ok && grp < p.num_main) ? __ldg(p.absmax_q + gn * kblocks + grp) : 0u;
    float S_nx = (row_ok && grp < p.num_main) ? __ldg(p.group_scale + ((gn * kblocks + grp) >> 8)) : 0.f;
    int64_t g_cur = -1;
    float t_cur = 0.f;
    for (int it = grp; it < total; it += kGroups) {
      const int gi = it / kGroups, cs = gi % kCodeSlots;
      if (!mbar_wait_bounded(&c_full[grp][cs], static_cast<uint32_t>(gi / kCodeSlots) & 1u, p.err, kErrTimeoutFullA))
        break;
      const uint32_t b_s = base + static_cast<uint32_t>(it % kStages) * kStageBytes + kABytes;
      const uint32_t rowaddr = b_s + row_off;
      if (it < p.num_main) {
        const uint32_t c_s = base + kCOff + static_cast<uint32_t>(grp * kCodeSlots + cs) * kCBytes;
        const uint4 f = lds128(c_s + static_cast<uint32_t>(dt) * 32u + first_half);
        const uint4 g2 = lds128(c_s + static_cast<uint32_t>(dt) * 32u + (16u - first_half));
        // The codes are in registers: release the code slot.
        __syncwarp();
        if (lane == 0) mbar_arrive(&c_empty[grp][cs]);
        const uint32_t qv = q_nx;
        const float S = S_nx;
        const int64_t blk = gn * kblocks + it;
        if (it + kGroups < p.num_main && row_ok) {
          q_nx = __ldg(p.absmax_q + blk + kGroups);
          S_nx = __ldg(p.group_scale + ((blk + kGroups) >> 8));
        }
        Bf16Table tb;
        if (row_ok) {
          const int64_t gidx = blk >> 8;
          if (gidx != g_cur) {
            g_cur = gidx;
            t_cur = __fdiv_rn(S, 255.0f);
          }
          make_table(p.tab, __fmul_rn(static_cast<float>(qv), t_cur), tb);
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) tb.lo[j] = tb.hi[j] = 0u;
        }
        const uint4 lo = first_half ? g2 : f, hi = first_half ? f : g2;
        const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[4];
          decode8(words[c], tb, o);
          sts128(rowaddr + ((static_cast<uint32_t>(c) ^ sw) << 4), o);
        }
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&c_empty[grp][cs]);
        // Adapter k-step: row gn of B (r columns), columns [64 l, 64 l + 64).
        // B is an input of the preceding kernel, not its output: no wait.
        const int l = it - p.num_main;
        const uint16_t *src = p.B2 + gn * p.r + static_cast<int64_t>(l) * kBK;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (row_ok && l * kBK + 8 * c < p.r) v = __ldg(reinterpret_cast<const uint4 *>(src) + c);
          const uint32_t o[4] = {v.x, v.y, v.z, v.w};
          sts128(rowaddr + ((static_cast<uint32_t>(c) ^ sw) << 4), o);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_b[it % kStages]);
    }

    // ------------------------------------------------------------ epilogue
    if (mbar_wait_bounded(&acc_bar, 0u, p.err, kErrTimeoutAcc, 20000000000ull)) {
      tc_fence_after();
      const int ew = warp - 2;
      const int quad = warp & 3;                      // TMEM lanes this warp may read
      const int h = ew >> 3;
      const int c_begin = ((ew >> 2) & 1) * (kBN / 2);
      const int64_t grow = static_cast<int64_t>(m_tile) * kBM + h * 128 + quad * 32 + lane;
      const bool out_ok = grow < p.m;
      for (int c0 = c_begin; c0 < c_begin + kBN / 2; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(h * kBN + c0), v);
        const int64_t gcol = static_cast<int64_t>(n_tile) * kBN + c0;
        if (!out_ok) continue;
        uint16_t *dst = p.out + grow * p.n + gcol;
        if (gcol + 32 <= p.n) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
            w.y = pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
            w.z = pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
            w.w = pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
            reinterpret_cast<uint4 *>(dst)[j] = w;
          }
        } else {
          for (int j = 0; j < 32; ++j)
            if (gcol + j < p.n) dst[j] = static_cast<uint16_t>(pack_bf16x2(__uint_as_float(v[j]), 0.f) & 0xFFFFu);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t fused_fwd_large(const uint16_t *X, int64_t m, const WeightView &w, const uint16_t *T, const uint16_t *B,
                            int32_t r, uint16_t *Y, cudaStream_t stream, bool pdl) {
  FwdParams p{};
  const bool lora = T != nullptr && B != nullptr && r > 0;
  if (!encode_bf16_map(&p.tmA, X, m, w.k, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_codes_map(&p.tmCodes, w.codes, w.n, w.k / 2, 32, kBN, false)) return cudaErrorInvalidValue;
  if (lora && !encode_bf16_map(&p.tmA2, T, m, r, 64, 128)) return cudaErrorInvalidValue;
  p.B2 = B;
  p.absmax_q = w.absmax_q;
  p.group_scale = w.group_scale;
  p.out = Y;
  p.err = device_error_word();
  p.n = w.n;
  p.k = w.k;
  p.m = static_cast<int>(m);
  p.r = lora ? r : 0;
  p.num_main = static_cast<int>(w.k / kBK);
  p.num_lora = lora ? (r + kBK - 1) / kBK : 0;
  p.pdl = (lora && pdl) ? 1 : 0;
  p.tab = *w.tab;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool configured[64] = {};
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(fused_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>((w.n + kBN - 1) / kBN), static_cast<unsigned>((m + kBM - 1) / kBM), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, fused_fwd_kernel, p);
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace qlora
