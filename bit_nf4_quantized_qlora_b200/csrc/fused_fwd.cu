// Fused NF4 forward for large M: Y = bf16(X . W^T + T . B^T), computed by CTA
// pairs.  Each pair of CTAs (a cluster of two) owns a 512 x 256 output tile;
// its MMAs are tcgen05 pair MMAs (M = 256 over the two CTAs, N = 256) with the
// fp32 accumulators in the two CTAs' tensor memory.
//
// "QLoRA and Quantized Training", The idea: each block is dequantized, used in
// the multiply and discarded; "A 65B fine-tune on the GPU you already have",
// figure 2: dequantized to bf16 only long enough to multiply.  The weight
// exists in bf16 only as a 128-byte-swizzled shared-memory tile that dequant
// warps write and the MMA reads.
//
// Why pairs: a pair MMA reads the N columns of its B operand half from each
// CTA, so each CTA expands only 128 of the tile's 256 weight rows per k-step
// while its tensor core still does the work of a 256 x 256 x 64 step.  That
// halves the dequant instructions per FLOP and the shared-memory bytes the
// tensor core reads per FLOP against a one-CTA tile of the same size.
//
// Per CTA (rank c of the pair; rows m0 = 512 p + 256 c of X, weight rows
// n0 + 128 c .. + 128 of the pair's tile n0):
//   stage ring, 4 x 52 KB  X rows [256 x 64] as two 128-row TMA boxes (the
//                          adapter T on the extra k-steps), the bf16 weight
//                          tile [128 x 64] (dequant warps; the adapter's B
//                          rows by TMA on the extra k-steps) and the packed
//                          codes [128 rows x 32 B] of the k-step
//   warp 0   producer: X / T boxes with pair TMA counted on the leader's
//            xfull barrier, codes with a local TMA on this CTA's cfull
//   warp 1   tensor-memory allocation (both CTAs, 512 columns); in the
//            leader CTA also the single thread that issues the pair MMAs
//   warps 2..17  four groups of four dequant warps; group g expands the
//            k-steps of stage g (one weight row = one NF4 block per thread)
//            and arrives on the leader's wfull barrier; then the epilogue.
// Barriers per stage: xfull (leader; X bytes of both CTAs), cfull (each CTA;
// its codes), wfull (leader; 8 arrivals, the 4 + 4 dequant warps), empty
// (each CTA; one arrival from the leader's multicast commit when the stage's
// MMAs are done).  Every barrier is waited on by each of its waiters at every
// phase (with four stages and four groups, group g owns stage g), so no parity
// wait can be satisfied by an older phase.  Every wait is bounded in time (a
// flag in the device error word on expiry); no kernel traps.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace qlora {
namespace {

constexpr int kRowsCta = 256;                   // X rows per CTA (two 128-row MMA halves)
constexpr int kBN = 256;                        // weight rows per pair tile
constexpr int kWRows = kBN / 2;                 // weight rows expanded per CTA
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kGroups = 4, kGroupWarps = 4;     // dequant: group g owns stage g
constexpr uint32_t kASub = 128u * kBK * 2u;     // 16 KB: 128 X rows of a k-step
constexpr uint32_t kABytes = 2u * kASub;
constexpr uint32_t kBBytes = static_cast<uint32_t>(kWRows) * kBK * 2u;   // 16 KB
constexpr uint32_t kCBytes = static_cast<uint32_t>(kWRows) * 32u;        // 4 KB
constexpr uint32_t kBOff = kABytes, kCOff = kABytes + kBBytes;
constexpr uint32_t kStageBytes = kABytes + kBBytes + kCBytes;            // 52 KB
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024u;
constexpr int kThreads = 32 * (2 + kGroups * kGroupWarps);
constexpr uint32_t kTmemCols = 512;             // two 128 x 256 fp32 accumulators per CTA
constexpr uint32_t kIdesc = make_idesc(kBN, false, false, 256);
static_assert(kStages == kGroups, "each dequant group owns one stage");
static_assert(kStageBytes % 1024u == 0, "1024-byte aligned operand tiles");
static_assert(kSmemBytes <= 227u * 1024u, "shared memory");

struct __align__(64) FwdParams {
  CUtensorMap tmA;       // X [m x k] bf16, box {64, 128}, 128B swizzle
  CUtensorMap tmCodes;   // codes [n x k/2] bytes, box {32, 128}
  CUtensorMap tmA2;      // T [m x r] bf16, box {64, 128}, 128B swizzle
  CUtensorMap tmB2;      // adapter B [n x r] bf16, box {64, 128}, 128B swizzle
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
  __shared__ __align__(8) uint64_t xfull[kStages], cfull[kStages], wfull[kStages], empty[kStages];
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ uint32_t tmem_slot;

  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int m_pair = static_cast<int>(blockIdx.x >> 1), n_tile = static_cast<int>(blockIdx.y);
  const int m0 = m_pair * (2 * kRowsCta) + static_cast<int>(rank) * kRowsCta;
  const int64_t w0 = static_cast<int64_t>(n_tile) * kBN + static_cast<int64_t>(rank) * kWRows;
  const int total = p.num_main + p.num_lora;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&cfull[s], 1);
      mbar_init(&wfull[s], 2 * kGroupWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmCodes);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers are initialised before either CTA counts bytes or
  // arrivals on the other's.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % kStages;
        const uint32_t use = static_cast<uint32_t>(it / kStages);
        if (!mbar_wait_bounded(&empty[s], (use & 1u) ^ 1u, p.err, kErrTimeoutEmpty)) break;
        const uint32_t st = base + static_cast<uint32_t>(s) * kStageBytes;
        const bool lora = it >= p.num_main;
        // The adapter operand T comes from the preceding projection kernel.
        if (lora && it == p.num_main && p.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint32_t xbar = mapa_shared(smem_u32(&xfull[s]), 0);
        if (leader) mbar_arrive_expect_tx(&xfull[s], 2u * (kABytes + (lora ? kBBytes : 0u)));
        const int kx = (lora ? it - p.num_main : it) * kBK;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // A 128-row half entirely past m loads rows 0..127 instead: its
          // accumulator rows are never stored, and every box stays in range.
          const int y = (m0 + h * 128 < p.m) ? m0 + h * 128 : 0;
          tma_load_2d_pair(st + h * kASub, lora ? &p.tmA2 : &p.tmA, xbar, kx, y);
        }
        const int wy = (w0 < p.n) ? static_cast<int>(w0) : 0;
        if (lora) {
          tma_load_2d_pair(st + kBOff, &p.tmB2, xbar, kx, wy);
          mbar_arrive(&cfull[s]);
        } else {
          mbar_arrive_expect_tx(&cfull[s], kCBytes);
          tma_load_2d(st + kCOff, &p.tmCodes, &cfull[s], it * 32, wy);
        }
        ++issued;
      }
      // Let this CTA's last copies land before it may exit (the leader's
      // xfull also counts the peer's X boxes).
      for (int it = issued - kStages < 0 ? 0 : issued - kStages; it < issued; ++it) {
        const uint32_t ph = static_cast<uint32_t>(it / kStages) & 1u;
        if (leader) mbar_wait_bounded(&xfull[it % kStages], ph, p.err, kErrTimeoutDrain);
        mbar_wait_bounded(&cfull[it % kStages], ph, p.err, kErrTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      bool ok = true;
      for (int it = 0; it < total && ok; ++it) {
        const int s = it % kStages;
        const uint32_t ph = static_cast<uint32_t>(it / kStages) & 1u;
        ok = mbar_wait_cluster_bounded(&xfull[s], ph, p.err, kErrTimeoutFullA) &&
             mbar_wait_cluster_bounded(&wfull[s], ph, p.err, kErrTimeoutFullB);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = base + static_cast<uint32_t>(s) * kStageBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc(st + h * kASub + kk * 32u, 16u, 1024u);
            const uint64_t bd = smem_desc(st + kBOff + kk * 32u, 16u, 1024u);
            umma_f16_pair(tmem + static_cast<uint32_t>(h * kBN), ad, bd, kIdesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit_pair_both(&empty[s]);
      }
      if (ok) umma_commit_pair_both(&acc_full);
    }
  } else {
    // ------------------------------------------------------------ dequant
    const int dq = warp - 2;
    const int grp = dq / kGroupWarps;                     // == the stage this group fills
    const int dt = (dq % kGroupWarps) * 32 + lane;        // weight row of this CTA's half tile
    const int64_t kblocks = p.k / 64;
    const int64_t gn = w0 + dt;
    const bool row_ok = gn < p.n;
    const uint32_t row_off = static_cast<uint32_t>(dt) * 128u;
    const uint32_t sw = static_cast<uint32_t>(dt & 7);
    const uint32_t first_half = ((lane >> 2) & 1u) ? 16u : 0u;
    const uint32_t wbar = mapa_shared(smem_u32(&wfull[grp]), 0);
    // Absmax code and group scale of this group's next k-step, fetched one
    // step of the group ahead; t = fp32(S / 255) recomputed only when the
    // group index changes (a thread walks one weight row).
    uint32_t q_nx = (row_ok && grp < p.num_main) ? __ldg(p.absmax_q + gn * kblocks + grp) : 0u;
    float S_nx = (row_ok && grp < p.num_main) ? __ldg(p.group_scale + ((gn * kblocks + grp) >> 8)) : 0.f;
    int64_t g_cur = -1;
    float t_cur = 0.f;
    for (int it = grp; it < total; it += kGroups) {
      const uint32_t use = static_cast<uint32_t>(it / kStages);
      if (!mbar_wait_bounded(&cfull[grp], use & 1u, p.err, kErrTimeoutFullA)) break;
      const uint32_t st = base + static_cast<uint32_t>(grp) * kStageBytes;
      if (it < p.num_main) {
        const uint32_t c_s = st + kCOff + static_cast<uint32_t>(dt) * 32u;
        const uint4 f = lds128(c_s + first_half);
        const uint4 g2 = lds128(c_s + (16u - first_half));
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
        const uint32_t rowaddr = st + kBOff + row_off;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[4];
          decode8(words[c], tb, o);
          sts128(rowaddr + ((static_cast<uint32_t>(c) ^ sw) << 4), o);
        }
        fence_proxy_async_smem();
      }
      // Adapter k-steps: the B rows came by TMA; the arrival keeps the
      // barrier's phases in step.
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(wbar);
    }

    // ------------------------------------------------------------ epilogue
    if (mbar_wait_bounded(&acc_full, 0u, p.err, kErrTimeoutAcc, 20000000000ull)) {
      tc_fence_after();
      const int quad = warp & 3;                          // TMEM lanes this warp may read
      const int q4 = dq >> 2;                             // column quarter of the 512 columns
      const int h = q4 >> 1;
      const int c_begin = (q4 & 1) * (kBN / 2);
      const int64_t grow = static_cast<int64_t>(m0) + h * 128 + quad * 32 + lane;
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

  // Neither CTA leaves (or frees tensor memory) while the other may still
  // count on its barriers or its tensor memory.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t fused_fwd_large(const uint16_t *X, int64_t m, const WeightView &w, const uint16_t *T, const uint16_t *B,
                            int32_t r, uint16_t *Y, cudaStream_t stream, bool pdl) {
  FwdParams p{};
  const bool lora = T != nullptr && B != nullptr && r > 0;
  if (!encode_bf16_map(&p.tmA, X, m, w.k, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_codes_map(&p.tmCodes, w.codes, w.n, w.k / 2, 32, kWRows, false)) return cudaErrorInvalidValue;
  if (lora) {
    if (!encode_bf16_map(&p.tmA2, T, m, r, 64, 128)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&p.tmB2, B, w.n, r, 64, kWRows)) return cudaErrorInvalidValue;
  }
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

  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(fused_fwd_kernel), static_cast<int>(kSmemBytes),
                                configured);
  if (e != cudaSuccess) return e;
  const int64_t pairs_m = (m + 2 * kRowsCta - 1) / (2 * kRowsCta);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs_m), static_cast<unsigned>((w.n + kBN - 1) / kBN), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.pdl ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, fused_fwd_kernel, p);
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace qlora
