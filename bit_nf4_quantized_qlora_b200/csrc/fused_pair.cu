// Fused NF4 products for large M on CTA pairs:
//   forward          Y  = bf16(X . W^T + T . B^T)     (weight rows are MMA N)
//   input gradient   dX = bf16(dY . W^ + U . A)       (weight columns are MMA N)
// Each pair of CTAs (a cluster of two) owns a 512 x 256 output tile; its MMAs
// are tcgen05 pair MMAs (M = 256 over the two CTAs, N = 256) with the fp32
// accumulators in the two CTAs' tensor memory.
//
// "QLoRA and Quantized Training", The idea: each block is dequantized, used in
// the multiply and discarded; "A 65B fine-tune on the GPU you already have",
// figure 2: dequantized to bf16 only long enough to multiply; "QLoRA", Follow
// one QLoRA training step, step 4: the input gradient flows through the same
// frozen weight.  The weight exists in bf16 only as a 128-byte-swizzled
// shared-memory tile that dequant warps write and the MMA reads.
//
// Why pairs: a pair MMA reads the N columns of its B operand half from each
// CTA, so each CTA expands only 128 of the tile's 256 weight rows (forward)
// or columns (input gradient) per k-step while its tensor core still does the
// work of a 256 x 256 x 64 step.  That halves the dequant instructions per
// FLOP and the shared-memory bytes the tensor core reads per FLOP against a
// one-CTA tile of the same size.
//
// The weight tile of a k-step holds 128 NF4 blocks per CTA, one per dequant
// thread.  Forward: the tile is K-major, [128 weight rows x 64] (one block
// per row).  Input gradient: the contraction runs over weight rows, so the
// tile is MN-major, two 64-column slabs of [64 weight rows x 64] (each
// 128-byte row of a slab is one block).  The same expansion writes both.
//
// Per CTA (rank c of the pair; activation rows m0 = 512 p + 256 c, output
// columns n0 + 128 c .. + 128 of the pair's tile n0):
//   activation ring, 4 x 32 KB  rows [256 x 64] as two 128-row TMA boxes (the
//                               adapter intermediate on the extra k-steps)
//   weight ring, 4 x 16 KB      the bf16 weight tile (dequant warps; the
//                               adapter matrix by TMA on the extra k-steps)
//   code ring, 8 x 4 KB         packed codes of a k-step, fetched up to eight
//                               k-steps ahead by their own producer
//   warp 0   activation producer: pair TMA counted on the leader's xfull
//   warp 1   tensor-memory allocation (both CTAs, 512 columns); in the
//            leader CTA also the single thread that issues the pair MMAs
//   warp 2   code producer: local TMA on cfull
//   warps 3..18  four groups of four dequant warps; group g expands the
//            k-steps of weight slot g: it reads the codes and builds the
//            block's table as soon as the codes land, waits only for the
//            slot's previous MMAs (the same empty barrier the activation
//            producer waits on) before writing, and arrives on the leader's
//            wfull barrier; then the epilogue (accumulators -> bf16 tile in
//            the idle activation ring -> four TMA stores).
// So after the MMAs of a stage complete, the activation copy and the weight
// expansion of the stage's next k-step run side by side, not one after the
// other.
// Barriers: xfull[4] (leader; activation bytes of both CTAs), wfull[4]
// (leader; 8 arrivals, the 4 + 4 dequant warps), empty[4] (each CTA; one
// arrival from the leader's multicast commit), cfull[8] / cempty[8] (each
// CTA; codes landed / read by the group's 4 warps).  Every barrier is waited
// on by each of its waiters at every phase (four groups own the four weight
// slots and, in turn, two code slots each), so no parity wait can be
// satisfied by an older phase.  Every wait is bounded in time (a flag in the
// device error word on expiry); no kernel traps.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace qlora {
namespace {

constexpr int kRowsCta = 256;                   // activation rows per CTA (two 128-row MMA halves)
constexpr int kBN = 256;                        // output columns per pair tile
constexpr int kHalfN = kBN / 2;                 // output columns per CTA
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kCodeSlots = 8;
constexpr int kGroups = 4, kGroupWarps = 4;     // dequant: group g owns weight slot g
constexpr int kFirstDqWarp = 3;
constexpr uint32_t kASub = 128u * kBK * 2u;     // 16 KB: 128 activation rows of a k-step
constexpr uint32_t kABytes = 2u * kASub;
constexpr uint32_t kBBytes = static_cast<uint32_t>(kHalfN) * kBK * 2u;   // 16 KB
constexpr uint32_t kCBytes = static_cast<uint32_t>(kHalfN) * 32u;        // 4 KB
constexpr uint32_t kBRing = kStages * kABytes;                            // 128 KB
constexpr uint32_t kCRing = kBRing + kStages * kBBytes;                   // 192 KB
constexpr uint32_t kSmemBytes = kCRing + kCodeSlots * kCBytes + 1024u;
constexpr int kThreads = 32 * (kFirstDqWarp + kGroups * kGroupWarps);
constexpr uint32_t kTmemCols = 512;             // two 128 x 256 fp32 accumulators per CTA
static_assert(kStages == kGroups && kCodeSlots % kGroups == 0, "each dequant group owns its slots");
static_assert(kSmemBytes <= 227u * 1024u, "shared memory");

struct __align__(64) PairParams {
  CUtensorMap tmA;       // X [m x k] or dY [m x n] bf16, box {64, 128}, 128B swizzle
  CUtensorMap tmCodes;   // codes [n x k/2] bytes; box {32, 128} (forward), {32, 64} (input gradient)
  CUtensorMap tmA2;      // T or U [m x r] bf16, box {64, 128}, 128B swizzle
  CUtensorMap tmB2;      // adapter B [n x r] box {64, 128} (forward); A [r x k] box {64, 64} (input gradient)
  CUtensorMap tmOut;     // Y [m x n] or dX [m x k] bf16, box {64, 256}, 128B swizzle (TMA stores)
  const uint8_t *absmax_q;
  const float *group_scale;
  const float *mu;                 // E4M3 + mean absmax format: the tensor mean; else null
  uint16_t *out;         // Y [m x n] or dX [m x k]
  unsigned *err;
  int64_t n, k;          // weight shape
  int64_t out_cols;      // n (forward) or k (input gradient)
  int m, r;
  int num_main, num_lora;
  int pdl;
  Nf4Tables tab;
};

template <bool BWD>
__global__ void __launch_bounds__(kThreads, 1) fused_pair_kernel(const __grid_constant__ PairParams p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t xfull[kStages], wfull[kStages], empty[kStages];
  __shared__ __align__(8) uint64_t cfull[kCodeSlots], cempty[kCodeSlots];
  __shared__ __align__(8) uint64_t acc_full;
  __shared__ uint32_t tmem_slot;
  constexpr uint32_t kIdesc = make_idesc(kBN, false, BWD, 256);

  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int m_pair = static_cast<int>(blockIdx.x >> 1), n_tile = static_cast<int>(blockIdx.y);
  const int m0 = m_pair * (2 * kRowsCta) + static_cast<int>(rank) * kRowsCta;
  // First output column of this CTA's half: a weight row (forward) or a
  // weight column (input gradient).
  const int64_t c0 = static_cast<int64_t>(n_tile) * kBN + static_cast<int64_t>(rank) * kHalfN;
  const int total = p.num_main + p.num_lora;
  const int64_t kblocks = p.k / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&wfull[s], 2 * kGroupWarps);
      mbar_init(&empty[s], 1);
    }
    for (int c = 0; c < kCodeSlots; ++c) {
      mbar_init(&cfull[c], 1);
      mbar_init(&cempty[c], kGroupWarps);
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
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < total; ++it) {
        const int s = it % kStages;
        const uint32_t use = static_cast<uint32_t>(it / kStages);
        if (!mbar_wait_bounded(&empty[s], (use & 1u) ^ 1u, p.err, kErrTimeoutEmpty)) break;
        const uint32_t xa = base + static_cast<uint32_t>(s) * kABytes;
        const uint32_t wb = base + kBRing + static_cast<uint32_t>(s) * kBBytes;
        const bool lora = it >= p.num_main;
        const int l = it - p.num_main;
        // The adapter intermediate comes from the preceding projection kernel.
        if (lora && l == 0 && p.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint32_t xbar = mapa_shared(smem_u32(&xfull[s]), 0);
        if (leader) mbar_arrive_expect_tx(&xfull[s], 2u * (kABytes + (lora ? kBBytes : 0u)));
        const int kx = (lora ? l : it) * kBK;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // A 128-row half entirely past m loads rows 0..127 instead: its
          // accumulator rows are never stored, and every box stays in range.
          const int y = (m0 + h * 128 < p.m) ? m0 + h * 128 : 0;
          tma_load_2d_pair(xa + h * kASub, lora ? &p.tmA2 : &p.tmA, xbar, kx, y);
        }
        if (lora) {
          if (!BWD) {
            tma_load_2d_pair(wb, &p.tmB2, xbar, kx, (c0 < p.n) ? static_cast<int>(c0) : 0);
          } else {
            // A [r x k]: rows l*64.. of the adapter, this CTA's 128 columns
            // as two 64-column slabs.
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int64_t col = c0 + 64 * j;
              tma_load_2d_pair(wb + j * 8192u, &p.tmB2, xbar, col < p.k ? static_cast<int>(col) : 0, kx);
            }
          }
        }
        ++issued;
      }
      // Let the last copies land before the CTA may exit (the leader's xfull
      // also counts the peer's boxes).
      if (leader)
        for (int it = issued - kStages < 0 ? 0 : issued - kStages; it < issued; ++it)
          mbar_wait_bounded(&xfull[it % kStages], static_cast<uint32_t>(it / kStages) & 1u, p.err, kErrTimeoutDrain);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ code producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < p.num_main; ++it) {
        const int c = it % kCodeSlots;
        const uint32_t use = static_cast<uint32_t>(it / kCodeSlots);
        if (!mbar_wait_bounded(&cempty[c], (use & 1u) ^ 1u, p.err, kErrTimeoutEmpty)) break;
        const uint32_t cs = base + kCRing + static_cast<uint32_t>(c) * kCBytes;
        mbar_arrive_expect_tx(&cfull[c], kCBytes);
        if (!BWD) {
          tma_load_2d(cs, &p.tmCodes, &cfull[c], it * 32, (c0 < p.n) ? static_cast<int>(c0) : 0);
        } else {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int64_t col = c0 + 64 * j;
            tma_load_2d(cs + j * 2048u, &p.tmCodes, &cfull[c], col < p.k ? static_cast<int>(col / 2) : 0, it * kBK);
          }
        }
        ++issued;
      }
      for (int it = issued - kCodeSlots < 0 ? 0 : issued - kCodeSlots; it < issued; ++it)
        mbar_wait_bounded(&cfull[it % kCodeSlots], static_cast<uint32_t>(it / kCodeSlots) & 1u, p.err,
                          kErrTimeoutDrain);
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
        const uint32_t xa = base + static_cast<uint32_t>(s) * kABytes;
        const uint32_t wb = base + kBRing + static_cast<uint32_t>(s) * kBBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc(xa + h * kASub + kk * 32u, 16u, 1024u);
            const uint64_t bd = BWD ? smem_desc(wb + kk * 2048u, 8192u, 1024u) : smem_desc(wb + kk * 32u, 16u, 1024u);
            umma_f16_pair(tmem + static_cast<uint32_t>(h * kBN), ad, bd, kIdesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit_pair_both(&empty[s]);
      }
      if (ok) umma_commit_pair_both(&acc_full);
    }
  } else {
    // ------------------------------------------------------------ dequant
    const int dq = warp - kFirstDqWarp;
    const int grp = dq / kGroupWarps;                     // == the weight slot this group fills
    const int dt = (dq % kGroupWarps) * 32 + lane;        // block slot of this CTA's half tile
    // Forward: weight row c0 + dt, block `it` of it.  Input gradient: weight
    // row it*64 + (dt & 63), block c0/64 + (dt >> 6).
    const int n_local = BWD ? (dt & 63) : dt;
    const int slab = BWD ? (dt >> 6) : 0;
    const uint32_t row_off = static_cast<uint32_t>(slab) * 8192u + static_cast<uint32_t>(n_local) * 128u;
    const uint32_t code_off = BWD ? static_cast<uint32_t>(slab) * 2048u + static_cast<uint32_t>(n_local) * 32u
                                  : static_cast<uint32_t>(dt) * 32u;
    const uint32_t sw = static_cast<uint32_t>(n_local & 7);
    const uint32_t first_half = ((lane >> 2) & 1u) ? 16u : 0u;
    const uint32_t wbar = mapa_shared(smem_u32(&wfull[grp]), 0);
    const uint32_t wslot = base + kBRing + static_cast<uint32_t>(grp) * kBBytes;
    // Block index of k-step `it` for this thread, or -1 outside the weight.
    const auto block_of = [&](int it) -> int64_t {
      int64_t gn, kb;
      if (!BWD) {
        gn = c0 + dt;
        kb = it;
      } else {
        gn = static_cast<int64_t>(it) * kBK + n_local;
        kb = c0 / 64 + slab;
      }
      return (gn < p.n && kb < kblocks) ? gn * kblocks + kb : -1;
    };
    // Absmax code and group scale of this group's next k-step, fetched one
    // step of the group ahead; the group constant t (fp32(S / 255) for
    // linear codes) recomputed only when the group index changes.
    const bool fp8 = p.mu != nullptr;
    const float mu = load_mu(p.mu);
    int64_t blk_nx = grp < p.num_main ? block_of(grp) : -1;
    uint32_t q_nx = blk_nx >= 0 ? __ldg(p.absmax_q + blk_nx) : 0u;
    float S_nx = blk_nx >= 0 ? __ldg(p.group_scale + (blk_nx >> 8)) : 0.f;
    int64_t g_cur = -1;
    float t_cur = 0.f;
    for (int it = grp; it < total; it += kGroups) {
      const uint32_t use = static_cast<uint32_t>(it / kStages);
      if (it < p.num_main) {
        const int c = it % kCodeSlots;
        if (!mbar_wait_bounded(&cfull[c], static_cast<uint32_t>(it / kCodeSlots) & 1u, p.err, kErrTimeoutFullA))
          break;
        const int64_t blk = blk_nx;
        const uint32_t qv = q_nx;
        const float S = S_nx;
        // Codes into registers, code slot released, block table built: all
        // before the weight slot is free.
        Bf16Table tb;
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = make_uint4(0u, 0u, 0u, 0u);
        if (blk >= 0) {
          const uint32_t c_s = base + kCRing + static_cast<uint32_t>(c) * kCBytes + code_off;
          const uint4 f = lds128(c_s + first_half);
          const uint4 g2 = lds128(c_s + (16u - first_half));
          lo = first_half ? g2 : f;
          hi = first_half ? f : g2;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[c]);
        if (blk >= 0) {
          const int64_t gidx = blk >> 8;
          if (gidx != g_cur) {
            g_cur = gidx;
            t_cur = group_constant(S, fp8);
          }
          make_table(p.tab, block_constant(qv, t_cur, fp8, mu), tb);
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) tb.lo[j] = tb.hi[j] = 0u;
        }
        if (!mbar_wait_bounded(&empty[grp], (use & 1u) ^ 1u, p.err, kErrTimeoutEmpty)) break;
        const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        const uint32_t rowaddr = wslot + row_off;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t o[4];
          decode8(words[cc], tb, o);
          sts128(rowaddr + ((static_cast<uint32_t>(cc) ^ sw) << 4), o);
        }
        fence_proxy_async_smem();
      } else {
        // Adapter k-steps: the adapter matrix comes by TMA once the slot is
        // free; the arrival keeps the barrier's phases in step.
        if (!mbar_wait_bounded(&empty[grp], (use & 1u) ^ 1u, p.err, kErrTimeoutEmpty)) break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(wbar);
      // The next k-step's absmax code and group scale, requested only now so
      // that the proxy fence above never waits for these loads.
      if (it + kGroups < p.num_main) {
        blk_nx = block_of(it + kGroups);
        q_nx = blk_nx >= 0 ? __ldg(p.absmax_q + blk_nx) : 0u;
        S_nx = blk_nx >= 0 ? __ldg(p.group_scale + (blk_nx >> 8)) : 0.f;
      }
    }

    // ------------------------------------------------------------ epilogue
    // The accumulators go out through shared memory: every operand copy and
    // MMA of the tile is done once acc_full completes, so the activation
    // ring (128 KB) holds the CTA's bf16 output tile [256 rows x 256 columns]
    // as four 64-column slabs of 128-byte rows, 128-byte swizzled (the TMA
    // box layout; a quarter-warp's 16-byte stores hit eight distinct bank
    // groups).  Four TMA stores then write whole lines of Y (or dX).
    const bool acc_ok = mbar_wait_bounded(&acc_full, 0u, p.err, kErrTimeoutAcc, 20000000000ull);
    if (acc_ok) {
      tc_fence_after();
      const int quad = warp & 3;                          // TMEM lanes this warp may read
      const int q4 = dq >> 2;                             // column quarter of the 512 columns
      const int h = q4 >> 1;
      const int c_begin = (q4 & 1) * (kBN / 2);
      const uint32_t row = static_cast<uint32_t>(h * 128 + quad * 32 + lane);   // row of the CTA's tile
      const uint32_t rsw = row & 7u;
      for (int cc = c_begin; cc < c_begin + kBN / 2; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(h * kBN + cc), v);
        const uint32_t slab_row = base + static_cast<uint32_t>(cc >> 6) * 32768u + row * 128u;
        const uint32_t c16 = static_cast<uint32_t>((cc & 63) >> 3);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t w[4] = {pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1])),
                                 pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                                 pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                                 pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]))};
          sts128(slab_row + (((c16 + static_cast<uint32_t>(j)) ^ rsw) << 4), w);
        }
      }
      fence_proxy_async_smem();
    }
    // All 16 epilogue warps (512 threads) take part, even after a timeout.
    named_barrier_sync(1, 32 * kGroups * kGroupWarps);
    if (dq == 0 && lane == 0 && acc_ok && m0 < p.m) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t col = static_cast<int64_t>(n_tile) * kBN + 64 * j;
        if (col < p.out_cols) tma_store_2d(&p.tmOut, base + static_cast<uint32_t>(j) * 32768u, static_cast<int>(col), m0);
      }
      tma_store_drain();
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

template <bool BWD>
cudaError_t launch_pair(const PairParams &p, int64_t m, int64_t out_cols, cudaStream_t stream) {
  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(fused_pair_kernel<BWD>), static_cast<int>(kSmemBytes),
                                configured);
  if (e != cudaSuccess) return e;
  const int64_t pairs_m = (m + 2 * kRowsCta - 1) / (2 * kRowsCta);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs_m), static_cast<unsigned>((out_cols + kBN - 1) / kBN), 1);
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
  e = cudaLaunchKernelEx(&cfg, fused_pair_kernel<BWD>, p);
  if (e == cudaSuccess) count_launches(1);
  return e;
}

PairParams common_params(const WeightView &w, int64_t m, int32_t r, bool lora, bool pdl, uint16_t *out) {
  PairParams p{};
  p.absmax_q = w.absmax_q;
  p.group_scale = w.group_scale;
  p.mu = w.mu;
  p.out = out;
  p.err = device_error_word();
  p.n = w.n;
  p.k = w.k;
  p.m = static_cast<int>(m);
  p.r = lora ? r : 0;
  p.num_lora = lora ? (r + kBK - 1) / kBK : 0;
  p.pdl = (lora && pdl) ? 1 : 0;
  p.tab = *w.tab;
  return p;
}

}  // namespace

cudaError_t fused_fwd_large(const uint16_t *X, int64_t m, const WeightView &w, const uint16_t *T, const uint16_t *B,
                            int32_t r, uint16_t *Y, cudaStream_t stream, bool pdl) {
  const bool lora = T != nullptr && B != nullptr && r > 0;
  PairParams p = common_params(w, m, r, lora, pdl, Y);
  if (!encode_bf16_map(&p.tmA, X, m, w.k, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_codes_map(&p.tmCodes, w.codes, w.n, w.k / 2, 32, kHalfN, false)) return cudaErrorInvalidValue;
  if (lora) {
    if (!encode_bf16_map(&p.tmA2, T, m, r, 64, 128)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&p.tmB2, B, w.n, r, 64, kHalfN)) return cudaErrorInvalidValue;
  }
  if (!encode_bf16_map(&p.tmOut, Y, m, w.n, 64, 256)) return cudaErrorInvalidValue;
  p.out_cols = w.n;
  p.num_main = static_cast<int>(w.k / kBK);
  return launch_pair<false>(p, m, w.n, stream);
}

cudaError_t fused_bwd_dx_large(const uint16_t *dY, int64_t m, const WeightView &w, const uint16_t *U,
                               const uint16_t *A, int32_t r, uint16_t *dX, cudaStream_t stream, bool pdl) {
  const bool lora = U != nullptr && A != nullptr && r > 0;
  PairParams p = common_params(w, m, r, lora, pdl, dX);
  if (!encode_bf16_map(&p.tmA, dY, m, w.n, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_codes_map(&p.tmCodes, w.codes, w.n, w.k / 2, 32, 64, false)) return cudaErrorInvalidValue;
  if (lora) {
    if (!encode_bf16_map(&p.tmA2, U, m, r, 64, 128)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&p.tmB2, A, r, w.k, 64, 64)) return cudaErrorInvalidValue;
  }
  if (!encode_bf16_map(&p.tmOut, dX, m, w.k, 64, 256)) return cudaErrorInvalidValue;
  p.out_cols = w.k;
  p.num_main = static_cast<int>((w.n + kBK - 1) / kBK);
  return launch_pair<true>(p, m, w.k, stream);
}

}  // namespace qlora
