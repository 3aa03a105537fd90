// tcgen05 / TMEM GEMMs for the QLoRA linear layer on sm_100a.
//
// One kernel template covers every dense contraction of the layer:
//
//   fused forward     D = X . W^T   (+ T . B^T as extra k-steps)
//   fused bwd_dx      D = dY . W^   (+ U . A   as extra k-steps)
//   skinny products   T = s X A^T, U = s dY B, dA^T = X^T U, dB = dY^T T
//
// "QLoRA and Quantized Training", The idea: compute happens in bf16, each block
// is dequantized, used in a matrix multiply and discarded; "A 65B fine-tune on
// the GPU you already have", figure 2: dequantized block by block to bf16 just
// long enough to multiply.  Here the NF4 weight never exists in bf16 outside
// shared memory: TMA stages the packed codes of one k-step (one NF4 block per
// weight row) into shared memory, eight dequant warps expand them into a
// 128-byte-swizzled bf16 tile, and one thread issues tcgen05.mma on it with
// the fp32 accumulator in tensor memory.
//
// Warp roles (one CTA per output tile, 1 CTA per SM):
//   warp 0      TMA producer (A operand, packed codes or B operand)
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..   dequant producers during the main loop (NF4 modes), then the
//               epilogue: tcgen05.ld -> scale -> bf16 -> global
// Stages are guarded by mbarriers: full_a (TMA bytes landed), full_b (dequant
// warps wrote the B tile), empty (the MMAs reading the stage completed, via
// tcgen05.commit), acc (all MMAs done).  Every wait is bounded in time: on a
// timeout a flag is set in the caller-visible error word and the roles drain
// and exit; no kernel traps.
//
// Shared-memory operand layouts (SWIZZLE_128B, 1024-byte aligned atoms):
//   K-major tile  [rows x 64] bf16: row r at r*128, 16-byte chunk c stored at
//                 chunk c ^ (r % 8)             (LBO 16 B, SBO 1024 B)
//   MN-major tile [64 k-rows x 64*j cols]: slab j (64 columns) at j*8192, k-row
//                 at 128 B pitch, same swizzle    (LBO 8192 B, SBO 1024 B)
// One NF4 block (64 consecutive weights of a row) is one 128-byte swizzled
// row in both layouts, so the forward (weight rows are MMA N, K-major) and the
// input gradient (weight rows are the contraction, MN-major) share the
// dequant routine and differ only in which (row, block) lands in which row.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "philox.cuh"
#include "tcgen05.cuh"

namespace qlora {
namespace {

// 16 bytes (four fp32) at the same offset in CTA `rank`'s shared memory;
// local_addr must be 16-byte aligned.
__device__ __forceinline__ float4 ld_dsmem_v4(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(remote)
               : "memory");
  return v;
}

constexpr int kBK = 64;                       // k-step: 64 bf16 = one swizzle row
constexpr uint32_t kASub = 128u * kBK * 2u;   // 16 KB: one 128-row A tile

struct __align__(64) TcParams {
  CUtensorMap tmA;      // main A operand
  CUtensorMap tmB;      // main B operand (bf16 modes)
  CUtensorMap tmCodes;  // packed codes viewed as [rows x bytes] (NF4 modes)
  CUtensorMap tmA2;     // adapter A operand (extra k-steps)
  CUtensorMap tmB2;     // adapter B operand (extra k-steps)
  const uint8_t *absmax_q;
  const float *group_scale;
  const float *mu;                 // E4M3 + mean absmax format: the tensor mean; else null
  uint16_t *out;
  unsigned *err;
  int64_t w_n, w_k;     // weight shape (NF4 modes)
  int64_t out_ld;
  int out_rows, out_cols;
  int num_main, num_lora;
  int pdl;              // launched as a programmatic dependent of the adapter projection
  float alpha;
  Nf4Tables tab;
  DropoutParams drop;   // masked-add epilogue only
};

// Epilogues: store bf16(alpha . acc), or (dropout) add the masked product to
// the bf16 output already there: out = bf16(out + D . acc . keep_scale).
enum : int { kEpiStore = 0, kEpiDropoutAdd = 1 };

// ---- compile-time configuration -------------------------------------------

template <int BN_, int MSUB_, bool A_MN_, bool B_NF4_, bool B_MN_, bool OUT_T_, bool SPLIT_ = false,
          int EPI_ = kEpiStore>
struct Cfg {
  static constexpr int EPI = EPI_;
  static constexpr bool SPLIT = SPLIT_;   // contraction split over a cluster, DSMEM reduction
  static constexpr int BN = BN_;
  static constexpr int MSUB = MSUB_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_NF4 = B_NF4_;
  static constexpr bool B_MN = B_MN_;
  static constexpr bool OUT_T = OUT_T_;
  static constexpr int BM = 128 * MSUB;
  static constexpr uint32_t A_BYTES = kASub * MSUB;
  static constexpr uint32_t B_BYTES = static_cast<uint32_t>(BN) * kBK * 2u;
  static constexpr uint32_t CODE_BYTES = B_NF4 ? static_cast<uint32_t>(BN) * 32u : 0u;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + CODE_BYTES;
  static constexpr int STAGES_RAW = static_cast<int>((224u * 1024u) / STAGE_BYTES);
  // Skinny (BN=64) configs keep 4 stages so two CTAs fit on an SM.
  // The masked-add product has at most four k-steps (K = r <= 256): two
  // stages, so that two CTAs share an SM.
  static constexpr int STAGES = B_NF4 ? (STAGES_RAW > 6 ? 6 : STAGES_RAW) : (EPI == kEpiDropoutAdd ? 2 : 4);
  static constexpr uint32_t SMEM_BYTES = STAGE_BYTES * STAGES + 1024u;
  // NF4 modes: two groups of 8 dequant warps take k-steps in turn (the
  // expansion of a k-step is latency-bound; two groups keep two in flight).
  static constexpr int DQ_GROUPS = B_NF4 ? 2 : 0;
  // The masked-add epilogue regenerates the dropout mask (one Philox call per
  // 16 outputs): sixteen warps share that work.
  static constexpr int NUM_EPI_WARPS = B_NF4 ? 8 * DQ_GROUPS : (EPI == kEpiDropoutAdd ? 16 : 4);
  static constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
  static constexpr uint32_t TMEM_RAW = static_cast<uint32_t>(BN * MSUB);
  static constexpr uint32_t TMEM_COLS = TMEM_RAW <= 32 ? 32 : TMEM_RAW <= 64 ? 64 : TMEM_RAW <= 128 ? 128 : TMEM_RAW <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC = make_idesc(BN, A_MN, B_MN);
  static_assert(STAGES >= 2, "not enough shared memory for two stages");
  static_assert(!(A_MN && MSUB != 1), "MN-major A supports one 128-row tile");
  static_assert(!B_NF4 || BN == 256, "NF4 modes use 256-wide tiles (one block per dequant thread)");
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  static_assert(!SPLIT || (MSUB == 1 && (B_NF4 ? BN == 256 : BN == 64)),
                "split-K: the skinny products and the small-M NF4 products");
  // Split-K partial tile, laid out along the output's contiguous dimension:
  // row-major with rows of BN fp32 padded by 16 bytes (the 16-byte pieces of
  // 8 consecutive rows land in 8 distinct bank groups) for a row-major
  // output, column-major (128 fp32 per column) for a transposed one.
  static constexpr uint32_t PART_LD = static_cast<uint32_t>(BN) + 4u;
  static_assert(!SPLIT || STAGE_BYTES * STAGES >= 128u * PART_LD * 4u, "room for the fp32 partial tile");
  static_assert(EPI == kEpiStore || (!SPLIT && !OUT_T && !B_NF4), "masked add: plain row-major output");
};

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1) tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_a[C::STAGES];
  __shared__ __align__(8) uint64_t full_b[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_slot;

  const uint32_t raw = smem_u32(dsmem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x;
  const int m_tile = blockIdx.y;
  // With split-K, CTA z of the cluster runs k-steps [it_begin, total); the
  // adapter k-steps, if any, go to the last CTA.
  int it_begin = 0, total = p.num_main + p.num_lora;
  if (C::SPLIT) {
    const int z = static_cast<int>(blockIdx.z), nz = static_cast<int>(gridDim.z);
    it_begin = static_cast<int>((static_cast<int64_t>(p.num_main) * z) / nz);
    if (z + 1 < nz) total = static_cast<int>((static_cast<int64_t>(p.num_main) * (z + 1)) / nz);
  }
  const int n_iters = total - it_begin;

  // A skinny projection lets the kernel that consumes its output launch now;
  // that kernel waits for this grid before it reads the output.
  if (C::SPLIT && !C::B_NF4) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full_a[s], 1);
      mbar_init(&full_b[s], C::B_NF4 ? 8 : 1);   // one group of 8 dequant warps per stage fill
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA);
    if (C::B_NF4) tma_prefetch_desc(&p.tmCodes); else tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(C::TMEM_COLS)
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
      for (int it = it_begin; it < total; ++it) {
        const int li = it - it_begin;
        const int s = li % C::STAGES;
        const uint32_t ph = static_cast<uint32_t>(li / C::STAGES) & 1u;
        if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, p.err, kErrTimeoutEmpty)) break;
        const uint32_t a_s = base + static_cast<uint32_t>(s) * C::STAGE_BYTES;
        const uint32_t b_s = a_s + C::A_BYTES;
        const uint32_t c_s = b_s + C::B_BYTES;
        if (it < p.num_main) {
          mbar_arrive_expect_tx(&full_a[s], C::A_BYTES + (C::B_NF4 ? C::CODE_BYTES : C::B_BYTES));
          if (!C::A_MN) {
#pragma unroll
            for (int h = 0; h < C::MSUB; ++h)
              tma_load_2d(a_s + h * kASub, &p.tmA, &full_a[s], it * kBK, m_tile * C::BM + h * 128);
          } else {
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d(a_s + j * 8192u, &p.tmA, &full_a[s], m_tile * 128 + j * 64, it * kBK);
          }
          if (C::B_NF4) {
            if (!C::B_MN) {
              tma_load_2d(c_s, &p.tmCodes, &full_a[s], it * 32, n_tile * C::BN);
            } else {
#pragma unroll
              for (int j = 0; j < C::BN / 64; ++j)
                tma_load_2d(c_s + j * 2048u, &p.tmCodes, &full_a[s], n_tile * (C::BN / 2) + 32 * j, it * kBK);
            }
          } else {
            if (!C::B_MN) {
              tma_load_2d(b_s, &p.tmB, &full_a[s], it * kBK, n_tile * C::BN);
            } else {
#pragma unroll
              for (int j = 0; j < C::BN / 64; ++j)
                tma_load_2d(b_s + j * 8192u, &p.tmB, &full_a[s], n_tile * C::BN + 64 * j, it * kBK);
            }
          }
        } else {
          const int l = it - p.num_main;
          // The adapter operand comes from the preceding projection kernel.
          if (l == 0 && p.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
          mbar_arrive_expect_tx(&full_a[s], C::A_BYTES + C::B_BYTES);
#pragma unroll
          for (int h = 0; h < C::MSUB; ++h)
            tma_load_2d(a_s + h * kASub, &p.tmA2, &full_a[s], l * kBK, m_tile * C::BM + h * 128);
          if (!C::B_MN) {
            tma_load_2d(b_s, &p.tmB2, &full_a[s], l * kBK, n_tile * C::BN);
          } else {
#pragma unroll
            for (int j = 0; j < C::BN / 64; ++j)
              tma_load_2d(b_s + j * 8192u, &p.tmB2, &full_a[s], n_tile * C::BN + 64 * j, l * kBK);
          }
        }
        ++issued;
      }
      // Drain: every issued copy has landed before the CTA may exit.
      for (int it = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; it < issued; ++it)
        mbar_wait_bounded(&full_a[it % C::STAGES], static_cast<uint32_t>(it / C::STAGES) & 1u, p.err,
                          kErrTimeoutDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int it = it_begin; it < total && ok; ++it) {
        const int li = it - it_begin;
        const int s = li % C::STAGES;
        const uint32_t ph = static_cast<uint32_t>(li / C::STAGES) & 1u;
        ok = mbar_wait_bounded(&full_a[s], ph, p.err, kErrTimeoutFullA);
        if (ok && C::B_NF4) ok = mbar_wait_bounded(&full_b[s], ph, p.err, kErrTimeoutFullB);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_s = base + static_cast<uint32_t>(s) * C::STAGE_BYTES;
        const uint32_t b_s = a_s + C::A_BYTES;
#pragma unroll
        for (int h = 0; h < C::MSUB; ++h) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = C::A_MN ? smem_desc(a_s + kk * 2048u, 8192u, 1024u)
                                        : smem_desc(a_s + h * kASub + kk * 32u, 16u, 1024u);
            const uint64_t bd = C::B_MN ? smem_desc(b_s + kk * 2048u, 8192u, 1024u)
                                        : smem_desc(b_s + kk * 32u, 16u, 1024u);
            umma_f16(tmem + static_cast<uint32_t>(h * C::BN), ad, bd, C::IDESC, (li > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty_bar[s]);
      }
      if (ok) umma_commit(&acc_bar);
    }
  } else {
    // ------------------------------------------------------------ dequant
    // Groups of 8 warps take k-steps in turn, so DQ_GROUPS B tiles are being
    // expanded at once; within a group thread dt fills one 128-byte row.
    const int grp = (warp - 2) >> 3;                 // 0 .. DQ_GROUPS-1 (NF4 modes)
    const int dt = (threadIdx.x - 64) & 255;
    bool ok = true;
    if (C::B_NF4) {
      const int64_t kblocks = p.w_k / 64;
      // Row of the B tile this thread fills, and which weight block goes there.
      const int n_local = C::B_MN ? (dt & 63) : dt;
      const int slab = C::B_MN ? (dt >> 6) : 0;
      const uint32_t row_off = static_cast<uint32_t>(slab) * 8192u + static_cast<uint32_t>(n_local) * 128u;
      const uint32_t code_off = C::B_MN ? static_cast<uint32_t>(slab) * 2048u + static_cast<uint32_t>(n_local) * 32u
                                        : static_cast<uint32_t>(dt) * 32u;
      const uint32_t first_half = ((lane >> 2) & 1u) ? 16u : 0u;
      const uint32_t sw = static_cast<uint32_t>(n_local & 7);
      // Block index of step `it` for this thread, or -1 outside the weight.
      auto block_of = [&](int it) -> int64_t {
        int64_t gn, kb;
        if (!C::B_MN) {
          gn = static_cast<int64_t>(n_tile) * C::BN + dt;
          kb = it;
        } else {
          gn = static_cast<int64_t>(it) * kBK + n_local;
          kb = static_cast<int64_t>(n_tile) * (C::BN / 64) + slab;
        }
        return (gn < p.w_n && kb < kblocks) ? gn * kblocks + kb : -1;
      };
      // Absmax code and group constant of this group's next step, fetched one
      // step of the group (DQ_GROUPS k-steps) ahead.  The group constant t
      // (fp32(S / 255) for linear codes) is recomputed only when the group
      // index changes (in the forward a thread walks one weight row, so that
      // is rare).
      const bool fp8 = p.mu != nullptr;
      const float mu = load_mu(p.mu);
      int64_t blk_nx = it_begin + grp < p.num_main ? block_of(it_begin + grp) : -1;
      uint32_t q_nx = blk_nx >= 0 ? __ldg(p.absmax_q + blk_nx) : 0u;
      float S_nx = blk_nx >= 0 ? __ldg(p.group_scale + (blk_nx >> 8)) : 0.f;
      int64_t g_cur = -1;
      float t_cur = 0.f;
      constexpr int kStride = C::DQ_GROUPS > 0 ? C::DQ_GROUPS : 1;
      // Each stage must be taken by one group only (STAGES a multiple of the
      // group count), so that a group waits on every phase of its stages'
      // barriers and a parity wait cannot be satisfied by an older phase.
      static_assert(C::DQ_GROUPS <= 1 || C::STAGES % C::DQ_GROUPS == 0, "stages per dequant group");
      for (int li = grp; li < n_iters; li += kStride) {
        const int it = it_begin + li;
        const int s = li % C::STAGES;
        const uint32_t ph = static_cast<uint32_t>(li / C::STAGES) & 1u;
        if (!mbar_wait_bounded(&full_a[s], ph, p.err, kErrTimeoutFullA)) { ok = false; break; }
        if (it < p.num_main) {
          const int64_t blk = blk_nx;
          const uint32_t qv = q_nx;
          const float S = S_nx;
          if (it + kStride < p.num_main) {
            blk_nx = block_of(it + kStride);
            q_nx = blk_nx >= 0 ? __ldg(p.absmax_q + blk_nx) : 0u;
            S_nx = blk_nx >= 0 ? __ldg(p.group_scale + (blk_nx >> 8)) : 0.f;
          }
          const uint32_t a_s = base + static_cast<uint32_t>(s) * C::STAGE_BYTES;
          const uint32_t b_s = a_s + C::A_BYTES;
          const uint32_t c_s = b_s + C::B_BYTES;
          Bf16Table tb;
          uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = make_uint4(0u, 0u, 0u, 0u);
          if (blk >= 0) {
            const int64_t gi = blk >> 8;
            if (gi != g_cur) {
              g_cur = gi;
              t_cur = group_constant(S, fp8);
            }
            const uint4 f = lds128(c_s + code_off + first_half);
            const uint4 g2 = lds128(c_s + code_off + (16u - first_half));
            lo = first_half ? g2 : f;
            hi = first_half ? f : g2;
            make_table(p.tab, block_constant(qv, t_cur, fp8, mu), tb);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) tb.lo[j] = tb.hi[j] = 0u;
          }
          const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
          const uint32_t rowaddr = b_s + row_off;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            decode8(words[c], tb, o);
            sts128(rowaddr + ((static_cast<uint32_t>(c) ^ sw) << 4), o);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&full_b[s]);
      }
    }

    // ------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait_bounded(&acc_bar, 0u, p.err, kErrTimeoutAcc, 20000000000ull);
    if (ok) {
      tc_fence_after();
      const int ew = warp - 2;
      const int quad = warp & 3;
      int h = 0, c_begin = 0, c_end = C::BN;
      if (C::NUM_EPI_WARPS == 8) {
        if (C::MSUB == 2) {
          h = ew >> 2;
        } else {
          c_begin = (ew >> 2) * (C::BN / 2);
          c_end = c_begin + C::BN / 2;
        }
      } else if (C::NUM_EPI_WARPS == 16) {
        // 16 warps: 4 lane quadrants x (accumulator half, column half) or
        // x column quarter.
        if (C::MSUB == 2) {
          h = ew >> 3;
          c_begin = ((ew >> 2) & 1) * (C::BN / 2);
          c_end = c_begin + C::BN / 2;
        } else {
          c_begin = (ew >> 2) * (C::BN / 4);
          c_end = c_begin + C::BN / 4;
        }
      }
      const int row_in_tile = h * 128 + quad * 32 + lane;
      const int64_t grow = static_cast<int64_t>(m_tile) * C::BM + row_in_tile;
      const bool row_ok = grow < p.out_rows;
      for (int c0 = c_begin; c0 < c_end; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(h * C::BN + c0), v);
        if (C::SPLIT) {
          // fp32 partial in this CTA's idle stage memory.
          if (!C::OUT_T) {
            const uint32_t dst =
                base + (static_cast<uint32_t>(row_in_tile) * C::PART_LD + static_cast<uint32_t>(c0)) * 4u;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) w[e] = n_iters > 0 ? v[4 * j + e] : 0u;
              sts128(dst + 16u * static_cast<uint32_t>(j), w);
            }
          } else {
            const uint32_t dst = base + (static_cast<uint32_t>(c0) * 128u + static_cast<uint32_t>(row_in_tile)) * 4u;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float val = n_iters > 0 ? __uint_as_float(v[j]) : 0.f;
              asm volatile("st.shared.f32 [%0], %1;" ::"r"(dst + static_cast<uint32_t>(j) * 512u), "f"(val) : "memory");
            }
          }
          continue;
        }
        const int64_t gcol = static_cast<int64_t>(n_tile) * C::BN + c0;
        if (C::EPI == kEpiDropoutAdd) {
          // 32 outputs starting at a multiple of 32 of a row whose length is
          // a multiple of 64: two whole mask blocks, never past the row.
          if (row_ok && gcol < p.out_cols) {
            uint16_t *dst = p.out + grow * p.out_ld + gcol;
            const uint64_t blk = static_cast<uint64_t>(grow * p.out_ld + gcol) >> 4;
            const uint32_t keep = dropout_keep_bits(blk, p.drop.seed, p.drop.offset, p.drop.threshold) |
                                  (dropout_keep_bits(blk + 1, p.drop.seed, p.drop.offset, p.drop.threshold) << 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint4 old = reinterpret_cast<const uint4 *>(dst)[j];
              const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
              uint32_t nw[4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const int e = 8 * j + 2 * t;
                const float a0 = (keep >> e) & 1u ? __fmul_rn(__uint_as_float(v[e]), p.drop.keep_scale) : 0.f;
                const float a1 =
                    (keep >> (e + 1)) & 1u ? __fmul_rn(__uint_as_float(v[e + 1]), p.drop.keep_scale) : 0.f;
                nw[t] = pack_bf16x2(__fadd_rn(bf16lo_to_f32(ow[t]), a0), __fadd_rn(bf16hi_to_f32(ow[t]), a1));
              }
              reinterpret_cast<uint4 *>(dst)[j] = make_uint4(nw[0], nw[1], nw[2], nw[3]);
            }
          }
          continue;
        }
        if (!C::OUT_T) {
          if (row_ok) {
            uint16_t *dst = p.out + grow * p.out_ld + gcol;
            if (gcol + 32 <= p.out_cols) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(v[8 * j + 0]) * p.alpha, __uint_as_float(v[8 * j + 1]) * p.alpha);
                w.y = pack_bf16x2(__uint_as_float(v[8 * j + 2]) * p.alpha, __uint_as_float(v[8 * j + 3]) * p.alpha);
                w.z = pack_bf16x2(__uint_as_float(v[8 * j + 4]) * p.alpha, __uint_as_float(v[8 * j + 5]) * p.alpha);
                w.w = pack_bf16x2(__uint_as_float(v[8 * j + 6]) * p.alpha, __uint_as_float(v[8 * j + 7]) * p.alpha);
                reinterpret_cast<uint4 *>(dst)[j] = w;
              }
            } else {
              for (int j = 0; j < 32; ++j)
                if (gcol + j < p.out_cols)
                  dst[j] = static_cast<uint16_t>(pack_bf16x2(__uint_as_float(v[j]) * p.alpha, 0.f) & 0xFFFFu);
            }
          }
        } else {
          if (row_ok) {
            for (int j = 0; j < 32; ++j)
              if (gcol + j < p.out_cols)
                p.out[(gcol + j) * p.out_ld + grow] =
                    static_cast<uint16_t>(pack_bf16x2(__uint_as_float(v[j]) * p.alpha, 0.f) & 0xFFFFu);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (C::SPLIT) {
    // Reduce the cluster's partial tiles through distributed shared memory:
    // CTA `rank` finishes a share of the tile's rows that exist in the output
    // (in whole groups of four rows for a transposed output).
    cluster_sync_all();
    const uint32_t rank = cluster_rank(), size = cluster_size();
    const int64_t left = static_cast<int64_t>(p.out_rows) - static_cast<int64_t>(m_tile) * C::BM;
    const uint32_t valid = static_cast<uint32_t>(left < 128 ? (left > 0 ? left : 0) : 128);
    const uint32_t units = C::OUT_T ? (valid + 3u) / 4u : valid;
    const int u_lo = static_cast<int>((units * rank) / size), u_hi = static_cast<int>((units * (rank + 1)) / size);
    const int nu = u_hi - u_lo;
    // Work items are 16-byte pieces along the partial's contiguous dimension:
    // (row, 4 columns) for a row-major output, (column, 4 rows) for a
    // transposed one; consecutive threads take consecutive pieces, so the
    // remote reads and the bf16 stores are contiguous.  A thread takes kBatch
    // pieces at a time and issues all their peer loads (up to 8 peers) before
    // the first add, so the remote-load latency is paid once per batch; each
    // piece's partials are added in peer order.
    constexpr int kBatch = C::NUM_THREADS > 256 ? 1 : 2;   // 32 registers of partials per piece
    constexpr int kPieces = C::BN / 4;                      // pieces per row (row-major output)
    const int nel = C::OUT_T ? nu * C::BN : nu * kPieces;
    const bool vec_ok = (p.out_ld & 3) == 0 && (reinterpret_cast<uintptr_t>(p.out) & 7u) == 0;
    for (int i0 = threadIdx.x; i0 < nel; i0 += kBatch * C::NUM_THREADS) {
      float4 part[kBatch][8];
      int row[kBatch], col[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int i = i0 + b * C::NUM_THREADS;
        const bool live = i < nel;
        const int ii = live ? i : 0;
        uint32_t off;
        if (!C::OUT_T) {
          row[b] = u_lo + ii / kPieces;
          col[b] = 4 * (ii % kPieces);
          off = base + (static_cast<uint32_t>(row[b]) * C::PART_LD + static_cast<uint32_t>(col[b])) * 4u;
        } else {
          row[b] = 4 * (u_lo + ii % nu);
          col[b] = ii / nu;
          off = base + (static_cast<uint32_t>(col[b]) * 128u + static_cast<uint32_t>(row[b])) * 4u;
        }
        if (!live) col[b] = -1;
#pragma unroll
        for (int pr = 0; pr < 8; ++pr)
          part[b][pr] = (live && static_cast<uint32_t>(pr) < size) ? ld_dsmem_v4(off, static_cast<uint32_t>(pr))
                                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        if (col[b] < 0) continue;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int pr = 0; pr < 8; ++pr) {
          if (static_cast<uint32_t>(pr) < size) {
            acc.x += part[b][pr].x;
            acc.y += part[b][pr].y;
            acc.z += part[b][pr].z;
            acc.w += part[b][pr].w;
          }
        }
        const int64_t grow = static_cast<int64_t>(m_tile) * C::BM + row[b];
        const int64_t gcol = static_cast<int64_t>(n_tile) * C::BN + col[b];
        const uint32_t h01 = pack_bf16x2(acc.x * p.alpha, acc.y * p.alpha);
        const uint32_t h23 = pack_bf16x2(acc.z * p.alpha, acc.w * p.alpha);
        const uint16_t h[4] = {static_cast<uint16_t>(h01 & 0xFFFFu), static_cast<uint16_t>(h01 >> 16),
                               static_cast<uint16_t>(h23 & 0xFFFFu), static_cast<uint16_t>(h23 >> 16)};
        if (!C::OUT_T) {
          // Row grow, columns gcol .. gcol + 3.
          if (grow >= p.out_rows) continue;
          if (vec_ok && gcol + 4 <= p.out_cols) {
            *reinterpret_cast<uint2 *>(p.out + grow * p.out_ld + gcol) = make_uint2(h01, h23);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (gcol + e < p.out_cols) p.out[grow * p.out_ld + gcol + e] = h[e];
          }
        } else {
          // Column gcol of the tile = row gcol of the transposed output, its
          // entries grow .. grow + 3.
          if (gcol >= p.out_cols) continue;
          if (vec_ok && grow + 4 <= p.out_rows) {
            *reinterpret_cast<uint2 *>(p.out + gcol * p.out_ld + grow) = make_uint2(h01, h23);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (grow + e < p.out_rows) p.out[gcol * p.out_ld + grow + e] = h[e];
          }
        }
      }
    }
    cluster_sync_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS) : "memory");
  }
}

// ---- host side ------------------------------------------------------------

template <class C>
cudaError_t launch(const TcParams &p, int grid_n, int grid_m, cudaStream_t stream, int split = 1,
                   bool pdl = false) {
  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(tc_kernel<C>), static_cast<int>(C::SMEM_BYTES),
                                configured);
  if (e != cudaSuccess) return e;
  if (grid_n <= 0 || grid_m <= 0) return cudaSuccess;
  if (split < 1 || !C::SPLIT) split = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid_n, grid_m, split);
  cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (C::SPLIT) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = static_cast<unsigned>(split);
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = na ? attr : nullptr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, tc_kernel<C>, p);
  if (e == cudaSuccess) count_launches(1);
  return e;
}

// Split of the contraction for a product with `tiles` output tiles and
// `ksteps` k-steps: fill about `per_sm` CTAs per SM (two for the skinny
// products, which fit two to an SM; one for the input gradient), at least two
// k-steps per CTA, at most 8 CTAs per cluster.
int choose_split(int64_t tiles, int ksteps, int per_sm = 2) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t sp = (static_cast<int64_t>(per_sm) * sms) / (tiles > 0 ? tiles : 1);
  if (sp > 8) sp = 8;
  if (sp > ksteps / 2) sp = ksteps / 2;
  return sp < 1 ? 1 : static_cast<int>(sp);
}

int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

using CfgFwd1 = Cfg<256, 1, false, true, false, false>;
using CfgFwd1S = Cfg<256, 1, false, true, false, false, true>;
using CfgBwd1 = Cfg<256, 1, false, true, true, false>;
using CfgBwd1S = Cfg<256, 1, false, true, true, false, true>;
using CfgProjK = Cfg<64, 1, false, false, false, false, true>;
using CfgProjMN = Cfg<64, 1, false, false, true, false, true>;
using CfgTN = Cfg<64, 1, true, false, true, false, true>;
using CfgTNT = Cfg<64, 1, true, false, true, true, true>;
using CfgDropAdd = Cfg<256, 1, false, false, true, false, false, kEpiDropoutAdd>;

}  // namespace

cudaError_t tc_fwd(const uint16_t *X, int64_t m, const WeightView &w, const uint16_t *T, const uint16_t *B,
                   int32_t r, uint16_t *Y, cudaStream_t stream, bool pdl) {
  // Above 128 rows: the 256 x 256 kernel with separate operand rings.
  if (m > 128) return fused_fwd_large(X, m, w, T, B, r, Y, stream, pdl);
  TcParams p{};
  const uint32_t bm = 128u;
  const bool lora = T != nullptr && B != nullptr && r > 0;
  if (!encode_bf16_map(&p.tmA, X, m, w.k, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_codes_map(&p.tmCodes, w.codes, w.n, w.k / 2, 32, 256, false)) return cudaErrorInvalidValue;
  if (lora) {
    if (!encode_bf16_map(&p.tmA2, T, m, r, 64, 128)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&p.tmB2, B, w.n, r, 64, 256)) return cudaErrorInvalidValue;
  }
  p.absmax_q = w.absmax_q;
  p.group_scale = w.group_scale;
  p.mu = w.mu;
  p.out = Y;
  p.err = device_error_word();
  p.w_n = w.n;
  p.w_k = w.k;
  p.out_ld = w.n;
  p.out_rows = static_cast<int>(m);
  p.out_cols = static_cast<int>(w.n);
  p.num_main = static_cast<int>(w.k / 64);
  p.num_lora = lora ? cdiv(r, 64) : 0;
  p.pdl = (lora && pdl) ? 1 : 0;
  p.alpha = 1.0f;
  p.tab = *w.tab;
  const int gn = cdiv(w.n, 256), gm = cdiv(m, bm);
  // Few 256-row weight tiles leave SMs idle: split the contraction over a
  // cluster (the adapter k-steps go to its last CTA).
  const int sp = choose_split(int64_t(gn) * gm, p.num_main, 1);
  return sp > 1 ? launch<CfgFwd1S>(p, gn, gm, stream, sp, p.pdl != 0)
                : launch<CfgFwd1>(p, gn, gm, stream, 1, p.pdl != 0);
}

cudaError_t tc_bwd_dx(const uint16_t *dY, int64_t m, const WeightView &w, const uint16_t *U, const uint16_t *A,
                      int32_t r, uint16_t *dX, cudaStream_t stream, bool pdl) {
  // Above 128 rows: the CTA-pair kernel.
  if (m > 128) return fused_bwd_dx_large(dY, m, w, U, A, r, dX, stream, pdl);
  TcParams p{};
  const uint32_t bm = 128u;
  const bool lora = U != nullptr && A != nullptr && r > 0;
  if (!encode_bf16_map(&p.tmA, dY, m, w.n, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_codes_map(&p.tmCodes, w.codes, w.n, w.k / 2, 32, 64, false)) return cudaErrorInvalidValue;
  if (lora) {
    if (!encode_bf16_map(&p.tmA2, U, m, r, 64, 128)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&p.tmB2, A, r, w.k, 64, 64)) return cudaErrorInvalidValue;
  }
  p.absmax_q = w.absmax_q;
  p.group_scale = w.group_scale;
  p.mu = w.mu;
  p.out = dX;
  p.err = device_error_word();
  p.w_n = w.n;
  p.w_k = w.k;
  p.out_ld = w.k;
  p.out_rows = static_cast<int>(m);
  p.out_cols = static_cast<int>(w.k);
  p.num_main = cdiv(w.n, 64);
  p.num_lora = lora ? cdiv(r, 64) : 0;
  p.pdl = (lora && pdl) ? 1 : 0;
  p.alpha = 1.0f;
  p.tab = *w.tab;
  const int gn = cdiv(w.k, 256), gm = cdiv(m, bm);
  // One 128-row tile per 256 columns leaves most SMs idle at small m: the
  // contraction over the weight rows is split over a cluster instead.
  const int sp = choose_split(int64_t(gn) * gm, p.num_main, 1);
  return sp > 1 ? launch<CfgBwd1S>(p, gn, gm, stream, sp, p.pdl != 0)
                : launch<CfgBwd1>(p, gn, gm, stream, 1, p.pdl != 0);
}

cudaError_t tc_proj_kmajor(const uint16_t *L, int64_t m, int64_t kc, const uint16_t *R, int32_t r, float scale,
                           uint16_t *out, cudaStream_t stream) {
  TcParams p{};
  if (!encode_bf16_map(&p.tmA, L, m, kc, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_bf16_map(&p.tmB, R, r, kc, 64, 64)) return cudaErrorInvalidValue;
  p.out = out;
  p.err = device_error_word();
  p.out_ld = r;
  p.out_rows = static_cast<int>(m);
  p.out_cols = r;
  p.num_main = cdiv(kc, 64);
  p.num_lora = 0;
  p.alpha = scale;
  const int gn = cdiv(r, 64), gm = cdiv(m, 128);
  return launch<CfgProjK>(p, gn, gm, stream, choose_split(int64_t(gn) * gm, p.num_main));
}

cudaError_t tc_proj_mnmajor(const uint16_t *L, int64_t m, int64_t kc, const uint16_t *R, int32_t r, float scale,
                            uint16_t *out, cudaStream_t stream) {
  TcParams p{};
  if (!encode_bf16_map(&p.tmA, L, m, kc, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_bf16_map(&p.tmB, R, kc, r, 64, 64)) return cudaErrorInvalidValue;
  p.out = out;
  p.err = device_error_word();
  p.out_ld = r;
  p.out_rows = static_cast<int>(m);
  p.out_cols = r;
  p.num_main = cdiv(kc, 64);
  p.num_lora = 0;
  p.alpha = scale;
  const int gn = cdiv(r, 64), gm = cdiv(m, 128);
  return launch<CfgProjMN>(p, gn, gm, stream, choose_split(int64_t(gn) * gm, p.num_main));
}

cudaError_t tc_tn_skinny(const uint16_t *Lt, int64_t mc, int64_t pdim, const uint16_t *R, int32_t r, uint16_t *out,
                         bool transposed, cudaStream_t stream) {
  TcParams p{};
  if (!encode_bf16_map(&p.tmA, Lt, mc, pdim, 64, 64)) return cudaErrorInvalidValue;
  if (!encode_bf16_map(&p.tmB, R, mc, r, 64, 64)) return cudaErrorInvalidValue;
  p.out = out;
  p.err = device_error_word();
  p.out_ld = transposed ? pdim : r;
  p.out_rows = static_cast<int>(pdim);
  p.out_cols = r;
  p.num_main = cdiv(mc, 64);
  p.num_lora = 0;
  p.alpha = 1.0f;
  const int gn = cdiv(r, 64), gm = cdiv(pdim, 128);
  const int sp = choose_split(int64_t(gn) * gm, p.num_main);
  return transposed ? launch<CfgTNT>(p, gn, gm, stream, sp) : launch<CfgTN>(p, gn, gm, stream, sp);
}

}  // namespace qlora

namespace qlora {

// dX[m x k] = bf16(dX + D . (U . A) . keep_scale): U [m x r] (K-major), A [r x k]
// (MN-major), the mask regenerated from (seed, offset) over dX's flat index.
cudaError_t tc_dropout_add(const uint16_t *U, int64_t m, int32_t r, const uint16_t *A, int64_t k,
                           const DropoutParams &d, uint16_t *dX, cudaStream_t stream) {
  TcParams p{};
  if (!encode_bf16_map(&p.tmA, U, m, r, 64, 128)) return cudaErrorInvalidValue;
  if (!encode_bf16_map(&p.tmB, A, r, k, 64, 64)) return cudaErrorInvalidValue;
  p.out = dX;
  p.err = device_error_word();
  p.out_ld = k;
  p.out_rows = static_cast<int>(m);
  p.out_cols = static_cast<int>(k);
  p.num_main = cdiv(r, 64);
  p.num_lora = 0;
  p.alpha = 1.0f;
  p.drop = d;
  return launch<CfgDropAdd>(p, cdiv(k, 256), cdiv(m, 128), stream);
}

}  // namespace qlora
