// Adapter merge: W' = W^ + s . B . A, exported as bf16 and/or fp32.
//
// "QLoRA", Training setup versus deployment setup and Common misconception:
// the adapter folds back into the frozen weight; the only base a quantized
// checkpoint has is W^ = bf16(fp32(L[code] * c')).  W' is formed in fp32 with
// one fused multiply-add, W^ + s * acc, acc the fp32 sum of the rank-r
// product, and rounded once to bf16 for the bf16 export.
//
// The output is cut into tiles of 128 rows x 128 columns (8 warps of 32 x 64
// per tile), and every CTA that fits on the GPU at once takes an equal run of
// them in band-major order, so a run crosses into a new band of 128 rows at
// most once or twice.  The band's 128 rows of B stay in shared memory; each
// tile's r x 128 slice of A (rows padded to 272 bytes), its code bytes and its
// 256 block constants c' go through a double buffer filled by asynchronous
// 16-byte copies one tile ahead, so the copies of the next tile run under the
// current tile's MMAs and epilogue.  Each warp accumulates B . A on m16n8k16
// tensor-core MMAs (A operand = rows of B as 32-bit words, B operand =
// columns of A by ldmatrix.trans, two n8 tiles per load, shared by the warp's
// two m16 tiles).  Each row of a warp's piece is one NF4 block, so the
// epilogue decodes it through one per-row bf16 table of the block's 16
// scaled levels (byte permutes, no per-element lookups), adds s . acc in
// fp32, and writes 16 rows at a time through a shared-memory stage as
// 16-byte row segments.  The floor is HBM on the output writes (2 or 4 bytes
// per weight against 0.52 read); what bounds it is instruction issue.
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

constexpr int kTM = 128, kTN = 128;
constexpr int kWarps = 8, kThreads = 32 * kWarps;
constexpr int kMaxR = 256;

struct MergeParams {
  const uint8_t *codes;
  const uint8_t *absmax_q;
  const float *group_scale;
  const float *mu;          // E4M3 + mean absmax format: the tensor mean; else null
  const uint16_t *A;      // [r x k]
  const uint16_t *B;      // [n x r]
  uint16_t *out_bf16;     // [n x k] or null
  float *out_f32;         // [n x k] or null
  int64_t n, k;
  int r;
  int nbuf;               // tile buffers in shared memory (2: copies one tile ahead)
  float scale;
  Nf4Tables tab;
};

// Shared-memory layout (bytes), for rank r.  Padding puts the 32 lanes of
// each access pattern in 32 distinct banks:
//   rows of B, r/2 + 4 words: fragment reads (rows g, words q) hit 4g + q;
//   rows of the A slice, 256 + 16 bytes: the eight 16-byte rows of an
//     ldmatrix piece start four banks apart;
//   rows of code bytes, 80 bytes: rows g start at banks 20g mod 32;
//   stage rows, 36 words (bf16 pairs) or 72 words (fp32): stores of rows g
//     hit 4g + 4t + q, or 8g + 8t + 2q per half-warp.
constexpr uint32_t kARowBytes = kTN * 2u + 16u;
constexpr uint32_t kCodeRow = 80u;
constexpr int kStageH = 36, kStageF = 72;                 // words per stage row
constexpr uint32_t kStageWarpBytes = 16u * kStageF * 4u;  // 16 rows, the larger of the two
constexpr uint32_t kSmemCap = 227u * 1024u;
struct Layout {
  uint32_t row_words, bs, buf, at, codes, cp, buf_bytes, stage, total;
  __host__ __device__ Layout(int r, int nbuf) {
    row_words = static_cast<uint32_t>(r / 2 + 4);
    bs = 0;
    // Per-tile buffer (two of them): A slice, code bytes, block constants.
    buf = (bs + kTM * row_words * 4u + 15u) & ~15u;
    at = 0;
    codes = at + static_cast<uint32_t>(r) * kARowBytes;
    cp = codes + kTM * kCodeRow;
    buf_bytes = (cp + kTM * 2 * 4u + 15u) & ~15u;
    stage = buf + static_cast<uint32_t>(nbuf) * buf_bytes;
    total = stage + kWarps * kStageWarpBytes;
  }
};

// 16-byte global -> shared copy that bypasses registers (zeros when !valid;
// src is then a valid address that is not read).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

template <bool F32>
__global__ void __launch_bounds__(kThreads, 2) merge_kernel(const __grid_constant__ MergeParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  const Layout L(p.r, p.nbuf);
  uint32_t *bs = reinterpret_cast<uint32_t *>(sm + L.bs);
  const uint32_t sbase = smem_u32(sm);

  // This CTA's run of tiles in band-major order: [t_begin, t_end) of
  // bands x tiles_k, split evenly over the grid.
  const int tiles_k = static_cast<int>((p.k + kTN - 1) / kTN);
  const int64_t bands = (p.n + kTM - 1) / kTM;
  const int64_t total = bands * tiles_k;
  const int64_t t_begin = total * blockIdx.x / gridDim.x;
  const int64_t t_end = total * (blockIdx.x + 1) / gridDim.x;
  const int tid = threadIdx.x;
  const int rw = static_cast<int>(L.row_words);
  const int chunks_r = p.r / 8;   // 16-byte pieces of a row of B

  // The band's 128 rows of B (a padded row is 2r + 16 bytes, a multiple of
  // 16); zeros past n.
  const auto issue_band = [&](int64_t n0) {
    for (int i = tid; i < kTM * chunks_r; i += kThreads) {
      const int row = i / chunks_r, c = i % chunks_r;
      const bool ok = n0 + row < p.n;
      cp_async16(sbase + L.bs + static_cast<uint32_t>(row * rw + 4 * c) * 4u,
                 ok ? static_cast<const void *>(p.B + (n0 + row) * p.r + 8 * c) : p.B, ok);
    }
  };
  // One tile's r x 128 slice of A (row-major) and code bytes (128 rows x 64
  // bytes) into buffer `b`; zeros past n and k.
  const auto issue_tile = [&](int64_t n0, int ct, int b) {
    const int64_t c0 = static_cast<int64_t>(ct) * kTN;
    const uint32_t bb = sbase + L.buf + static_cast<uint32_t>(b) * L.buf_bytes;
    for (int i = tid; i < p.r * (kTN / 8); i += kThreads) {
      const int j = i / (kTN / 8), c = i % (kTN / 8);
      const bool ok = c0 + 8 * c < p.k;
      cp_async16(bb + L.at + static_cast<uint32_t>(j) * kARowBytes + 16u * c,
                 ok ? static_cast<const void *>(p.A + static_cast<int64_t>(j) * p.k + c0 + 8 * c) : p.A, ok);
    }
    for (int i = tid; i < kTM * 4; i += kThreads) {
      const int row = i >> 2, c = i & 3;
      const bool ok = n0 + row < p.n && c0 + 32 * c < p.k;
      cp_async16(bb + L.codes + static_cast<uint32_t>(row) * kCodeRow + 16u * c,
                 ok ? static_cast<const void *>(p.codes + ((n0 + row) * p.k + c0) / 2 + 16 * c) : p.codes, ok);
    }
  };
  const bool fp8 = p.mu != nullptr;
  const float mu = load_mu(p.mu);
  // W' = fma(s, acc, W^).  Without an adapter the sum starts at -0 and s is
  // 1, which returns W^ exactly (-0 + x = x for every x, FP4's -0 level
  // included), so no element needs a branch.
  const float acc0 = p.r > 0 ? 0.f : -0.f;
  const float s_eff = p.r > 0 ? p.scale : 1.f;
  // c' of this thread's block of a tile (row tid / 2, block tid % 2).
  const auto cprime = [&](int64_t n0, int ct) {
    const int row = tid >> 1, b = tid & 1;
    const int64_t c0 = static_cast<int64_t>(ct) * kTN;
    float c = 0.f;
    if (n0 + row < p.n && c0 + 64 * b < p.k) {
      const int64_t blk = ((n0 + row) * p.k + c0) / 64 + b;
      const float sg = __ldg(p.group_scale + (blk >> 8));
      c = block_constant(__ldg(p.absmax_q + blk), fp8 ? sg : div255_rn(sg), fp8, mu);
    }
    return c;
  };
  float c_next = 0.f;
  if (t_begin < t_end) {
    const int64_t n0 = (t_begin / tiles_k) * kTM;
    const int ct = static_cast<int>(t_begin % tiles_k);
    issue_band(n0);
    issue_tile(n0, ct, 0);
    c_next = cprime(n0, ct);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");

  // Copy groups: each tile's copies are one group, committed either at the
  // top of the tile before it (a prefetch within the band, two buffers) or at
  // the end of that tile (a new band, whose rows of B replace the old ones
  // once every warp is done with them, or a single buffer).  Every top
  // commits a group (possibly empty), so waiting for all but the newest
  // group finds this tile's copies done.
  for (int64_t tile = t_begin, it = 0; tile < t_end; ++tile, ++it) {
    const int b = p.nbuf == 2 ? static_cast<int>(it & 1) : 0;
    const int64_t band = tile / tiles_k;
    const int64_t n0 = band * kTM;
    const int ct = static_cast<int>(tile % tiles_k);
    const bool has_next = tile + 1 < t_end;
    const bool same_band = has_next && (tile + 1) / tiles_k == band;
    const bool prefetch = p.nbuf == 2 && same_band;
    uint8_t *cs = sm + L.buf + static_cast<uint32_t>(b) * L.buf_bytes + L.codes;
    float *cp = reinterpret_cast<float *>(sm + L.buf + static_cast<uint32_t>(b) * L.buf_bytes + L.cp);
    cp[tid] = c_next;
    // The next tile's copies run under this tile's MMAs and epilogue.
    if (prefetch) issue_tile(n0, ct + 1, b ^ 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (prefetch) c_next = cprime(n0, ct + 1);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const int64_t c0 = static_cast<int64_t>(ct) * kTN;
    const uint32_t at_base = L.buf + static_cast<uint32_t>(b) * L.buf_bytes + L.at;

    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const int rg = warp & 3, ch = warp >> 2;   // rows 32 rg .. +32, columns 64 ch .. +64
    float acc[2][8][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[mt][t][0] = acc[mt][t][1] = acc[mt][t][2] = acc[mt][t][3] = acc0;
    const uint32_t *ar[2] = {bs + (32 * rg + g) * rw, bs + (32 * rg + 16 + g) * rw};
    // ldmatrix.x4.trans for n8 tiles t, t + 1: lane l addresses row (l & 7) of
    // piece l >> 3; pieces 0 / 1 are k rows 0..7 / 8..15 of tile t (its b0 /
    // b1), pieces 2 / 3 the same of tile t + 1.
    const uint32_t lm_row = static_cast<uint32_t>(((lane >> 3) & 1) * 8 + (lane & 7));
    const uint32_t lm_col = static_cast<uint32_t>(64 * ch + (lane >> 4) * 8);
    const uint32_t lm_base = smem_u32(sm) + at_base + lm_row * kARowBytes + 2u * lm_col;
    for (int kk = 0; kk < p.r / 16; ++kk) {
      uint32_t a[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        a[mt][0] = ar[mt][8 * kk + q];
        a[mt][1] = ar[mt][8 * rw + 8 * kk + q];
        a[mt][2] = ar[mt][8 * kk + 4 + q];
        a[mt][3] = ar[mt][8 * rw + 8 * kk + 4 + q];
      }
#pragma unroll
      for (int t = 0; t < 8; t += 2) {
        uint32_t b[4];
        const uint32_t addr = lm_base + static_cast<uint32_t>(kk) * 16u * kARowBytes + 16u * static_cast<uint32_t>(t);
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                     : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                     : "r"(addr));
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          mma_bf16_16816(acc[mt][t], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b[0], b[1]);
          mma_bf16_16816(acc[mt][t + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b[2], b[3]);
        }
      }
    }

    // Epilogue.  Each row of the warp's 32 x 64 piece is one NF4 block, so a
    // lane decodes its row's codes through one per-row bf16 table: lane (g, q)
    // holds columns 8t + 2q, 8t + 2q + 1 of n8 tiles t = 0..7, whose shared
    // code byte is byte q of word t of the row's 32 code bytes (high nibble
    // first).  The lane gathers those eight bytes into two words and expands
    // them into the eight bf16 pairs of W^ in tile order.
    float *stage = reinterpret_cast<float *>(sm + L.stage + static_cast<uint32_t>(warp) * kStageWarpBytes);
    uint32_t *stage_h = reinterpret_cast<uint32_t *>(stage);
    const uint32_t sel_q = static_cast<uint32_t>(q) | (static_cast<uint32_t>(q + 4) << 4);
    const int64_t gcol0 = c0 + 64 * ch;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = 32 * rg + 16 * mt + g + 8 * h;
        const uint4 *crow = reinterpret_cast<const uint4 *>(cs + row * kCodeRow + 32 * ch);
        const uint4 v0 = crow[0], v1 = crow[1];
        const uint32_t wlo = prmt(prmt(v0.x, v0.y, sel_q), prmt(v0.z, v0.w, sel_q), 0x5410);
        const uint32_t whi = prmt(prmt(v1.x, v1.y, sel_q), prmt(v1.z, v1.w, sel_q), 0x5410);
        Bf16Table tb;
        make_table(p.tab, cp[row * 2 + ch], tb);
        uint32_t wv[8];
        decode8(wlo, tb, wv);
        decode8(whi, tb, wv + 4);
        const int lr = g + 8 * h;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float m0 = __fmaf_rn(s_eff, acc[mt][t][2 * h], bf16lo_to_f32(wv[t]));
          const float m1 = __fmaf_rn(s_eff, acc[mt][t][2 * h + 1], bf16hi_to_f32(wv[t]));
          if (F32)
            *reinterpret_cast<float2 *>(stage + lr * kStageF + 8 * t + 2 * q) = make_float2(m0, m1);
          else
            stage_h[lr * kStageH + 4 * t + q] = pack_bf16x2(m0, m1);
        }
      }
      __syncwarp();
      // 16 rows of 64 columns leave as 16-byte row segments.
      const int64_t grow0 = n0 + 32 * rg + 16 * mt;
      if (gcol0 < p.k) {
        if (F32) {
          // 16 rows x 256 bytes: lane l writes piece l & 15 of rows l / 16 + 2i.
          const int lr0 = lane >> 4, pc = lane & 15;
          float *dst = p.out_f32 + (grow0 + lr0) * p.k + gcol0 + 4 * pc;
          uint16_t *dsth = p.out_bf16 ? p.out_bf16 + (grow0 + lr0) * p.k + gcol0 + 4 * pc : nullptr;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int lr = lr0 + 2 * i;
            if (grow0 + lr < p.n) {
              const float4 v = *reinterpret_cast<const float4 *>(stage + lr * kStageF + 4 * pc);
              *reinterpret_cast<float4 *>(dst + 2 * i * p.k) = v;
              if (dsth) {
                uint2 hh;
                hh.x = pack_bf16x2(v.x, v.y);
                hh.y = pack_bf16x2(v.z, v.w);
                *reinterpret_cast<uint2 *>(dsth + 2 * i * p.k) = hh;
              }
            }
          }
        } else {
          // 16 rows x 128 bytes: lane l writes piece l & 7 of rows l / 8 + 4i.
          const int lr0 = lane >> 3, pc = lane & 7;
          uint16_t *dst = p.out_bf16 + (grow0 + lr0) * p.k + gcol0 + 8 * pc;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int lr = lr0 + 4 * i;
            if (grow0 + lr < p.n)
              *reinterpret_cast<uint4 *>(dst + 4 * i * p.k) =
                  *reinterpret_cast<const uint4 *>(stage_h + lr * kStageH + 4 * pc);
          }
        }
      }
      __syncwarp();   // the stage is rewritten by the next m16 tile
    }
    // Every warp is done with this tile's buffers (and the band's rows of B)
    // before they are refilled.
    __syncthreads();
    if (has_next && !prefetch) {
      const int64_t nn0 = ((tile + 1) / tiles_k) * kTM;
      const int nct = static_cast<int>((tile + 1) % tiles_k);
      if (!same_band) issue_band(nn0);
      issue_tile(nn0, nct, p.nbuf == 2 ? b ^ 1 : 0);
      asm volatile("cp.async.commit_group;" ::: "memory");
      c_next = cprime(nn0, nct);
    }
  }
}

}  // namespace

cudaError_t launch_merge(const WeightView &w, const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                         uint16_t *out_bf16, float *out_f32, cudaStream_t stream) {
  if (r < 0 || r > kMaxR || r % 16 != 0) return cudaErrorInvalidValue;
  MergeParams p{};
  p.codes = w.codes;
  p.absmax_q = w.absmax_q;
  p.group_scale = w.group_scale;
  p.mu = w.mu;
  p.A = r > 0 ? A : nullptr;
  p.B = r > 0 ? B : nullptr;
  p.out_bf16 = out_bf16;
  p.out_f32 = out_f32;
  p.n = w.n;
  p.k = w.k;
  p.r = r;
  p.scale = scale;
  p.tab = *w.tab;
  p.nbuf = Layout(r, 2).total <= kSmemCap ? 2 : 1;
  const uint32_t smem = Layout(r, p.nbuf).total;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // The limit is raised once per device to the most any rank uses, so
  // concurrent calls with different ranks never lower it under one another.
  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  static std::atomic<bool> configured_f32[kMaxDevicesPerProcess] = {};
  const void *fn = out_f32 ? reinterpret_cast<const void *>(merge_kernel<true>)
                           : reinterpret_cast<const void *>(merge_kernel<false>);
  e = set_smem_once(fn, static_cast<int>(kSmemCap), out_f32 ? configured_f32 : configured);
  if (e != cudaSuccess) return e;
  // Every CTA that fits at once takes an equal run of the bands x column
  // tiles, in band-major order.
  const int64_t tiles = ((w.n + kTM - 1) / kTM) * ((w.k + kTN - 1) / kTN);
  const int per_sm = smem <= kSmemCap / 2 ? 2 : 1;
  const int64_t slots = static_cast<int64_t>(per_sm) * sms;
  const dim3 grid(static_cast<unsigned>(tiles < slots ? tiles : slots), 1, 1);
  if (out_f32)
    merge_kernel<true><<<grid, kThreads, smem, stream>>>(p);
  else
    merge_kernel<false><<<grid, kThreads, smem, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
