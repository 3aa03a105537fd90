// Adapter merge: W' = W^ + s . B . A, exported as bf16 and/or fp32.
//
// "QLoRA", Training setup versus deployment setup and Common misconception:
// the adapter folds back into the frozen weight; the only base a quantized
// checkpoint has is W^ = bf16(fp32(L[code] * c')).  W' is formed in fp32 with
// one fused multiply-add, W^ + s * acc, acc the fp32 sum of the rank-r
// product, and rounded once to bf16 for the bf16 export.
//
// One CTA per 128 x 128 tile of W', 8 warps of 32 x 64.  The CTA stages the
// tile's 128 rows of B [128 x r], its r x 128 slice of A (rows padded to 272
// bytes), the tile's code bytes and its 256 block constants c' in shared
// memory with asynchronous 16-byte copies; each warp accumulates B . A on m16n8k16
// tensor-core MMAs (A operand = rows of B as 32-bit words, B operand =
// columns of A by ldmatrix.trans, two n8 tiles per load, shared by the warp's
// two m16 tiles), then decodes the code byte of each accumulator pair (two
// neighbouring columns share one byte), adds, and writes its piece 16 rows
// at a time through a shared-memory stage as 16-byte row segments.  Bound by
// HBM on the output writes (2 or 4 bytes per weight against 0.52 read).
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
struct Layout {
  uint32_t row_words, bs, at, codes, cp, lv, stage, total;
  __host__ __device__ explicit Layout(int r) {
    row_words = static_cast<uint32_t>(r / 2 + 4);
    bs = 0;
    at = bs + kTM * row_words * 4u;
    codes = at + static_cast<uint32_t>(r) * kARowBytes;
    cp = codes + kTM * kCodeRow;
    lv = cp + kTM * 2 * 4u;
    stage = (lv + 16 * 4u + 15u) & ~15u;
    total = stage + kWarps * kStageWarpBytes;
  }
};

// 16-byte global -> shared copy that bypasses registers (zeros when !valid;
// src is then a valid address that is not read).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

__global__ void __launch_bounds__(kThreads) merge_kernel(const __grid_constant__ MergeParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  const Layout L(p.r);
  uint32_t *bs = reinterpret_cast<uint32_t *>(sm + L.bs);
  uint8_t *cs = sm + L.codes;
  float *cp = reinterpret_cast<float *>(sm + L.cp);
  float *lv = reinterpret_cast<float *>(sm + L.lv);

  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kTM;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTN;
  const int tid = threadIdx.x;
  const int rw = static_cast<int>(L.row_words);
  const int chunks_r = p.r / 8;   // 16-byte pieces of a row of B

  // Staging by asynchronous 16-byte copies, all in flight together: rows of B
  // (a padded row is 2r + 16 bytes, a multiple of 16), the r x 128 slice of
  // A row-major, the tile's code bytes (128 rows x 64 bytes); zeros past n
  // and k.
  const uint32_t sbase = smem_u32(sm);
  for (int i = tid; i < kTM * chunks_r; i += kThreads) {
    const int row = i / chunks_r, c = i % chunks_r;
    const bool ok = n0 + row < p.n;
    cp_async16(sbase + L.bs + static_cast<uint32_t>(row * rw + 4 * c) * 4u,
               ok ? static_cast<const void *>(p.B + (n0 + row) * p.r + 8 * c) : p.B, ok);
  }
  for (int i = tid; i < p.r * (kTN / 8); i += kThreads) {
    const int j = i / (kTN / 8), c = i % (kTN / 8);
    const bool ok = c0 + 8 * c < p.k;
    cp_async16(sbase + L.at + static_cast<uint32_t>(j) * kARowBytes + 16u * c,
               ok ? static_cast<const void *>(p.A + static_cast<int64_t>(j) * p.k + c0 + 8 * c) : p.A, ok);
  }
  for (int i = tid; i < kTM * 4; i += kThreads) {
    const int row = i >> 2, c = i & 3;
    const bool ok = n0 + row < p.n && c0 + 32 * c < p.k;
    cp_async16(sbase + L.codes + static_cast<uint32_t>(row) * kCodeRow + 16u * c,
               ok ? static_cast<const void *>(p.codes + ((n0 + row) * p.k + c0) / 2 + 16 * c) : p.codes, ok);
  }
  // c' of the tile's blocks (two per row).
  {
    const int row = tid >> 1, b = tid & 1;
    float c = 0.f;
    if (n0 + row < p.n && c0 + 64 * b < p.k) {
      const int64_t blk = ((n0 + row) * p.k + c0) / 64 + b;
      const bool fp8 = p.mu != nullptr;
      const float sg = __ldg(p.group_scale + (blk >> 8));
      c = block_constant(__ldg(p.absmax_q + blk), fp8 ? sg : div255_rn(sg), fp8, load_mu(p.mu));
    }
    cp[tid] = c;
  }
  if (tid < 16) lv[tid] = p.tab.level[tid];
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int rg = warp & 3, ch = warp >> 2;   // rows 32 rg .. +32, columns 64 ch .. +64
  float acc[2][8][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[mt][t][0] = acc[mt][t][1] = acc[mt][t][2] = acc[mt][t][3] = 0.f;
  const uint32_t *ar[2] = {bs + (32 * rg + g) * rw, bs + (32 * rg + 16 + g) * rw};
  // ldmatrix.x4.trans for n8 tiles t, t + 1: lane l addresses row (l & 7) of
  // piece l >> 3; pieces 0 / 1 are k rows 0..7 / 8..15 of tile t (its b0 /
  // b1), pieces 2 / 3 the same of tile t + 1.
  const uint32_t lm_row = static_cast<uint32_t>(((lane >> 3) & 1) * 8 + (lane & 7));
  const uint32_t lm_col = static_cast<uint32_t>(64 * ch + (lane >> 4) * 8);
  const uint32_t lm_base = smem_u32(sm) + L.at + lm_row * kARowBytes + 2u * lm_col;
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

  // Epilogue, one m16 tile at a time: lane (g, q) holds rows g, g + 8 and
  // columns 2q, 2q + 1 of each n8 tile t; the two columns share one code byte
  // (high nibble first).
  float *stage = reinterpret_cast<float *>(sm + L.stage + static_cast<uint32_t>(warp) * kStageWarpBytes);
  uint32_t *stage_h = reinterpret_cast<uint32_t *>(stage);
  const int64_t gcol0 = c0 + 64 * ch;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int col = 64 * ch + 8 * t + 2 * q;   // within the tile
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = 32 * rg + 16 * mt + g + 8 * h;
        const uint32_t byte = cs[row * kCodeRow + col / 2];
        const float c = cp[row * 2 + (col >> 6)];
        const float w0 = bf16lo_to_f32(pack_bf16x2(__fmul_rn(lv[byte >> 4], c), 0.f));
        const float w1 = bf16lo_to_f32(pack_bf16x2(__fmul_rn(lv[byte & 15u], c), 0.f));
        // Without an adapter W' is W^ itself (an added +0 would turn FP4's
        // -0 level into +0).
        const float m0 = p.r > 0 ? __fmaf_rn(p.scale, acc[mt][t][2 * h], w0) : w0;
        const float m1 = p.r > 0 ? __fmaf_rn(p.scale, acc[mt][t][2 * h + 1], w1) : w1;
        const int lr = g + 8 * h, lc = 8 * t + 2 * q;
        if (p.out_f32)
          *reinterpret_cast<float2 *>(stage + lr * kStageF + lc) = make_float2(m0, m1);
        else
          stage_h[lr * kStageH + lc / 2] = pack_bf16x2(m0, m1);
      }
    }
    __syncwarp();
    const int64_t grow0 = n0 + 32 * rg + 16 * mt;
    if (gcol0 < p.k) {
      if (p.out_f32) {
        // 16 rows x 256 bytes: 256 pieces of 16 bytes, 8 per lane.
        for (int i = lane; i < 256; i += 32) {
          const int lr = i >> 4, pc = i & 15;
          if (grow0 + lr >= p.n) continue;
          const float4 v = *reinterpret_cast<const float4 *>(stage + lr * kStageF + 4 * pc);
          *reinterpret_cast<float4 *>(p.out_f32 + (grow0 + lr) * p.k + gcol0 + 4 * pc) = v;
          if (p.out_bf16) {
            uint2 hh;
            hh.x = pack_bf16x2(v.x, v.y);
            hh.y = pack_bf16x2(v.z, v.w);
            *reinterpret_cast<uint2 *>(p.out_bf16 + (grow0 + lr) * p.k + gcol0 + 4 * pc) = hh;
          }
        }
      } else {
        // 16 rows x 128 bytes: 128 pieces of 16 bytes, 4 per lane.
        for (int i = lane; i < 128; i += 32) {
          const int lr = i >> 3, pc = i & 7;
          if (grow0 + lr >= p.n) continue;
          const uint4 v = *reinterpret_cast<const uint4 *>(stage_h + lr * kStageH + 4 * pc);
          *reinterpret_cast<uint4 *>(p.out_bf16 + (grow0 + lr) * p.k + gcol0 + 8 * pc) = v;
        }
      }
    }
    __syncwarp();   // the stage is rewritten by the next m16 tile
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
  const uint32_t smem = Layout(r).total;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // The limit is raised once per device to what the largest rank needs, so
  // concurrent calls with different ranks never lower it under one another.
  static std::atomic<bool> configured[kMaxDevicesPerProcess] = {};
  e = set_smem_once(reinterpret_cast<const void *>(merge_kernel), static_cast<int>(Layout(256).total), configured);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((w.k + kTN - 1) / kTN), static_cast<unsigned>((w.n + kTM - 1) / kTM), 1);
  merge_kernel<<<grid, kThreads, smem, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace qlora
