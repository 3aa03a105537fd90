// Device helpers shared by the kernels of libqlora (sm_100a only).
//
// NF4 decode used by every kernel that expands codes to bf16:
//   Per block of 64 weights the 16 possible outputs bf16_rne(fp32(L[i] * c'))
//   are computed once (16 multiplies, 8 packed conversions) and split into a
//   low-byte plane and a high-byte plane of four 32-bit words each.  A 32-bit
//   word of packed codes (8 weights) is then expanded with byte permutes:
//   the low three bits of each code select a byte from the 8-entry half
//   tables, bit 3 (replicated to a byte mask with the sign-replicate mode of
//   prmt) chooses between the two halves, and two more permutes interleave
//   the planes back into bf16 pairs.  No memory lookups, no divergence.
//   The packed order is byte j = (code[2j] << 4) | code[2j+1].
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "types.h"

namespace qlora {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// (a & ~m) | (b & m)
__device__ __forceinline__ uint32_t bitselect(uint32_t a, uint32_t b, uint32_t m) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xD8;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
  return d;
}

// Two fp32 -> packed bf16x2 (round to nearest even); `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Per-block bf16 output table in byte planes.
struct Bf16Table {
  uint32_t lo[4];  // lo[j] = low bytes of entries 4j .. 4j+3
  uint32_t hi[4];  // hi[j] = high bytes of entries 4j .. 4j+3
};

// c' = fp32(float(q) * fp32(S / 255)), with IEEE division and multiply.
__device__ __forceinline__ float absmax_dequant(uint32_t q, float S) {
  return __fmul_rn(static_cast<float>(q), __fdiv_rn(S, 255.0f));
}

// The fp32 value of an E4M3 bit pattern (1 sign, 4 exponent bits with bias
// 7, 3 mantissa bits; exponent field 0 holds m/8 * 2^-6), built from its bits.
__device__ __forceinline__ float e4m3_to_f32(uint32_t q) {
  const uint32_t e = (q >> 3) & 15u, m = q & 7u;
  const float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0x1p-9f;
  return (q & 0x80u) ? -mag : mag;
}

// The two storage formats of the block absmax (fp8 == false: linear 8-bit;
// true: E4M3 offsets from the tensor mean mu):
//   linear 8-bit:  t = fp32(S_g / 255),  c' = fp32(q * t)
//   E4M3 + mean:   t = S'_g (stored),    c' = fp32(fp32(E4M3(q) * t) + mu)
// Kernels carry the format as a pointer to mu, null for linear 8-bit.
__device__ __forceinline__ float group_constant(float stored, bool fp8) {
  return fp8 ? stored : __fdiv_rn(stored, 255.0f);
}
__device__ __forceinline__ float code_value(uint32_t q, bool fp8) {
  return fp8 ? e4m3_to_f32(q) : static_cast<float>(q);
}
__device__ __forceinline__ float block_constant(uint32_t q, float t, bool fp8, float mu) {
  return fp8 ? __fadd_rn(__fmul_rn(e4m3_to_f32(q), t), mu) : __fmul_rn(static_cast<float>(q), t);
}
__device__ __forceinline__ float load_mu(const float *mu) { return mu ? __ldg(mu) : 0.f; }

__device__ __forceinline__ void make_table(const Nf4Tables &tab, float cprime, Bf16Table &t) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    p[j] = pack_bf16x2(__fmul_rn(tab.level[2 * j], cprime), __fmul_rn(tab.level[2 * j + 1], cprime));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    t.lo[j] = prmt(p[2 * j], p[2 * j + 1], 0x6420);
    t.hi[j] = prmt(p[2 * j], p[2 * j + 1], 0x7531);
  }
}

// Expand one word of packed codes (8 weights, e0 first in memory) into four
// bf16x2 words in natural order: out[j] = {e_{2j} (bits 0..15), e_{2j+1}}.
__device__ __forceinline__ void decode8(uint32_t w, const Bf16Table &t, uint32_t out[4]) {
  // Nibble i of w holds: 0:e1 1:e0 2:e3 3:e2 4:e5 5:e4 6:e7 7:e6.
  const uint32_t sel = w & 0x77777777u;
  const uint32_t sel_hi = sel >> 16;
  const uint32_t w4 = w << 4;
  // Byte masks 0xFF where bit 3 of the code is set, in lookup order.
  const uint32_t m_lo = prmt(w, w4, 0x9D8C);
  const uint32_t m_hi = prmt(w, w4, 0xBFAE);
  // lookups for e1 e0 e3 e2
  uint32_t lo = bitselect(prmt(t.lo[0], t.lo[1], sel), prmt(t.lo[2], t.lo[3], sel), m_lo);
  uint32_t hi = bitselect(prmt(t.hi[0], t.hi[1], sel), prmt(t.hi[2], t.hi[3], sel), m_lo);
  out[0] = prmt(lo, hi, 0x4051);  // {e0, e1}
  out[1] = prmt(lo, hi, 0x6273);  // {e2, e3}
  // lookups for e5 e4 e7 e6
  lo = bitselect(prmt(t.lo[0], t.lo[1], sel_hi), prmt(t.lo[2], t.lo[3], sel_hi), m_hi);
  hi = bitselect(prmt(t.hi[0], t.hi[1], sel_hi), prmt(t.hi[2], t.hi[3], sel_hi), m_hi);
  out[2] = prmt(lo, hi, 0x4051);  // {e4, e5}
  out[3] = prmt(lo, hi, 0x6273);  // {e6, e7}
}

// ---------------------------------------------------------------------------
// Thread-block clusters, distributed shared memory, warp-level MMA
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster; orders shared-memory writes
// before the barrier with distributed reads after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// fp32 at `local_addr` in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// d += A(16x16, row) . B(16x8, col), bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A(16x16, row) . B(16x8, col) with a zero accumulator.
__device__ __forceinline__ void mma_bf16_16816_zero(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                    uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// Byte-pair table: entry b (two weights) holds {NF4[b >> 4], NF4[b & 15]} as a
// bf16 pair, in 32 lane-private copies 256 bytes apart (entry b of lane l at
// b * 256 + 4 l), so the 32 lookups of a warp always fall in 32 banks.
constexpr uint32_t kPairLutBytes = 256u * 256u;

__device__ __forceinline__ void build_pair_lut(uint8_t *lut, const Nf4Tables &tab, int tid, int nthreads) {
  uint4 *lw = reinterpret_cast<uint4 *>(lut);
  for (int i = tid; i < 256 * 16; i += nthreads) {
    const int b = i >> 4;
    const uint32_t v = pack_bf16x2(tab.level[b >> 4], tab.level[b & 15]);
    lw[i] = make_uint4(v, v, v, v);
  }
}

// Table offset of byte J (0..3) of `word` for the lane whose lane*4 is lane4.
template <int J>
__device__ __forceinline__ uint32_t pair_lut_off(uint32_t word, uint32_t lane4) {
  return prmt(word, lane4, 0x5504u | (J << 4));
}

// Byte J of w as an exact float (0..255).
template <int J>
__device__ __forceinline__ float byte_to_f32(uint32_t w) {
  return __uint_as_float(prmt(w, 0x4B000000u, 0x7650u | J)) - 8388608.0f;
}

// fp32(s / 255) correctly rounded: Markstein's division with the correctly
// rounded reciprocal y = RN(1/255): q0 = RN(s y), the remainder
// rho = s - 255 q0 is exact in one fma, and q0 + rho y rounds to the nearest
// quotient.  IEEE division below 2^-100, where the remainder could lose bits.
__device__ __forceinline__ float div255_rn(float s) {
  if (!(s >= 0x1p-100f)) return __fdiv_rn(s, 255.0f);
  const float y = 1.0f / 255.0f;
  const float q0 = __fmul_rn(s, y);
  const float rho = __fmaf_rn(-q0, 255.0f, s);
  return __fmaf_rn(rho, y, q0);
}

// ---------------------------------------------------------------------------
// mbarrier / fences / timers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete, for at most
// `limit_ns` nanoseconds.  Returns false (and sets `flag` in *err) on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, unsigned *err,
                                                  unsigned flag, uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && global_timer_ns() - t0 > limit_ns) {
      if (err) atomicOr(err, flag);
      return false;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm("mov.u32 %0, %laneid;" : "=r"(l));
  return l;
}

}  // namespace qlora
