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
