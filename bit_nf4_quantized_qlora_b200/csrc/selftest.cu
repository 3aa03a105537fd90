// Self-tests of the library's device-side guards, exported for test suites.
//
// qlora_selftest_bounded_wait runs the bounded mbarrier wait every pipelined
// kernel uses on a barrier that nothing arrives at, so the wait runs out, sets
// its bit in the device error word and returns: the path a kernel takes when
// a copy or an MMA it waits for never completes, exercised without any fault.
// qlora_selftest_div255 compares the library's fp32(s / 255) (Markstein's
// correctly rounded division, used by the decode and merge kernels) with IEEE
// division on a range of fp32 bit patterns.
#include "../../include/qlora.h"
#include "common.cuh"
#include "internal.h"

namespace qlora {
namespace {

__global__ void bounded_wait_kernel(unsigned *err, uint64_t limit_ns, unsigned *expired) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) mbar_init(&bar, 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    // Phase 0 never completes: no thread arrives and no copy is in flight.
    const bool ok = mbar_wait_bounded(&bar, 0u, err, kErrTimeoutSelfTest, limit_ns);
    if (expired) *expired = ok ? 0u : 1u;
  }
}

__global__ void div255_kernel(uint32_t first_bits, uint32_t count, unsigned long long *mismatches) {
  unsigned long long local = 0;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x) {
    const float s = __uint_as_float(first_bits + i);
    local += __float_as_uint(div255_rn(s)) != __float_as_uint(__fdiv_rn(s, 255.0f)) ? 1ull : 0ull;
  }
  if (local) atomicAdd(mismatches, local);
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" int qlora_selftest_bounded_wait(uint64_t limit_ns, unsigned *expired, qlora_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 2000000000ull) return QLORA_ERR_SHAPE;
  if (expired && (reinterpret_cast<uintptr_t>(expired) & 3u) != 0) return QLORA_ERR_ALIGN;
  int st = check_device();
  if (st != QLORA_OK) return st;
  unsigned *err = device_error_word();
  if (!err) return status_from_cuda(cudaErrorInvalidSymbol);
  bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err, limit_ns, expired);
  count_launches(1);
  return status_from_cuda(cudaGetLastError());
}

extern "C" int qlora_selftest_div255(uint32_t first_bits, uint32_t count, unsigned long long *mismatches,
                                     qlora_stream_t stream) {
  if (!mismatches) return QLORA_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(mismatches) & 7u) != 0) return QLORA_ERR_ALIGN;
  if (count == 0 || static_cast<uint64_t>(first_bits) + count > 0x7F800000ull) return QLORA_ERR_SHAPE;
  int st = check_device();
  if (st != QLORA_OK) return st;
  div255_kernel<<<4 * 148, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(first_bits, count, mismatches);
  count_launches(1);
  return status_from_cuda(cudaGetLastError());
}

constexpr bool same_bit(unsigned kernel_bit, unsigned header_bit) { return kernel_bit == header_bit; }
static_assert(same_bit(qlora::kErrTimeoutFullA, QLORA_DEVERR_OPERANDS) &&
                  same_bit(qlora::kErrTimeoutFullB, QLORA_DEVERR_WEIGHT_TILE) &&
                  same_bit(qlora::kErrTimeoutEmpty, QLORA_DEVERR_FREE_STAGE) &&
                  same_bit(qlora::kErrTimeoutAcc, QLORA_DEVERR_ACCUMULATOR) &&
                  same_bit(qlora::kErrTimeoutDrain, QLORA_DEVERR_DRAIN) &&
                  same_bit(qlora::kErrTimeoutSelfTest, QLORA_DEVERR_SELFTEST),
              "device error bits of the kernels and of the C header");
