// Plain types shared by host and device code of libqlora.
#pragma once

#include <cstdint>

namespace qlora {

// The 4-bit codebooks a weight may be stored in (NF4, or one of the two
// uniform-bin baselines it is compared with).
enum : int { kCodebookNF4 = 0, kCodebookFP4 = 1, kCodebookINT4 = 2, kCodebookCount = 3 };

// How the block absmax constants are stored (double quantization): unsigned
// linear 8-bit codes with one fp32 max per group of 256, or E4M3 codes of the
// offsets from the tensor's mean with one fp32 scale per group and the mean
// after the group scales.
enum : int { kDqLinear8 = 0, kDqFp8Mean = 1, kDqFormatCount = 2 };

// The fp32 codebook and the 15 decision midpoints, passed by value as a
// kernel parameter (uniform across the grid).
struct Nf4Tables {
  float level[16];
  float mid[15];
  float pad_;
};

// The code of a quotient x in [-1, 1] by bucket: b = rn(15.4 x + 16), in
// [1, 31] (one fp32 FMA with the 1.5 * 2^23 rounding constant: b is the low
// bits of the result), then code = code[b] + (x > thr[b]), with code[b] the
// number of midpoints in lower buckets and thr[b] the next midpoint (+inf
// past the last).  The bucket index is monotone in x, so a midpoint in a
// lower bucket is below x and one in a higher bucket above it; this is exact
// when no bucket holds a second midpoint that some |x| <= 1 can exceed
// (ok == 1).  zero_mid: a midpoint is exactly 0, so the sign of a quotient
// below the normal range decides a code.
struct QuantBuckets {
  uint32_t code[32];
  float thr[32];
  int32_t ok;
  int32_t zero_mid;
};

// Device-side error codes written to the caller-visible error word when a
// bounded wait gives up (no kernel ever traps).
enum : unsigned {
  kErrTimeoutFullA = 1u << 0,
  kErrTimeoutFullB = 1u << 1,
  kErrTimeoutEmpty = 1u << 2,
  kErrTimeoutAcc = 1u << 3,
  kErrTimeoutDrain = 1u << 4,
  kErrTimeoutSelfTest = 1u << 5,
};

}  // namespace qlora
