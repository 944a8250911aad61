// Philox4x32-10 counter-based generator, library side (host and device).
//
// Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
// (SC'11). Ten rounds of
//   (c0,c1,c2,c3) <- (hi(B*c2) ^ c1 ^ k0, lo(B*c2), hi(A*c0) ^ c3 ^ k1, lo(A*c0))
// with A = 0xD2511F53 and B = 0xCD9E8D57. Between rounds the key advances by
// the Weyl increments (0x9E3779B9, 0xBB67AE85).
//
// The pages draw S, D_r, D_g and the dither at random but fix no generator.
// The library draws them from this counter-based stream:
// counter = (index_lo, index_hi, block, stream) under key = seed.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define QJL_HD __host__ __device__ __forceinline__
#else
#define QJL_HD inline
#endif

namespace qjl {

enum : uint32_t { kStreamGauss = 0, kStreamRademacher = 1, kStreamPerm = 2, kStreamDither = 3 };

struct U32x4 {
  uint32_t x, y, z, w;
};

QJL_HD void mul_hi_lo(uint32_t a, uint32_t b, uint32_t& hi, uint32_t& lo) {
  const uint64_t p = (uint64_t)a * (uint64_t)b;
  hi = (uint32_t)(p >> 32);
  lo = (uint32_t)p;
}

QJL_HD U32x4 philox(U32x4 ctr, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint32_t hA, lA, hB, lB;
    mul_hi_lo(0xD2511F53u, ctr.x, hA, lA);
    mul_hi_lo(0xCD9E8D57u, ctr.z, hB, lB);
    ctr = U32x4{hB ^ ctr.y ^ k0, lB, hA ^ ctr.w ^ k1, lA};
  }
  return ctr;
}

}  // namespace qjl
