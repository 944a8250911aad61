// Arithmetic shared by the key kernels: sm_100 packed-fp32 pair operations,
// bf16 sums of squares, Philox4x32-10 on four counters at once, and the
// Box-Muller dither.
#pragma once

#include <stdint.h>

#include "philox.h"

namespace qjl_km {

// ---- packed fp32 pair arithmetic (sm_100 f32x2) ----------------------------------------------

// (a, b) <- (a + b, a - b), both lanes of the pair
__device__ __forceinline__ void bfly2(float2& a, float2& b) {
  asm("{\n\t.reg .b64 x, y, s, d;\n\t"
      "mov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "add.rn.f32x2 s, x, y;\n\tsub.rn.f32x2 d, x, y;\n\t"
      "mov.b64 {%0, %1}, s;\n\tmov.b64 {%2, %3}, d;\n\t}"
      : "+f"(a.x), "+f"(a.y), "+f"(b.x), "+f"(b.y));
}

// a <- a * b
__device__ __forceinline__ void mul2(float2& a, float2 b) {
  asm("{\n\t.reg .b64 x, y;\n\t"
      "mov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "mul.rn.f32x2 x, x, y;\n\t"
      "mov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a.x), "+f"(a.y)
      : "f"(b.x), "f"(b.y));
}

// a <- fma(a, b, +0): the product, with an exact zero always +0
__device__ __forceinline__ void mulz2(float2& a, float2 b) {
  asm("{\n\t.reg .b64 x, y, z;\n\t"
      "mov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\tmov.b64 z, {%4, %4};\n\t"
      "fma.rn.f32x2 x, x, y, z;\n\t"
      "mov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a.x), "+f"(a.y)
      : "f"(b.x), "f"(b.y), "f"(0.f));
}

// a <- fma(b, a, c) pairwise
__device__ __forceinline__ void fma2(float2& a, float2 b, float2 c) {
  asm("{\n\t.reg .b64 x, y, z;\n\t"
      "mov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\tmov.b64 z, {%4, %5};\n\t"
      "fma.rn.f32x2 x, y, x, z;\n\t"
      "mov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a.x), "+f"(a.y)
      : "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
}

// a <- fma(sg, a, p) with the same sign sg on both lanes
__device__ __forceinline__ void sfma2(float2& a, float sg, float2 p) {
  asm("{\n\t.reg .b64 x, s, q;\n\t"
      "mov.b64 x, {%0, %1};\n\tmov.b64 s, {%2, %2};\n\tmov.b64 q, {%3, %4};\n\t"
      "fma.rn.f32x2 x, s, x, q;\n\t"
      "mov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a.x), "+f"(a.y)
      : "f"(sg), "f"(p.x), "f"(p.y));
}

// acc += a * a (pairwise)
__device__ __forceinline__ void sq_acc2(float2& acc, float2 a) {
  asm("{\n\t.reg .b64 x, c;\n\t"
      "mov.b64 x, {%2, %3};\n\tmov.b64 c, {%0, %1};\n\t"
      "fma.rn.f32x2 c, x, x, c;\n\t"
      "mov.b64 {%0, %1}, c;\n\t}"
      : "+f"(acc.x), "+f"(acc.y)
      : "f"(a.x), "f"(a.y));
}

// acc += lo^2 + hi^2 for the two bf16 halves of u, with sm_100's mixed-precision
// FMA (bf16 operands widened exactly, fp32 accumulate): no unpacking.
__device__ __forceinline__ void sq_acc_bf16x2(uint32_t u, float& acc) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tfma.rn.f32.bf16 %0, lo, lo, %0;\n\t"
      "fma.rn.f32.bf16 %0, hi, hi, %0;\n\t}"
      : "+f"(acc)
      : "r"(u));
}

// ---- dither ------------------------------------------------------------------------------------

// Box-Muller on the two 16-bit halves of x, scaled by amp: (amp r cos 2 pi v, amp r sin 2 pi v)
// with r = sqrt(-2 ln u), u = ((x & 0xFFFF) + 1/2) 2^-16 from the low half and v = (x >> 16) 2^-16
// from the high half. A byte permute puts a half under the exponent of 1.0, h = 1 + k 2^-23,
// and one FMA rescales it exactly: u = 128 h - (128 - 2^-17) = (2k + 1) 2^-17 (the constant has
// 24 significant bits, the product and the sum are exact), and the angle 256 pi (h - 1) =
// 2 pi k 2^-16 carries one rounding of 256 pi and one of the product.
__device__ __forceinline__ float2 box_muller16(uint32_t x, float amp) {
  const float hu = __uint_as_float(__byte_perm(x, 0x3f800000u, 0x7610));  // 1 + (x & 0xFFFF) 2^-23
  const float hv = __uint_as_float(__byte_perm(x, 0x3f800000u, 0x7632));  // 1 + (x >> 16) 2^-23
  const float u = fmaf(hu, 128.f, -127.99999237060546875f);
  const float th = fmaf(hv, 804.247741699f, -804.247741699f);
  float l, rt, sn, cs;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(u));
  // sqrt(-2 ln u) = sqrt(-log2 u) sqrt(2 ln 2); the negation can ride on the sqrt's operand
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(rt) : "f"(-l));
  const float r = rt * (amp * 1.17741002f);
  asm("sin.approx.ftz.f32 %0, %1;" : "=f"(sn) : "f"(th));
  asm("cos.approx.ftz.f32 %0, %1;" : "=f"(cs) : "f"(th));
  return make_float2(r * cs, r * sn);
}

// acc <- acc + dither: the Box-Muller pair of x (box_muller16) scaled by amp, with the radius
// multiplying both outputs in one packed FMA
__device__ __forceinline__ void add_box_muller16(float2& acc, uint32_t x, float amp) {
  const float hu = __uint_as_float(__byte_perm(x, 0x3f800000u, 0x7610));
  const float hv = __uint_as_float(__byte_perm(x, 0x3f800000u, 0x7632));
  const float u = fmaf(hu, 128.f, -127.99999237060546875f);
  const float th = fmaf(hv, 804.247741699f, -804.247741699f);
  float l, rt, sn, cs;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(u));
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(rt) : "f"(-l));
  const float r = rt * (amp * 1.17741002f);
  asm("sin.approx.ftz.f32 %0, %1;" : "=f"(sn) : "f"(th));
  asm("cos.approx.ftz.f32 %0, %1;" : "=f"(cs) : "f"(th));
  asm("{\n\t.reg .b64 a, rr, cs;\n\t"
      "mov.b64 a, {%0, %1};\n\tmov.b64 rr, {%2, %2};\n\tmov.b64 cs, {%3, %4};\n\t"
      "fma.rn.f32x2 a, rr, cs, a;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "+f"(acc.x), "+f"(acc.y)
      : "f"(r), "f"(cs), "f"(sn));
}

// a <- a + b pairwise
__device__ __forceinline__ void add2(float2& a, float2 b) {
  asm("{\n\t.reg .b64 x, y;\n\t"
      "mov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "add.rn.f32x2 x, x, y;\n\t"
      "mov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a.x), "+f"(a.y)
      : "f"(b.x), "f"(b.y));
}

// Philox4x32-10 on N counters at once, rounds interleaved for instruction-level parallelism.
template <int N>
__device__ __forceinline__ void philox_xn(qjl::U32x4 (&c)[N], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      uint32_t hA, lA, hB, lB;
      qjl::mul_hi_lo(0xD2511F53u, c[j].x, hA, lA);
      qjl::mul_hi_lo(0xCD9E8D57u, c[j].z, hB, lB);
      c[j] = qjl::U32x4{hB ^ c[j].y ^ k0, lB, hA ^ c[j].w ^ k1, lA};
    }
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

// The same on round keys given as a table: rk[2 r], rk[2 r + 1] = the key after r bumps. A
// table in a kernel's parameters is read straight from the constant bank by the XORs.
template <int N>
__device__ __forceinline__ void philox_xn_rk(qjl::U32x4 (&c)[N], const uint32_t (&rk)[20]) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      uint32_t hA, lA, hB, lB;
      qjl::mul_hi_lo(0xD2511F53u, c[j].x, hA, lA);
      qjl::mul_hi_lo(0xCD9E8D57u, c[j].z, hB, lB);
      c[j] = qjl::U32x4{hB ^ c[j].y ^ rk[2 * r], lB, hA ^ c[j].w ^ rk[2 * r + 1], lA};
    }
  }
}

// Philox round keys of the key (k0, k1) as the table philox_xn_rk reads.
__host__ __device__ inline void philox_round_keys(uint32_t k0, uint32_t k1, uint32_t (&rk)[20]) {
  for (int r = 0; r < 10; ++r) {
    rk[2 * r] = k0 + (uint32_t)r * 0x9E3779B9u;
    rk[2 * r + 1] = k1 + (uint32_t)r * 0xBB67AE85u;
  }
}

__device__ __forceinline__ void philox_x4(qjl::U32x4 (&c)[4], uint32_t k0, uint32_t k1) { philox_xn<4>(c, k0, k1); }

}  // namespace qjl_km
