// KIVI per-channel 2-bit keys: the like-for-like baseline of the QJL key
// sketch on the same shapes.
//
// KIVI abstract ("Vladimir Braverman" page, "KIVI: A Tuning-Free Asymmetric
// 2bit Quantization for KV Cache"): the key cache is quantised per channel and
// the value cache per token, both to 2 bits. A channel's group here is a block
// of 32 consecutive tokens of one key head (the last block of a ragged N is
// shorter). Per (block, channel): zero = fp16(min), scale =
// fp16(fp32(max - min) / 3), code = clamp(rint_even(fp32(fp32(k - zero) /
// scale)), 0, 3), or 0 when scale is 0, every step an IEEE round-to-nearest
// operation. Codes are stored per token like the values (channel c at bits
// 2*(c % 16) of word c / 16). That is 2 bits per channel plus 4 bytes of
// scale and zero per 32 tokens and channel: 48 bytes per key at d = 128,
// against m/8 + 4 = 36 for the QJL sketch at m = 256.
//
// Quantise: one warp per (key head, token block). Lane l owns channels
// CPL*l .. CPL*l + CPL - 1 (CPL = d/32), so each token row is one coalesced
// load. A first pass over the block's tokens takes min/max, a second (from
// L1) the codes. The 16/CPL lanes of a code word merge their bits with xor
// shuffles.
//
// Scores: <q, k_hat> = sum_c (q_c s_c) code_c + sum_c q_c z_c. One warp per
// (key head, token block, query) computes a_c = q_c s_c 4^-(c % 8) into shared
// memory and b = sum_c q_c z_c. Each lane then scores one key of the block.
// code * 4^(c % 8) comes out of the code word as float(2^23 | (chunk & mask))
// - 2^23 with no conversion instruction (the mask keeps the bits in the
// mantissa), and the 4^-(c % 8) in a_c undoes the weight exactly.

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "qjl_internal.h"

namespace {

constexpr int kKB = 32;        // tokens per block
constexpr int kKWarps = 8;

template <int DTYPE, int CPL>
__device__ __forceinline__ void load_cpl(const void* base, int64_t elem, float (&v)[CPL]) {
  if (DTYPE == QJL_F32) {
    const float* p = reinterpret_cast<const float*>(base) + elem;
#pragma unroll
    for (int i = 0; i < CPL; i += 2) {
      const float2 f = *reinterpret_cast<const float2*>(p + i);
      v[i] = f.x;
      v[i + 1] = f.y;
    }
  } else {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(base) + elem);
#pragma unroll
    for (int i = 0; i < CPL; i += 2) {
      const uint32_t w = p[i / 2];
      v[i] = __uint_as_float(w << 16);
      v[i + 1] = __uint_as_float(w & 0xFFFF0000u);
    }
  }
}

// element i (0..3) of four packed bf16 values, as fp32
__device__ __forceinline__ float bf16_lane(uint2 v, int i) {
  const uint32_t w = (i < 2) ? v.x : v.y;
  return __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

template <int DTYPE, int CPL>
__global__ void __launch_bounds__(kKWarps * 32) kivi_keys_quantize_kernel(const void* __restrict__ keys, int64_t G,
                                                                          int64_t N, uint32_t* __restrict__ codes,
                                                                          uint16_t* __restrict__ scale,
                                                                          uint16_t* __restrict__ zero) {
  constexpr int d = 32 * CPL;
  constexpr int LPW = 16 / CPL;  // lanes per 16-channel code word
  const int lane = threadIdx.x & 31;
  const int64_t nb = (N + kKB - 1) / kKB;
  const int64_t items = G * nb;
  const int c0 = CPL * lane;
  for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items;
       it += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t g = it / nb, b = it - (it / nb) * nb;
    const int64_t t0 = b * kKB;
    const int cnt = (int)min((int64_t)kKB, N - t0);
    const int64_t row0 = g * N + t0;
    // a whole bf16 block at d = 128 lives in registers (32 rows x 8 bytes per lane): all its row
    // loads are in flight at once, and the code pass reads no memory
    constexpr bool REG = DTYPE == QJL_BF16 && CPL == 4;
    const bool whole = REG && cnt == kKB;
    uint2 rowv[REG ? kKB : 1];
    float mn[CPL], mx[CPL];
    if (whole) {
#pragma unroll
      for (int t = 0; t < kKB; ++t)
        rowv[t] = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(keys) + (row0 + t) * d + c0));
#pragma unroll
      for (int i = 0; i < CPL; ++i) mn[i] = mx[i] = bf16_lane(rowv[0], i);
#pragma unroll
      for (int t = 1; t < kKB; ++t)
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
          mn[i] = fminf(mn[i], bf16_lane(rowv[t], i));
          mx[i] = fmaxf(mx[i], bf16_lane(rowv[t], i));
        }
    } else {
      {
        float v[CPL];
        load_cpl<DTYPE, CPL>(keys, row0 * d + c0, v);
#pragma unroll
        for (int i = 0; i < CPL; ++i) mn[i] = mx[i] = v[i];
      }
#pragma unroll 4
      for (int t = 1; t < cnt; ++t) {
        float v[CPL];
        load_cpl<DTYPE, CPL>(keys, (row0 + t) * d + c0, v);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
          mn[i] = fminf(mn[i], v[i]);
          mx[i] = fmaxf(mx[i], v[i]);
        }
      }
    }
    float zf[CPL], sf[CPL], yf[CPL];
    uint16_t zh[CPL], sh[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const __half z = __float2half_rn(mn[i]);
      const __half s = __float2half_rn(__fdiv_rn(__fsub_rn(mx[i], mn[i]), 3.0f));
      zf[i] = __half2float(z);
      sf[i] = __half2float(s);
      yf[i] = sf[i] != 0.f ? __frcp_rn(sf[i]) : 0.f;  // RN(1/s), for the quotient below
      zh[i] = __half_as_ushort(z);
      sh[i] = __half_as_ushort(s);
    }
    uint16_t* sp = scale + (g * nb + b) * d + c0;
    uint16_t* zp = zero + (g * nb + b) * d + c0;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      sp[i] = sh[i];
      zp[i] = zh[i];
    }
    auto code_row = [&](int t, const float (&v)[CPL]) {
      uint32_t bits = 0;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        uint32_t q = 0;
        if (sf[i] != 0.f) {
          // RN(dv / s) without a division (Markstein, IBM J. Res. Dev. 34(1), 1990): with y = RN(1/s)
          // and q0 = RN(dv y), the residual fma(-q0, s, dv) is exact and RN(q0 + r y) = RN(dv / s)
          const float dv = __fsub_rn(v[i], zf[i]);
          const float q0 = __fmul_rn(dv, yf[i]);
          const float r = __fmaf_rn(-q0, sf[i], dv);
          const float t = rintf(__fmaf_rn(r, yf[i], q0));
          q = (uint32_t)fminf(fmaxf(t, 0.f), 3.f);
        }
        bits |= q << (2 * ((c0 + i) & 15));
      }
#pragma unroll
      for (int o = 1; o < LPW; o <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, o);
      if ((lane % LPW) == 0) codes[(row0 + t) * (d / 16) + c0 / 16] = bits;
    };
    if (whole) {
#pragma unroll
      for (int t = 0; t < kKB; ++t) {
        float v[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) v[i] = bf16_lane(rowv[REG ? t : 0], i);
        code_row(t, v);
      }
    } else {
#pragma unroll 4
      for (int t = 0; t < cnt; ++t) {
        float v[CPL];
        load_cpl<DTYPE, CPL>(keys, (row0 + t) * d + c0, v);
        code_row(t, v);
      }
    }
  }
}

template <int CPL>
__global__ void __launch_bounds__(kKWarps * 32) kivi_key_scores_kernel(const uint32_t* __restrict__ codes,
                                                                       const uint16_t* __restrict__ scale,
                                                                       const uint16_t* __restrict__ zero,
                                                                       int64_t G, int64_t N, int J,
                                                                       const float* __restrict__ q,
                                                                       float* __restrict__ scores) {
  constexpr int d = 32 * CPL;
  constexpr int WPK = d / 16;  // code words per key
  __shared__ __align__(16) float s_a[kKWarps][d];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* a = s_a[warp];
  const int64_t nb = (N + kKB - 1) / kKB;
  const int64_t items = G * nb * J;
  const int c0 = CPL * lane;
  for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items;
       it += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t gb = it / J;
    const int j = (int)(it - gb * J);
    const int64_t g = gb / nb, b = gb - (gb / nb) * nb;
    const float* qj = q + (g * J + j) * d;
    const uint16_t* sp = scale + (g * nb + b) * d;
    const uint16_t* zp = zero + (g * nb + b) * d;
    // this lane's key: its code words are loaded first, so they are in flight with the block's q, scale
    // and zero loads
    const int64_t n = b * kKB + lane;
    uint4 cwv[WPK / 4];
    if (n < N) {
      const uint32_t* cw = codes + (g * N + n) * WPK;
#pragma unroll
      for (int w4 = 0; w4 < WPK; w4 += 4) cwv[w4 / 4] = __ldg(reinterpret_cast<const uint4*>(cw + w4));
    }
    float bpart = 0.f;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int c = c0 + i;
      const float qc = __ldg(qj + c);
      const float s = __half2float(__ushort_as_half(__ldg(sp + c)));
      const float z = __half2float(__ushort_as_half(__ldg(zp + c)));
      // 4^-(c % 8): exact power of two
      a[c] = qc * s * __uint_as_float((uint32_t)(127 - 2 * (c & 7)) << 23);
      bpart = fmaf(qc, z, bpart);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) bpart += __shfl_xor_sync(0xffffffffu, bpart, o);
    __syncwarp();
    if (n < N) {
      float acc = 0.f;
#pragma unroll
      for (int w4 = 0; w4 < WPK; w4 += 4) {
        const uint4 wv = cwv[w4 / 4];
        const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t chunk = h ? (ws[u] >> 16) : ws[u];
            // the 8 weights as two broadcast 16-byte reads
            const float4 a0 = *reinterpret_cast<const float4*>(a + 16 * (w4 + u) + 8 * h);
            const float4 a1 = *reinterpret_cast<const float4*>(a + 16 * (w4 + u) + 8 * h + 4);
            const float ac[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float v = __uint_as_float(0x4B000000u | (chunk & (3u << (2 * k)))) - 8388608.f;
              acc = fmaf(v, ac[k], acc);
            }
          }
        }
      }
      scores[(g * J + j) * N + n] = acc + bpart;
    }
  }
}

int grid_for(int64_t items) {
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t want = (items + kKWarps - 1) / kKWarps;
  return (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)qjl_num_sms(dev) * 8));
}

template <int CPL>
qjl_status launch_quant(const void* keys, int dtype, int64_t G, int64_t N, uint32_t* codes, uint16_t* scale,
                        uint16_t* zero, cudaStream_t st) {
  const int64_t items = G * ((N + kKB - 1) / kKB);
  if (dtype == QJL_F32)
    kivi_keys_quantize_kernel<QJL_F32, CPL><<<grid_for(items), kKWarps * 32, 0, st>>>(keys, G, N, codes, scale, zero);
  else
    kivi_keys_quantize_kernel<QJL_BF16, CPL><<<grid_for(items), kKWarps * 32, 0, st>>>(keys, G, N, codes, scale,
                                                                                        zero);
  return qjl_check_launch("kivi_keys_quantize_kernel");
}

template <int CPL>
qjl_status launch_kscores(const uint32_t* codes, const uint16_t* scale, const uint16_t* zero, int64_t G, int64_t N,
                          int J, const float* q, float* scores, cudaStream_t st) {
  const int64_t items = G * ((N + kKB - 1) / kKB) * J;
  kivi_key_scores_kernel<CPL><<<grid_for(items), kKWarps * 32, 0, st>>>(codes, scale, zero, G, N, J, q, scores);
  return qjl_check_launch("kivi_key_scores_kernel");
}

}  // namespace

extern "C" {

qjl_status qjl_kivi_quantize_keys_2bit(const void* keys, qjl_dtype dtype, int64_t groups, int64_t N, int d,
                                       uint32_t* codes, uint16_t* scale, uint16_t* zero, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (dtype != QJL_F32 && dtype != QJL_BF16) return qjl_set_error(QJL_ERR_INVALID_ARG, "unknown dtype");
  if (groups < 0 || N < 0 || groups > (1 << 24) || N > ((int64_t)1 << 36))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "groups/N out of range");
  if (d != 64 && d != 128 && d != 256) return qjl_set_error(QJL_ERR_UNSUPPORTED, "KIVI keys support d in {64, 128, 256}");
  if (groups == 0 || N == 0) return QJL_OK;
  if (!keys || !codes || !scale || !zero) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(keys) || !aligned16(codes) || !aligned16(scale) || !aligned16(zero))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "keys, codes, scale and zero must be 16-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  switch (d) {
    case 64: return launch_quant<2>(keys, dtype, groups, N, codes, scale, zero, st);
    case 128: return launch_quant<4>(keys, dtype, groups, N, codes, scale, zero, st);
    default: return launch_quant<8>(keys, dtype, groups, N, codes, scale, zero, st);
  }
}

qjl_status qjl_kivi_key_scores(const uint32_t* codes, const uint16_t* scale, const uint16_t* zero, int64_t groups,
                               int64_t N, int d, const float* q, int q_per_group, float* scores, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (groups < 0 || N < 0 || groups > (1 << 24) || N > ((int64_t)1 << 36))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "groups/N out of range");
  if (q_per_group < 1 || q_per_group > 64) return qjl_set_error(QJL_ERR_INVALID_ARG, "q_per_group must be in 1..64");
  if (d != 64 && d != 128 && d != 256) return qjl_set_error(QJL_ERR_UNSUPPORTED, "KIVI keys support d in {64, 128, 256}");
  if (groups == 0 || N == 0) return QJL_OK;
  if (!codes || !scale || !zero || !q || !scores) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(codes) || ((uintptr_t)scale & 1u) || ((uintptr_t)zero & 1u) || ((uintptr_t)q & 3u) ||
      ((uintptr_t)scores & 3u))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "codes must be 16-byte aligned; scale/zero, q and scores naturally");
  cudaStream_t st = (cudaStream_t)stream;
  switch (d) {
    case 64: return launch_kscores<2>(codes, scale, zero, groups, N, q_per_group, q, scores, st);
    case 128: return launch_kscores<4>(codes, scale, zero, groups, N, q_per_group, q, scores, st);
    default: return launch_kscores<8>(codes, scale, zero, groups, N, q_per_group, q, scores, st);
  }
}

}  // extern "C"
