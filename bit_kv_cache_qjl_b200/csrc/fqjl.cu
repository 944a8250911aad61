// D-FQJL / P-FQJL sketch and query map by fast Walsh-Hadamard transforms.
//
// "Fast Quantized Johnson - Lindenstrauss Transforms" ("In short", "Key
// concepts", "The paper" abstract): the dense Gaussian projection is
// replaced by two randomized Hadamard transforms with a Gaussian diagonal in
// the second stage, at O(d log d) per vector. P-FQJL puts a uniform random
// permutation between the Hadamard stages. D-FQJL adds Gaussian dither before
// the sign ("Transcript: The paper's improvements").
//
// Per block b of m/d stacked blocks (normalised H_n = H / sqrt(d)):
//   y = sqrt(d) H_n D_g Pi H_n D_r x = (1/sqrt(d)) H D_g Pi H D_r x   (default)
//   y = (1/sqrt(d)) D_g H Pi H D_r x                                  (dg_outer)
// followed, for D-FQJL keys, by y += sigma_rel ||x|| xi with
// xi = Box-Muller(Philox(b*d + i, t_lo, t_hi, stream 3)) evaluated in fp32.
//
// One warp per row. Element i = 32 e + lane sits in register e of that lane.
// Butterfly strides below 32 cross lanes (shfl_xor). Larger strides stay
// within a lane. The sign word for coordinates 32 e .. 32 e + 31 of the
// block is then a single __ballot_sync.

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "philox.h"
#include "qjl_internal.h"

namespace {

template <int E>
__device__ __forceinline__ void fwht_warp(float (&v)[E], int lane) {
  // strides 1..16: partner lane = lane ^ h
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float p = __shfl_xor_sync(0xffffffffu, v[e], h);
      v[e] = (lane & h) ? (p - v[e]) : (v[e] + p);
    }
  }
  // strides 32, 64, ...: register index bit
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (!(e & h)) {
        const float a = v[e], b = v[e + h];
        v[e] = a + b;
        v[e + h] = a - b;
      }
    }
  }
}

template <int E, int DTYPE>
__global__ void __launch_bounds__(256) fqjl_kernel(const void* __restrict__ x, int64_t rows, int64_t ld,
                                                   int m, const float* __restrict__ D_r,
                                                   const int32_t* __restrict__ perm,
                                                   const float* __restrict__ D_g, int permute,
                                                   int dg_outer, float sigma_rel, uint64_t seed,
                                                   uint64_t first_token, uint32_t* __restrict__ bits,
                                                   float* __restrict__ norms,
                                                   float* __restrict__ proj_out) {
  constexpr int d = 32 * E;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  float* buf = smem + wib * d;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int nb = m / d;
  const int W = m >> 5;
  const float inv_sqrt_d = rsqrtf((float)d);
  const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);

  for (int64_t row = warp; row < rows; row += nwarps) {
    float xv[E];
    float sumsq = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int64_t idx = row * ld + 32 * e + lane;
      xv[e] = (DTYPE == QJL_F32) ? __ldg(reinterpret_cast<const float*>(x) + idx)
                                 : __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(x) + idx) << 16);
      sumsq = fmaf(xv[e], xv[e], sumsq);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
    const float norm = sqrtf(sumsq);
    if (norms && lane == 0) norms[row] = norm;
    const uint64_t tok = first_token + (uint64_t)row;

    for (int b = 0; b < nb; ++b) {
      const float* dr = D_r + (int64_t)b * d;
      const int32_t* pb = perm + (int64_t)b * d;
      const float* dg = D_g + (int64_t)b * d;
      float v[E];
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = xv[e] * __ldg(dr + 32 * e + lane);
      fwht_warp<E>(v, lane);
      if (permute) {
        // gather u'[i] = u[pi[i]] through this warp's shared-memory row
#pragma unroll
        for (int e = 0; e < E; ++e) buf[32 * e + lane] = v[e];
        __syncwarp();
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = buf[__ldg(pb + 32 * e + lane)];
        __syncwarp();
      }
      if (!dg_outer) {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] *= __ldg(dg + 32 * e + lane);
      }
      fwht_warp<E>(v, lane);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float y = v[e] * inv_sqrt_d;
        if (dg_outer) y *= __ldg(dg + 32 * e + lane);
        const int i = 32 * e + lane;
        if (bits && sigma_rel != 0.f) {
          qjl::U32x4 r = qjl::philox({(uint32_t)(b * d + i), (uint32_t)tok, (uint32_t)(tok >> 32),
                                      qjl::kStreamDither}, k0, k1);
          const float u0 = fmaf((float)r.x, 0x1p-32f, 0x1p-33f);
          const float u1 = fmaf((float)r.y, 0x1p-32f, 0x1p-33f);
          const float xi = sqrtf(-2.f * logf(u0)) * cospif(2.f * u1);
          y = fmaf(sigma_rel * norm, xi, y);
        }
        if (bits) {
          const uint32_t word = __ballot_sync(0xffffffffu, y >= 0.f);
          if (lane == 0) bits[row * W + b * (d >> 5) + e] = word;
        }
        if (proj_out) proj_out[row * (int64_t)m + b * d + i] = y;
      }
    }
  }
}

template <int E>
qjl_status launch_e(const qjl_projection* P, const void* x, int dtype, int64_t n, int64_t ld,
                    uint64_t first_token, uint32_t* bits, float* norms, float* proj_out,
                    cudaStream_t st) {
  const int threads = 256;
  const size_t smem = (size_t)(threads / 32) * 32 * E * sizeof(float);
  const int64_t want = (n + 7) / 8;
  const int blocks = (int)std::min<int64_t>(want, (int64_t)qjl_num_sms(P->device) * 16);
  const int permute = P->kind == QJL_PFQJL;
  const float sig = bits ? P->dither_sigma : 0.f;
  if (smem > 48 * 1024) {
    auto k = dtype == QJL_F32 ? fqjl_kernel<E, QJL_F32> : fqjl_kernel<E, QJL_BF16>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return qjl_check_launch("fqjl_kernel smem attribute");
  }
  if (dtype == QJL_F32)
    fqjl_kernel<E, QJL_F32><<<blocks, threads, smem, st>>>(x, n, ld, P->m, P->D_r, P->perm, P->D_g, permute,
                                                          P->opt.dg_outer, sig, P->seed, first_token,
                                                          bits, norms, proj_out);
  else
    fqjl_kernel<E, QJL_BF16><<<blocks, threads, smem, st>>>(x, n, ld, P->m, P->D_r, P->perm, P->D_g, permute,
                                                           P->opt.dg_outer, sig, P->seed, first_token,
                                                           bits, norms, proj_out);
  return qjl_check_launch("fqjl_kernel");
}

}  // namespace

qjl_status launch_fqjl(const qjl_projection* P, const void* x, int dtype, int64_t n, int64_t ld,
                       uint64_t first_token, uint32_t* bits, float* norms, float* proj_out,
                       cudaStream_t st) {
  switch (P->d) {
    case 32: return launch_e<1>(P, x, dtype, n, ld, first_token, bits, norms, proj_out, st);
    case 64: return launch_e<2>(P, x, dtype, n, ld, first_token, bits, norms, proj_out, st);
    case 128: return launch_e<4>(P, x, dtype, n, ld, first_token, bits, norms, proj_out, st);
    case 256: return launch_e<8>(P, x, dtype, n, ld, first_token, bits, norms, proj_out, st);
    case 512: return launch_e<16>(P, x, dtype, n, ld, first_token, bits, norms, proj_out, st);
    case 1024: return launch_e<32>(P, x, dtype, n, ld, first_token, bits, norms, proj_out, st);
  }
  return qjl_set_error(QJL_ERR_UNSUPPORTED, "FQJL kernel supports d in {32,...,1024}");
}
