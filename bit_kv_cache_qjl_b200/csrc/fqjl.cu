// D-FQJL / P-FQJL query map: the unquantised FQJL projection of queries.
//
// "Fast Quantized Johnson - Lindenstrauss Transforms" ("In short", "Key
// concepts", "The paper" abstract): the key side is sketched by two
// randomized Hadamard transforms with a Gaussian diagonal in the second stage
// (P-FQJL adds a random permutation between them); the estimator pairs the
// key bits with the same map applied to the query without quantisation. Per
// block b of the m/d stacked blocks (normalised H_n = H / sqrt(d)):
//   Sq = sqrt(d) H_n D_g Pi H_n D_r q = (1/sqrt(d)) H D_g Pi H D_r q   (default)
//   Sq = (1/sqrt(d)) D_g H Pi H D_r q                                  (dg_outer)
// Queries are few (one per head and decode step), so this is a simple kernel:
// one warp per query, element 32 e + lane in register e of that lane,
// butterfly strides below 32 across lanes (shfl_xor) and larger ones in
// registers, the permutation as a gather through the warp's shared row. The
// key side, where the bulk of the work is, lives in fqjl_keys.cu.

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>

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

template <int E>
__global__ void __launch_bounds__(256) fqjl_query_kernel(const float* __restrict__ x, int64_t rows, int64_t ld,
                                                         int m, const float* __restrict__ D_r,
                                                         const int32_t* __restrict__ perm,
                                                         const float* __restrict__ D_g, int permute,
                                                         int dg_outer, float* __restrict__ proj_out) {
  constexpr int d = 32 * E;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  float* buf = smem + wib * d;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int nb = m / d;
  const float inv_sqrt_d = rsqrtf((float)d);

  for (int64_t row = warp; row < rows; row += nwarps) {
    float xv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) xv[e] = __ldg(x + row * ld + 32 * e + lane);
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
        proj_out[row * (int64_t)m + b * d + 32 * e + lane] = y;
      }
    }
  }
}

template <int E>
qjl_status launch_e(const qjl_projection* P, const float* q, int64_t nq, int64_t ld, float* out, cudaStream_t st) {
  const int threads = 256;
  const size_t smem = (size_t)(threads / 32) * 32 * E * sizeof(float);
  const int64_t want = (nq + 7) / 8;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)qjl_num_sms(P->device) * 16));
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(fqjl_query_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return qjl_check_launch("fqjl_query_kernel smem attribute");
  fqjl_query_kernel<E><<<blocks, threads, smem, st>>>(q, nq, ld, P->m, P->D_r, P->perm, P->D_g,
                                                      P->kind == QJL_PFQJL, P->opt.dg_outer, out);
  return qjl_check_launch("fqjl_query_kernel");
}

}  // namespace

qjl_status launch_fqjl_queries(const qjl_projection* P, const float* q, int64_t nq, int64_t ld, float* out,
                               cudaStream_t st) {
  switch (P->d) {
    case 32: return launch_e<1>(P, q, nq, ld, out, st);
    case 64: return launch_e<2>(P, q, nq, ld, out, st);
    case 128: return launch_e<4>(P, q, nq, ld, out, st);
    case 256: return launch_e<8>(P, q, nq, ld, out, st);
    case 512: return launch_e<16>(P, q, nq, ld, out, st);
    case 1024: return launch_e<32>(P, q, nq, ld, out, st);
  }
  return qjl_set_error(QJL_ERR_UNSUPPORTED, "FQJL query kernel supports d in {32,...,1024}");
}
