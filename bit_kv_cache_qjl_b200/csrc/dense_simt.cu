// Dense JL projection on the fp32 SIMT pipe (QJL abstract: "a JL transform
// followed by sign-bit quantization"; the query side is the same transform
// without quantisation).
//
// One warp per row (key or query). Lane l owns output coordinates
// c0 + 32 r + l, so __ballot_sync over the lanes yields packed sign word
// (c0/32 + r) directly (bit = 1 iff y >= 0). S_eff^T is read from global
// memory in coalesced 128-byte rows; every warp reads the same matrix, so it
// stays in L1/L2. This path serves fp32 keys, fp32 S_eff and every query
// projection. bf16 keys with bf16 S_eff go to the tcgen05 kernel.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qjl_internal.h"

namespace {

constexpr int kRowsPerPass = 8;  // 8 x 32 = 256 output coordinates per pass

template <int DTYPE>
__device__ __forceinline__ float load_elem(const void* base, int64_t idx) {
  if (DTYPE == QJL_F32) return __ldg(reinterpret_cast<const float*>(base) + idx);
  const unsigned short b = __ldg(reinterpret_cast<const unsigned short*>(base) + idx);
  return __uint_as_float((uint32_t)b << 16);
}

template <int DTYPE>
__global__ void __launch_bounds__(256) dense_simt_kernel(const void* __restrict__ x, int64_t rows,
                                                         int64_t ld, int d, int m,
                                                         const float* __restrict__ St,
                                                         uint32_t* __restrict__ bits,
                                                         float* __restrict__ norms,
                                                         float* __restrict__ proj_out, PageMap pm,
                                                         int* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int W = m >> 5;
  for (int64_t row = warp; row < rows; row += nwarps) {
    const int64_t xoff = row * ld;
    // output row: the same row, or the key's page slot when appending to a paged cache
    const int64_t orow = pm.slot(row);
    if (orow < 0) {
      if (lane == 0 && err) atomicOr(err, QJL_DEVERR_PAGE);
      continue;
    }
    float sumsq = 0.f;
    for (int c0 = 0; c0 < m; c0 += 32 * kRowsPerPass) {
      float acc[kRowsPerPass];
#pragma unroll
      for (int r = 0; r < kRowsPerPass; ++r) acc[r] = 0.f;
      for (int j0 = 0; j0 < d; j0 += 32) {
        const int j = j0 + lane;
        const float xv = (j < d) ? load_elem<DTYPE>(x, xoff + j) : 0.f;
        if (c0 == 0) sumsq = fmaf(xv, xv, sumsq);
        const int jn = min(32, d - j0);
        for (int jj = 0; jj < jn; ++jj) {
          const float xj = __shfl_sync(0xffffffffu, xv, jj);
          const float* srow = St + (int64_t)(j0 + jj) * m + c0 + lane;
#pragma unroll
          for (int r = 0; r < kRowsPerPass; ++r)
            if (c0 + 32 * r < m) acc[r] = fmaf(__ldg(srow + 32 * r), xj, acc[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < kRowsPerPass; ++r) {
        const int c = c0 + 32 * r;
        if (c >= m) break;
        if (bits) {
          const uint32_t word = __ballot_sync(0xffffffffu, acc[r] >= 0.f);
          if (lane == 0) bits[orow * W + (c >> 5)] = word;
        }
        if (proj_out) proj_out[orow * (int64_t)m + c + lane] = acc[r];
      }
    }
    if (norms) {
#pragma unroll
      for (int o = 16; o; o >>= 1) sumsq += __shfl_xor_sync(0xffffffffu, sumsq, o);
      if (lane == 0) norms[orow] = sqrtf(sumsq);
    }
  }
}

// Query projection Sq = S_eff q: one CTA per query, q staged in shared memory.
// Thread i owns coordinates i, i + 256, ... Its column of S_eff^T is read with
// consecutive threads on consecutive addresses, using four partial sums for ILP.
__global__ void __launch_bounds__(256) project_dense_kernel(const float* __restrict__ q, int64_t ld, int d, int m,
                                                           const float* __restrict__ St,
                                                           float* __restrict__ out) {
  extern __shared__ float qs[];
  const int64_t row = blockIdx.x;
  for (int j = threadIdx.x; j < d; j += blockDim.x) qs[j] = __ldg(q + row * ld + j);
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int j = 0;
    for (; j + 4 <= d; j += 4) {
      a0 = fmaf(__ldg(St + (int64_t)(j + 0) * m + i), qs[j + 0], a0);
      a1 = fmaf(__ldg(St + (int64_t)(j + 1) * m + i), qs[j + 1], a1);
      a2 = fmaf(__ldg(St + (int64_t)(j + 2) * m + i), qs[j + 2], a2);
      a3 = fmaf(__ldg(St + (int64_t)(j + 3) * m + i), qs[j + 3], a3);
    }
    for (; j < d; ++j) a0 = fmaf(__ldg(St + (int64_t)j * m + i), qs[j], a0);
    out[row * (int64_t)m + i] = (a0 + a1) + (a2 + a3);
  }
}

}  // namespace

qjl_status launch_project_dense(const qjl_projection* P, const float* q, int64_t nq, int64_t ld, float* out,
                                cudaStream_t st) {
  // many queries (a prefill projects every position): with a bf16 S_eff the tensor cores at fp32
  // accuracy (three bf16 parts of each query), else one warp per query row, the same fp32 sum over
  // j as below, with far less launch overhead than one CTA per query
  if (nq >= 1024 && project_mma_supported(P, q, ld, out)) return launch_project_mma(P, q, nq, ld, out, st);
  if (nq >= 1024) return launch_dense_simt(P, q, QJL_F32, nq, ld, nullptr, nullptr, out, st);
  const size_t smem = (size_t)P->d * sizeof(float);
  for (int64_t r0 = 0; r0 < nq; r0 += 65535) {
    const int64_t cnt = std::min<int64_t>(65535, nq - r0);
    project_dense_kernel<<<(unsigned)cnt, 256, smem, st>>>(q + r0 * ld, ld, P->d, P->m, P->St_f32,
                                                           out + r0 * (int64_t)P->m);
    qjl_status s = qjl_check_launch("project_dense_kernel");
    if (s != QJL_OK) return s;
  }
  return QJL_OK;
}

qjl_status launch_dense_simt(const qjl_projection* P, const void* x, int dtype, int64_t n, int64_t ld,
                             uint32_t* bits, float* norms, float* proj_out, cudaStream_t st, const PageMap& pm) {
  if (n <= 0) return QJL_OK;
  int* err = pm.pos ? qjl_error_flag(P->device) : nullptr;
  const int threads = 256;
  const int64_t want = (n + 7) / 8;
  const int blocks = (int)std::min<int64_t>(want, (int64_t)qjl_num_sms(P->device) * 16);
  if (dtype == QJL_F32)
    dense_simt_kernel<QJL_F32><<<blocks, threads, 0, st>>>(x, n, ld, P->d, P->m, P->St_f32, bits,
                                                           norms, proj_out, pm, err);
  else
    dense_simt_kernel<QJL_BF16><<<blocks, threads, 0, st>>>(x, n, ld, P->d, P->m, P->St_f32, bits,
                                                            norms, proj_out, pm, err);
  return qjl_check_launch("dense_simt_kernel");
}
