// Dense query projection Sq = S_eff q for many queries (a prefill projects
// every position) on the bf16 tensor-core path, at fp32 accuracy.
//
// The QJL estimator (QJL abstract, "Majid Daliri" page) projects the query
// with the same S as the keys but does not quantise it. With the bf16 matrix
// option S_eff holds bf16 values exactly. An fp32 query element x splits into
// three bf16 parts x = h + u + l + r with h = bf16(x), u = bf16(x - h),
// l = bf16(x - h - u): each subtraction is exact in fp32 and |r| <= 2^-27 |x|.
// Every product S_ij * part is exact in fp32 (8 x 8 significant bits), so
// three m16n8k16 MMAs per tile, accumulating in fp32, give the fp32 dot
// product up to the accumulation order.
//
// One warp computes 16 queries x 128 outputs (16 n8 tiles) per work item, the
// query rows read straight into the A fragment layout one k16 chunk ahead.
// S_eff [m][d] sits in shared memory with rows padded by 16 bytes, so the
// ldmatrix row addresses of an 8 x 8 tile fall in distinct banks. The warps
// of a persistent grid stride over the (query tile, column block) items.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "qjl_internal.h"

namespace {

constexpr int kThreads = 256;  // 8 warps
constexpr int kCols = 128;     // output columns per work item

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// (x0, x1) -> the three bf16x2 parts of the pair
__device__ __forceinline__ void split3(float2 x, uint32_t& h, uint32_t& u, uint32_t& l) {
  const float h0 = __bfloat162float(__float2bfloat16_rn(x.x)), h1 = __bfloat162float(__float2bfloat16_rn(x.y));
  const float r0 = x.x - h0, r1 = x.y - h1;
  const float u0 = __bfloat162float(__float2bfloat16_rn(r0)), u1 = __bfloat162float(__float2bfloat16_rn(r1));
  h = bf16x2(h0, h1);
  u = bf16x2(u0, u1);
  l = bf16x2(r0 - u0, r1 - u1);
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

__global__ void __launch_bounds__(kThreads, 2) project_mma_kernel(const float* __restrict__ q, int64_t nq,
                                                                  int64_t ld, int d, int m,
                                                                  const uint16_t* __restrict__ S,
                                                                  float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* Ss = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  const int ds = d + 8;  // padded row stride (bf16)
  {
    // S_eff rows, 16 bytes at a time
    const int cpr = d / 8;
    for (int i = threadIdx.x; i < m * cpr; i += kThreads) {
      const int r = i / cpr, c = i % cpr;
      *reinterpret_cast<uint4*>(Ss + r * ds + 8 * c) = __ldg(reinterpret_cast<const uint4*>(S + (int64_t)r * d) + c);
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, t = lane & 3;
  const int ncb = m / kCols, kc_n = d / 16;
  const int64_t tiles = (nq + 15) / 16, items = tiles * ncb;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  // ldmatrix row address of this lane within a pair of n8 tiles: matrix lane / 8 (n half, k half)
  const int mi = lane >> 3, lr = lane & 7;
  const int ldm_off = (8 * (mi >> 1) + lr) * ds + 8 * (mi & 1);
  for (int64_t it = (int64_t)blockIdx.x * (kThreads / 32) + warp; it < items; it += nwarps) {
    const int64_t tile = it / ncb;
    const int cb = (int)(it % ncb);
    const int64_t ra = tile * 16 + gq, rb = ra + 8;
    const bool va = ra < nq, vb = rb < nq;
    const float* qa = q + (va ? ra : 0) * ld + 2 * t;
    const float* qb = q + (vb ? rb : 0) * ld + 2 * t;
    float acc[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[n][j] = 0.f;
    const float2 z = make_float2(0.f, 0.f);
    // A elements of chunk 0: rows a and b, columns 2t and 2t + 8
    float2 xa0 = va ? __ldg(reinterpret_cast<const float2*>(qa)) : z;
    float2 xa1 = va ? __ldg(reinterpret_cast<const float2*>(qa + 8)) : z;
    float2 xb0 = vb ? __ldg(reinterpret_cast<const float2*>(qb)) : z;
    float2 xb1 = vb ? __ldg(reinterpret_cast<const float2*>(qb + 8)) : z;
    const __nv_bfloat16* Sb = Ss + cb * kCols * ds + ldm_off;
    for (int kc = 0; kc < kc_n; ++kc) {
      uint32_t ah[4], au[4], al[4];
      split3(xa0, ah[0], au[0], al[0]);
      split3(xb0, ah[1], au[1], al[1]);
      split3(xa1, ah[2], au[2], al[2]);
      split3(xb1, ah[3], au[3], al[3]);
      if (kc + 1 < kc_n) {
        const int k1 = 16 * (kc + 1);
        xa0 = va ? __ldg(reinterpret_cast<const float2*>(qa + k1)) : z;
        xa1 = va ? __ldg(reinterpret_cast<const float2*>(qa + k1 + 8)) : z;
        xb0 = vb ? __ldg(reinterpret_cast<const float2*>(qb + k1)) : z;
        xb1 = vb ? __ldg(reinterpret_cast<const float2*>(qb + k1 + 8)) : z;
      }
      const __nv_bfloat16* Sk = Sb + 16 * kc;
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b[4];
        ldm_x4(b, Sk + 16 * np * ds);
        mma_bf16(acc[2 * np], al[0], al[1], al[2], al[3], b[0], b[1]);
        mma_bf16(acc[2 * np + 1], al[0], al[1], al[2], al[3], b[2], b[3]);
        mma_bf16(acc[2 * np], au[0], au[1], au[2], au[3], b[0], b[1]);
        mma_bf16(acc[2 * np + 1], au[0], au[1], au[2], au[3], b[2], b[3]);
        mma_bf16(acc[2 * np], ah[0], ah[1], ah[2], ah[3], b[0], b[1]);
        mma_bf16(acc[2 * np + 1], ah[0], ah[1], ah[2], ah[3], b[2], b[3]);
      }
    }
    float* oa = out + ra * (int64_t)m + cb * kCols + 2 * t;
    float* ob = out + rb * (int64_t)m + cb * kCols + 2 * t;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      if (va) *reinterpret_cast<float2*>(oa + 8 * n) = make_float2(acc[n][0], acc[n][1]);
      if (vb) *reinterpret_cast<float2*>(ob + 8 * n) = make_float2(acc[n][2], acc[n][3]);
    }
  }
}

}  // namespace

size_t project_mma_smem(const qjl_projection* P) { return (size_t)P->m * (P->d + 8) * 2; }

bool project_mma_supported(const qjl_projection* P, const float* q, int64_t ld, const float* out) {
  return P->S_bf16 != nullptr && P->d % 16 == 0 && P->m % kCols == 0 && project_mma_smem(P) <= 200 * 1024 &&
         ((uintptr_t)q & 7u) == 0 && (ld & 1) == 0 && ((uintptr_t)out & 7u) == 0;
}

qjl_status launch_project_mma(const qjl_projection* P, const float* q, int64_t nq, int64_t ld, float* out,
                              cudaStream_t st) {
  if (nq <= 0) return QJL_OK;
  const size_t smem = project_mma_smem(P);
  if (cudaFuncSetAttribute(project_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return qjl_check_launch("project_mma_kernel smem attribute");
  const int per_sm = smem * 2 <= 220 * 1024 ? 2 : 1;
  const int64_t items = (nq + 15) / 16 * (P->m / kCols);
  const int64_t want = (items + kThreads / 32 - 1) / (kThreads / 32);
  const int blocks = (int)std::min<int64_t>(want, (int64_t)qjl_num_sms(P->device) * per_sm);
  project_mma_kernel<<<blocks, kThreads, smem, st>>>(q, nq, ld, P->d, P->m, P->S_bf16, out);
  return qjl_check_launch("project_mma_kernel");
}
