// Fused decode attention over sketched keys and 2-bit per-token values.
//
// One decode step reads the whole compressed cache once (KIVI abstract,
// "Vladimir Braverman" page). The logits are QJL estimates (QJL abstract,
// "Majid Daliri" page):
//   out[g][j] = sum_n softmax_n(softmax_scale * est[g][j][n]) * v_hat[g][n]
// with v_hat = code * scale + zero per 32-channel group.
//
// Pass 1 (decode_partial_kernel): grid (splits, G). Each CTA walks a
// contiguous range of 16-token tiles of one group. Per tile, each warp:
//   * computes the tile's estimates with the s8 tensor-core sign sums shared
//     with the score kernel;
//   * updates an online softmax (running max and sum per query, base-2
//     exponent);
//   * stages the tile's codes, scales and zeros in its shared memory slice;
//   * accumulates p * code * scale and p * zero per channel. Lane l owns
//     channels l*CPL .. l*CPL + CPL - 1, which lie in one 32-channel group.
//     Codes are turned into floats exactly with the 2^23 mantissa trick
//     rather than the quarter-rate integer-to-float converter.
// The CTA's warps are merged in shared memory, and one partial
// (max, sum, acc[d]) per query goes to the workspace.
// Pass 2 (decode_combine_kernel): a log-sum-exp merge of the splits.

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "qjl_internal.h"
#include "sign_mma.cuh"

namespace {

using namespace qjl_sign;
constexpr int kWarps = 4;
constexpr int kMaxJ = 4;
constexpr float kLog2e = 1.4426950408889634f;

int64_t decode_splits(int64_t G, int64_t N) {
  const int64_t ntiles = (N + 15) / 16;
  const int64_t target = 148 * 4;  // fixed, so the workspace size depends only on the shapes
  int64_t s = (target + G - 1) / G;
  s = std::max<int64_t>(1, std::min<int64_t>(s, (ntiles + kWarps - 1) / kWarps));
  const int64_t tpc = (ntiles + s - 1) / s;
  return (ntiles + tpc - 1) / tpc;
}

template <int W, int CPL>
__global__ void __launch_bounds__(kWarps * 32) decode_partial_kernel(
    const uint32_t* __restrict__ bits, const float* __restrict__ norms,
    const uint32_t* __restrict__ codes, const uint16_t* __restrict__ scale,
    const uint16_t* __restrict__ zero, const float* __restrict__ sq, int64_t N, int J,
    float est_scale, float logit_scale, int64_t tiles_per_cta, float* __restrict__ ws) {
  constexpr int d = 32 * CPL;
  constexpr int CW = d / 16;   // code words per token
  constexpr int GW = d / 32;   // scale/zero halves per token
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* s_inv = reinterpret_cast<float*>(smem_raw);
  float* s_mul = s_inv + 64;
  int* s_qsum = reinterpret_cast<int*>(s_mul + 64);
  uint2* Btab = reinterpret_cast<uint2*>(smem_raw + 3 * 64 * 4);
  uint32_t* s_codes = reinterpret_cast<uint32_t*>(Btab + W * 32);     // [warp][16][CW]
  uint16_t* s_sz = reinterpret_cast<uint16_t*>(s_codes + kWarps * 16 * CW);  // [warp][16][2][GW]
  float* s_red = reinterpret_cast<float*>(s_sz + kWarps * 16 * 2 * GW);      // [warp][J][d + 2]

  const int64_t gi = blockIdx.y;
  build_tables<W>(sq + gi * (int64_t)J * (32 * W), J, 1, est_scale, s_inv, s_mul, s_qsum, Btab, kWarps);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int64_t ntiles = (N + 15) >> 4;
  const int64_t t_begin = (int64_t)blockIdx.x * tiles_per_cta;
  const int64_t t_end = min(ntiles, t_begin + tiles_per_cta);
  const uint32_t* gbits = bits + gi * N * W;
  const float* gnorm = norms + gi * N;
  const uint32_t* gcodes = codes + gi * N * CW;
  const uint16_t* gscale = scale + gi * N * GW;
  const uint16_t* gzero = zero + gi * N * GW;
  uint32_t* wcodes = s_codes + warp * 16 * CW;
  uint16_t* wsz = s_sz + warp * 16 * 2 * GW;

  // This lane's channels: c0 .. c0 + CPL - 1, all in group grp.
  const int c0 = lane * CPL;
  const int grp = c0 >> 5;
  const int cw = c0 >> 4, cshift = 2 * (c0 & 15);

  float m_run[kMaxJ], l_run[kMaxJ], accz[kMaxJ], acc[kMaxJ][CPL];
#pragma unroll
  for (int j = 0; j < kMaxJ; ++j) {
    m_run[j] = -INFINITY;
    l_run[j] = 0.f;
    accz[j] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[j][c] = 0.f;
  }
  const float mulq = (q < J) ? s_mul[q] * logit_scale : 0.f;
  const long long qs32 = (q < J) ? 32LL * s_qsum[q] : 0;

  for (int64_t t = t_begin + warp; t < t_end; t += kWarps) {
    const int64_t row0 = t * 16 + g;
    uint32_t w0[W / 4], w1[W / 4];
    load_words<W>(gbits, row0, N, q, w0);
    load_words<W>(gbits, row0 + 8, N, q, w1);
    // stage codes / scale / zero of the tile (rows past N are zero-filled)
    for (int i = lane; i < 16 * CW; i += 32) {
      const int64_t row = t * 16 + i / CW;
      wcodes[i] = row < N ? __ldg(gcodes + t * 16 * CW + i) : 0u;
    }
    for (int i = lane; i < 16 * GW; i += 32) {
      const int r = i / GW, k = i % GW;
      const int64_t row = t * 16 + r;
      wsz[(r * 2 + 0) * GW + k] = row < N ? __ldg(gscale + t * 16 * GW + i) : (uint16_t)0;
      wsz[(r * 2 + 1) * GW + k] = row < N ? __ldg(gzero + t * 16 * GW + i) : (uint16_t)0;
    }
    int hi[2], lo[2];
    tile_sums<W>(w0, w1, Btab, lane, hi, lo);
    float x[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int64_t row = row0 + 8 * r;
      const float nrm = row < N ? __ldg(gnorm + row) : 0.f;
      const long long D = 256LL * hi[r] + lo[r] - qs32;
      x[r] = (row < N && q < J) ? mulq * kLog2e * nrm * ((float)D * 0.03125f) : -INFINITY;
    }
    // tile max per query (lanes sharing q), then the new running max
    float mt = fmaxf(x[0], x[1]);
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
    float mnew_q = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxJ; ++j) {
      if (j >= J) break;
      const float mtj = __shfl_sync(0xffffffffu, mt, j);
      const float mn = fmaxf(m_run[j], mtj);
      const float corr = exp2f(m_run[j] - mn);  // 0 on the first tile (m_run = -inf)
      m_run[j] = mn;
      l_run[j] *= corr;
      accz[j] *= corr;
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc[j][c] *= corr;
      if (q == j) mnew_q = mn;
    }
    float p[2];
    p[0] = (q < J) ? exp2f(x[0] - mnew_q) : 0.f;
    p[1] = (q < J) ? exp2f(x[1] - mnew_q) : 0.f;
    float ps = p[0] + p[1];
    ps += __shfl_xor_sync(0xffffffffu, ps, 4);
    ps += __shfl_xor_sync(0xffffffffu, ps, 8);
    ps += __shfl_xor_sync(0xffffffffu, ps, 16);
#pragma unroll
    for (int j = 0; j < kMaxJ; ++j) {
      if (j >= J) break;
      l_run[j] += __shfl_sync(0xffffffffu, ps, j);
    }
    __syncwarp();
    // value accumulation: token r of the tile is held by lane 4*(r%8) + j
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const uint32_t cword = wcodes[r * CW + cw] >> cshift;
      const float sc = __half2float(__ushort_as_half(wsz[(r * 2 + 0) * GW + grp]));
      const float zr = __half2float(__ushort_as_half(wsz[(r * 2 + 1) * GW + grp]));
      float cf[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c)
        cf[c] = __uint_as_float(0x4B000000u | ((cword >> (2 * c)) & 3u)) - 8388608.f;
#pragma unroll
      for (int j = 0; j < kMaxJ; ++j) {
        if (j >= J) break;
        const float pr = __shfl_sync(0xffffffffu, p[r >> 3], 4 * (r & 7) + j);
        const float pw = pr * sc;
        accz[j] = fmaf(pr, zr, accz[j]);
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[j][c] = fmaf(pw, cf[c], acc[j][c]);
      }
    }
    __syncwarp();
  }

  // merge the CTA's warps: each warp writes (m, l, acc[d]) per query
  float* red = s_red + warp * J * (d + 2);
#pragma unroll
  for (int j = 0; j < kMaxJ; ++j) {
    if (j >= J) break;
    float* rj = red + j * (d + 2);
#pragma unroll
    for (int c = 0; c < CPL; ++c) rj[2 + c0 + c] = acc[j][c] + accz[j];
    if (lane == 0) {
      rj[0] = m_run[j];
      rj[1] = l_run[j];
    }
  }
  __syncthreads();
  const int64_t split = blockIdx.x;
  const int64_t nsplit = gridDim.x;
  for (int idx = threadIdx.x; idx < J * (d + 2); idx += blockDim.x) {
    const int j = idx / (d + 2), k = idx % (d + 2);
    float M = -INFINITY;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_red[(w * J + j) * (d + 2)]);
    float v = 0.f;
    if (k == 0) {
      v = M;
    } else {
      for (int w = 0; w < kWarps; ++w) {
        const float mw = s_red[(w * J + j) * (d + 2)];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        v += f * s_red[(w * J + j) * (d + 2) + k];
      }
    }
    ws[((gi * nsplit + split) * J + j) * (d + 2) + k] = v;
  }
}

// out[g][j][c] = sum_s acc_s[c] 2^(m_s - M) / sum_s l_s 2^(m_s - M)
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ ws, int64_t G,
                                                             int J, int d, int64_t nsplit,
                                                             float* __restrict__ out) {
  const int64_t gj = blockIdx.x;
  if (gj >= G * J) return;
  const int64_t gi = gj / J;
  const int j = (int)(gj % J);
  float M = -INFINITY;
  for (int64_t s = 0; s < nsplit; ++s) M = fmaxf(M, ws[((gi * nsplit + s) * J + j) * (d + 2)]);
  float L = 0.f;
  for (int64_t s = 0; s < nsplit; ++s) {
    const float* e = ws + ((gi * nsplit + s) * J + j) * (d + 2);
    L += (e[0] == -INFINITY) ? 0.f : e[1] * exp2f(e[0] - M);
  }
  const float invL = 1.f / L;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float v = 0.f;
    for (int64_t s = 0; s < nsplit; ++s) {
      const float* e = ws + ((gi * nsplit + s) * J + j) * (d + 2);
      if (e[0] != -INFINITY) v += e[2 + c] * exp2f(e[0] - M);
    }
    out[gj * d + c] = v * invL;
  }
}

template <int W, int CPL>
qjl_status launch_wc(const qjl_projection* P, const uint32_t* bits, const float* norms,
                     const uint32_t* codes, const uint16_t* scale, const uint16_t* zero, int64_t G,
                     int64_t N, const float* sq, int J, float softmax_scale, float* out, float* ws,
                     cudaStream_t st) {
  constexpr int d = 32 * CPL;
  const size_t smem = 3 * 64 * 4 + (size_t)W * 32 * sizeof(uint2) + (size_t)kWarps * 16 * (d / 16) * 4 +
                      (size_t)kWarps * 16 * 2 * (d / 32) * 2 + (size_t)kWarps * J * (d + 2) * 4;
  auto kern = decode_partial_kernel<W, CPL>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return qjl_check_launch("decode_partial_kernel smem attribute");
  const int64_t splits = decode_splits(G, N);
  const int64_t ntiles = (N + 15) / 16;
  const int64_t tpc = (ntiles + splits - 1) / splits;
  dim3 grid((unsigned)splits, (unsigned)G);
  kern<<<grid, kWarps * 32, smem, st>>>(bits, norms, codes, scale, zero, sq, N, J, P->est_scale,
                                        softmax_scale, tpc, ws);
  qjl_status s = qjl_check_launch("decode_partial_kernel");
  if (s != QJL_OK) return s;
  decode_combine_kernel<<<(unsigned)(G * J), 128, 0, st>>>(ws, G, J, d, splits, out);
  return qjl_check_launch("decode_combine_kernel");
}

template <int W>
qjl_status launch_w(const qjl_projection* P, const uint32_t* bits, const float* norms,
                    const uint32_t* codes, const uint16_t* scale, const uint16_t* zero, int64_t G,
                    int64_t N, const float* sq, int J, float softmax_scale, float* out, float* ws,
                    cudaStream_t st) {
  switch (P->d) {
    case 32: return launch_wc<W, 1>(P, bits, norms, codes, scale, zero, G, N, sq, J, softmax_scale, out, ws, st);
    case 64: return launch_wc<W, 2>(P, bits, norms, codes, scale, zero, G, N, sq, J, softmax_scale, out, ws, st);
    case 128: return launch_wc<W, 4>(P, bits, norms, codes, scale, zero, G, N, sq, J, softmax_scale, out, ws, st);
    case 256: return launch_wc<W, 8>(P, bits, norms, codes, scale, zero, G, N, sq, J, softmax_scale, out, ws, st);
  }
  return qjl_set_error(QJL_ERR_UNSUPPORTED, "decode attention supports d in {32, 64, 128, 256}");
}

}  // namespace

size_t decode_workspace_bytes(int64_t G, int J, int64_t N, int d) {
  return (size_t)G * (size_t)decode_splits(G, N) * (size_t)J * (size_t)(d + 2) * sizeof(float);
}

qjl_status launch_decode(const qjl_projection* P, const uint32_t* bits, const float* norms,
                         const uint32_t* codes, const uint16_t* scale, const uint16_t* zero,
                         int64_t G, int64_t N, const float* sq, int J, float softmax_scale,
                         float* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  (void)ws_bytes;
  if (J > kMaxJ) return qjl_set_error(QJL_ERR_UNSUPPORTED, "decode attention supports q_per_group <= 4");
  if (G > 65535) return qjl_set_error(QJL_ERR_UNSUPPORTED, "groups > 65535");
  float* w = reinterpret_cast<float*>(ws);
  switch (P->m) {
    case 256: return launch_w<8>(P, bits, norms, codes, scale, zero, G, N, sq, J, softmax_scale, out, w, st);
    case 512: return launch_w<16>(P, bits, norms, codes, scale, zero, G, N, sq, J, softmax_scale, out, w, st);
    case 1024: return launch_w<32>(P, bits, norms, codes, scale, zero, G, N, sq, J, softmax_scale, out, w, st);
  }
  return qjl_set_error(QJL_ERR_UNSUPPORTED, "decode attention supports m in {256, 512, 1024}");
}
