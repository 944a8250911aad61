// Asymmetric QJL estimator over packed sign bits (QJL abstract, "Majid
// Daliri" page): est = c * alpha * ||k|| * sum_i (2 b_i - 1) * Sq_i.
//
// Decode reads every key's bits once per query step (KIVI abstract: the
// whole cache is loaded per generated token), so the kernel must stay at the
// HBM roof, where each SM has under two clocks per 40-byte key. A plain
// bit-serial sign-dot costs several instructions per bit, and on sm_100a the
// 1-bit mma.sync is emulated, so the sign sums run on the s8 tensor-core
// path instead:
//
//   * Sq is rounded per (group, query) to 16-bit fixed point,
//     Q = rint(Sq * 32639 / max|Sq|), and split as Q = 256 hi + lo with
//     int8 halves. Columns 2j and 2j+1 of an n8 B tile hold hi and lo of
//     query j, so one tile serves 4 queries.
//   * A 16-key x 32-k A tile takes 32 bits from each key. A register is
//     (word >> s) & (0x01010101 << J): four bits (8e + J + s), e = 0..3, of
//     one word, each worth 2^J. That is one AND per 4 bits, with no
//     unpacking. The k order is free as long as the B tile uses the same
//     order, so B is laid out to match.
//   * Four accumulators (J = 0, 2, 4, 6) are merged exactly in int32 as
//     64 * sum b Q. The estimate is (2 sum b Q - sum Q) * scale, formed in
//     int64 before one rounding to fp32.
// The sign sums are exact. The only error is the 16-bit rounding of Sq:
// at most m * max|Sq| / 65278 before scaling.
//
// Layout: bits [G][N][W] uint32, norms [G][N], sq [G][J][m], scores [G][J][N].
// Grid: (splits, G). Each CTA covers a contiguous range of 16-key tiles of
// one group, and each warp streams every 8th tile with the next tile's words
// prefetched into registers.

#include <cuda_runtime.h>
#include <stdint.h>

#include "qjl_internal.h"
#include "sign_mma.cuh"

namespace {

using namespace qjl_sign;
constexpr int kWarps = 8;

// NTR column tiles (4 queries each) per pass over the keys' bits.
template <int W, int NTR>
__global__ void __launch_bounds__(kWarps * 32) scores_mma_kernel(
    const uint32_t* __restrict__ bits, const float* __restrict__ norms, const float* __restrict__ sq,
    int64_t N, int J, float est_scale, int64_t tiles_per_cta, float* __restrict__ scores) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int NT = (J + 3) / 4;
  const int npass = (NT + NTR - 1) / NTR;
  const int NTP = npass * NTR;
  float* s_inv = reinterpret_cast<float*>(smem_raw);
  float* s_mul = s_inv + 64;
  int* s_qsum = reinterpret_cast<int*>(s_mul + 64);
  uint2* Btab = reinterpret_cast<uint2*>(smem_raw + 3 * 64 * 4);

  const int64_t gi = blockIdx.y;
  build_tables<W>(sq + gi * (int64_t)J * (32 * W), J, NTP, est_scale, s_inv, s_mul, s_qsum, Btab,
                  kWarps);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int64_t ntiles = (N + 15) >> 4;
  const int64_t t_begin = (int64_t)blockIdx.x * tiles_per_cta;
  const int64_t t_end = min(ntiles, t_begin + tiles_per_cta);
  const uint32_t* gbits = bits + gi * N * W;
  const float* gnorm = norms + gi * N;

  int64_t t = t_begin + warp;
  uint32_t cur[2][W / 4], nxt[2][W / 4];
  if (t < t_end) {
    load_words<W>(gbits, t * 16 + g, N, q, cur[0]);
    load_words<W>(gbits, t * 16 + g + 8, N, q, cur[1]);
  }
  for (; t < t_end; t += kWarps) {
    const int64_t tn = t + kWarps;
    if (tn < t_end) {
      load_words<W>(gbits, tn * 16 + g, N, q, nxt[0]);
      load_words<W>(gbits, tn * 16 + g + 8, N, q, nxt[1]);
    }
    const int64_t row0 = t * 16 + g, row1 = row0 + 8;
    float nrm[2] = {0.f, 0.f};
    if (row0 < N) nrm[0] = __ldg(gnorm + row0);
    if (row1 < N) nrm[1] = __ldg(gnorm + row1);
    for (int pass = 0; pass < npass; ++pass) {
      int acc[NTR][4][4];
#pragma unroll
      for (int a = 0; a < NTR; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[a][b][c] = 0;
#pragma unroll
      for (int p = 0; p < W / 8; ++p) {
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const uint32_t x0 = cur[0][2 * p] >> s, x1 = cur[1][2 * p] >> s;
          const uint32_t x2 = cur[0][2 * p + 1] >> s, x3 = cur[1][2 * p + 1] >> s;
#pragma unroll
          for (int Ji = 0; Ji < 4; ++Ji) {
            const uint32_t M = 0x01010101u << (2 * Ji);
            const int mu = 8 * p + 2 * Ji + s;
#pragma unroll
            for (int nt = 0; nt < NTR; ++nt) {
              const uint2 bb = Btab[((pass * NTR + nt) * W + mu) * 32 + lane];
              mma_u8s8(acc[nt][Ji], x0 & M, x1 & M, x2 & M, x3 & M, bb.x, bb.y);
            }
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < NTR; ++nt) {
        const int jq = (pass * NTR + nt) * 4 + q;
        if (jq >= J) continue;
        const float mul = s_mul[jq];
        const long long qs32 = 32LL * s_qsum[jq];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int64_t row = row0 + 8 * r;
          if (row >= N) continue;
          const int hi = ((acc[nt][0][2 * r] * 4 + acc[nt][1][2 * r]) * 4 + acc[nt][2][2 * r]) * 4 +
                         acc[nt][3][2 * r];
          const int lo = ((acc[nt][0][2 * r + 1] * 4 + acc[nt][1][2 * r + 1]) * 4 +
                          acc[nt][2][2 * r + 1]) * 4 + acc[nt][3][2 * r + 1];
          const long long D = 256LL * hi + lo - qs32;  // 32 * sum (2b - 1) Q
          scores[(gi * J + jq) * N + row] = mul * nrm[r] * ((float)D * 0.03125f);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < W / 4; ++k) {
      cur[0][k] = nxt[0][k];
      cur[1][k] = nxt[1][k];
    }
  }
}

// Any m (multiple of 32): one warp per key, lane l owns coordinate 32 w + l.
__global__ void __launch_bounds__(256) scores_simt_kernel(
    const uint32_t* __restrict__ bits, const float* __restrict__ norms, const float* __restrict__ sq,
    int64_t G, int64_t N, int J, int W, float est_scale, float* __restrict__ scores) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int m = 32 * W;
  for (int64_t key = warp; key < G * N; key += nwarps) {
    const int64_t gi = key / N, row = key - gi * N;
    const float nrm = __ldg(norms + key);
    for (int j = 0; j < J; ++j) {
      const float* s = sq + (gi * J + j) * m;
      float acc = 0.f;
      for (int w = 0; w < W; ++w) {
        const uint32_t word = __ldg(bits + key * W + w);
        const float v = __ldg(s + 32 * w + lane);
        acc += ((word >> lane) & 1u) ? v : -v;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) scores[(gi * J + j) * N + row] = est_scale * nrm * acc;
    }
  }
}

template <int W, int NTR>
qjl_status launch_mma(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G,
                      int64_t N, const float* sq, int J, float* scores, cudaStream_t st) {
  const int NT = (J + 3) / 4;
  const int NTP = ((NT + NTR - 1) / NTR) * NTR;
  const size_t smem = 3 * 64 * 4 + (size_t)NTP * W * 32 * sizeof(uint2);
  auto kern = scores_mma_kernel<W, NTR>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return qjl_check_launch("scores_mma_kernel smem attribute");
  const int64_t ntiles = (N + 15) / 16;
  const int64_t target = (int64_t)qjl_num_sms(P->device) * 4;
  int64_t splits = (target + G - 1) / G;
  splits = std::max<int64_t>(1, std::min<int64_t>(splits, (ntiles + kWarps - 1) / kWarps));
  const int64_t tpc = (ntiles + splits - 1) / splits;
  splits = (ntiles + tpc - 1) / tpc;
  dim3 grid((unsigned)splits, (unsigned)G);
  kern<<<grid, kWarps * 32, smem, st>>>(bits, norms, sq, N, J, P->est_scale, tpc, scores);
  return qjl_check_launch("scores_mma_kernel");
}

}  // namespace

bool scores_mma_supported(int m) { return m == 256 || m == 512 || m == 1024; }

qjl_status launch_scores(const qjl_projection* P, const uint32_t* bits, const float* norms,
                         int64_t G, int64_t N, const float* sq, int J, float* scores, cudaStream_t st) {
  if (G > 65535) return qjl_set_error(QJL_ERR_UNSUPPORTED, "groups > 65535");
  const int NTR = J > 4 ? 2 : 1;
  switch (scores_mma_supported(P->m) ? P->m : 0) {
    case 256: return NTR == 1 ? launch_mma<8, 1>(P, bits, norms, G, N, sq, J, scores, st)
                              : launch_mma<8, 2>(P, bits, norms, G, N, sq, J, scores, st);
    case 512: return NTR == 1 ? launch_mma<16, 1>(P, bits, norms, G, N, sq, J, scores, st)
                              : launch_mma<16, 2>(P, bits, norms, G, N, sq, J, scores, st);
    case 1024: return NTR == 1 ? launch_mma<32, 1>(P, bits, norms, G, N, sq, J, scores, st)
                               : launch_mma<32, 2>(P, bits, norms, G, N, sq, J, scores, st);
    default: break;
  }
  const int64_t want = (G * N + 7) / 8;
  const int blocks = (int)std::min<int64_t>(want, (int64_t)qjl_num_sms(P->device) * 16);
  scores_simt_kernel<<<blocks, 256, 0, st>>>(bits, norms, sq, G, N, J, P->m / 32, P->est_scale, scores);
  return qjl_check_launch("scores_simt_kernel");
}
