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
#include "mbarrier.cuh"
#include "sign_mma.cuh"

namespace {

using namespace qjl_sign;
using qjl_sync::named_sync;
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

// ---------------------------------------------------------------------------
// Streaming fused decode for one query per group (the decode step proper).
// Each CTA owns one split of one group. A producer lane moves stages of 64
// tokens per consumer warp (bits, norms, codes, scales, zeros) into a
// shared-memory ring with cp.async.bulk. The consumer warps (12 at m = 256,
// d <= 128, three per SM sub-partition, so that their latencies overlap;
// 8 where 12 would spill, where two stages would not fit, and for the paged
// cache, whose 256-token pages split 768-token stages into three copies per
// array and measured slower) take 64 tokens each per stage:
//   * estimates by the class-in-column s8 MMAs (one fragment per tile, two
//     xor-shuffles merge the four weight classes; each lane ends with the
//     logits of 2 tokens);
//   * an online softmax per warp (base 2);
//   * p * v_hat accumulated per lane for its d/32 channels, which lie in one
//     32-channel group: acc_c += (p s) (code_c 4^c) and accz += p z. The
//     term code_c 4^c comes out exactly as (word & (3 << 2c)) | 2^23 - 2^23,
//     with no shift and no int-to-float conversion, and the 4^c is divided
//     out once at the end.
// The warps are merged in shared memory into one (max, sum, acc[d]) partial.
template <int W, int CPL, bool PAGED>
__host__ __device__ constexpr int ds_consumers() { return (W == 8 && CPL <= 4 && !PAGED) ? 12 : 8; }
template <int W, int CPL, bool PAGED>
__host__ __device__ constexpr int ds_threads() { return (ds_consumers<W, CPL, PAGED>() + 1) * 32; }
template <int W, int CPL, bool PAGED>
__host__ __device__ constexpr int ds_stage() { return ds_consumers<W, CPL, PAGED>() * 64; }

__device__ __forceinline__ void mma_u8s8_acc(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8s8_zero(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// acc_j += (p s) (code_j 4^(j % 8)) for this lane's PL channels of one token, and accz += p z.
// The lane's channels are c0 .. c0 + PL - 1 (one 32-channel group). The code words are read in
// 8-channel chunks (16 bits each), so code_j 4^(j % 8) = float(2^23 | (chunk & (3 << 2(j % 8))))
// - 2^23 exactly: the bits stay in the mantissa, and no int-to-float conversion is needed.
// Channel pairs go through sm_100's packed fp32 subtract and FMA.
template <int PL>
__device__ __forceinline__ void pv_accum(const uint32_t* cw, int c0, uint16_t sraw, uint16_t zraw, float pt,
                                         float (&acc)[PL], float& accz) {
  const float pw = pt * __half2float(__ushort_as_half(sraw));
  accz = fmaf(pt, __half2float(__ushort_as_half(zraw)), accz);
  constexpr int NCH = PL < 8 ? 1 : PL / 8;     // 8-channel chunks
  constexpr int CL = PL < 8 ? PL : 8;          // channels per chunk
#pragma unroll
  for (int h = 0; h < NCH; ++h) {
    // chunk h covers channels c0 + 8h ..; it sits in word (c0 + 8h) / 16 at bit 2 ((c0 + 8h) % 16)
    const uint32_t chunk = PL < 16 ? cw[0] >> (2 * ((c0 + 8 * h) & 15)) : cw[h >> 1] >> (16 * (h & 1));
#pragma unroll
    for (int k = 0; k < CL; k += 2) {
      const uint32_t u0 = 0x4B000000u | (chunk & (3u << (2 * k)));
      const uint32_t u1 = 0x4B000000u | (chunk & (3u << (2 * k + 2)));
      float& a0 = acc[8 * h + k];
      float& a1 = acc[8 * h + k + 1];
      asm("{\n\t.reg .b64 f, m, w, a;\n\t"
          "mov.b64 f, {%2, %3};\n\t"
          "mov.b64 m, {%4, %4};\n\t"
          "sub.rn.f32x2 f, f, m;\n\t"
          "mov.b64 w, {%5, %5};\n\t"
          "mov.b64 a, {%0, %1};\n\t"
          "fma.rn.f32x2 a, w, f, a;\n\t"
          "mov.b64 {%0, %1}, a;\n\t}"
          : "+f"(a0), "+f"(a1)
          : "r"(u0), "r"(u1), "f"(8388608.f), "f"(pw));
    }
  }
}

struct DsLayout {
  // byte offsets inside one stage
  uint32_t bits, norms, codes, scale, zero, bytes;
};

__host__ __device__ inline DsLayout ds_layout(int W, int d, int stage) {
  DsLayout L;
  L.bits = 0;
  L.norms = L.bits + stage * W * 4;
  L.codes = L.norms + stage * 4;
  L.scale = L.codes + stage * (d / 16) * 4;
  L.zero = L.scale + stage * (d / 32) * 2;
  L.bytes = L.zero + stage * (d / 32) * 2;
  return L;
}

// Work split of the one-query streaming kernel: the flattened (group, 16-token tile) space is cut
// into ncta equal slices, one persistent CTA each (at least 64 tiles per CTA), so every SM runs
// one uninterrupted ring. A CTA writes one partial per group its slice touches: at most maxseg.
constexpr int64_t kStreamCTAs = 148;

struct StreamPlan {
  int64_t ntg, TT, ncta, maxseg;   // tiles per group, all tiles, CTAs, partial slots per CTA
};

__host__ __device__ inline StreamPlan stream_plan(int64_t G, int64_t N) {
  StreamPlan p;
  p.ntg = (N + 15) / 16;
  p.TT = G * p.ntg;
  const int64_t c = p.TT / 64;
  p.ncta = c < 1 ? 1 : (c > kStreamCTAs ? kStreamCTAs : c);
  const int64_t per = (p.TT + p.ncta - 1) / p.ncta;
  p.maxseg = (per + p.ntg - 1) / p.ntg + 1;
  return p;
}

// first tile of CTA c (c = ncta gives TT)
__host__ __device__ inline int64_t stream_tile0(const StreamPlan& p, int64_t c) { return c * p.TT / p.ncta; }

// the CTA whose slice holds tile t
__host__ __device__ inline int64_t stream_cta_of(const StreamPlan& p, int64_t t) {
  int64_t c = t * p.ncta / p.TT;
  while (c + 1 < p.ncta && stream_tile0(p, c + 1) <= t) ++c;
  while (c > 0 && stream_tile0(p, c) > t) --c;
  return c;
}

__device__ __forceinline__ bool bulk_ok(const void* src, uint32_t bytes) {
  return (((uintptr_t)src & 15u) == 0) && (bytes % 16u == 0);
}

// PAGED reads group g's tokens t < seq_lens[g] through the block table
// (PagedRead); N is then the bound max_len. Every array is bulk-copied per page
// segment, rounded up to 4 tokens (never past the page: pages hold a multiple
// of 16 tokens, and segments start 16-token aligned).
template <int W, int CPL, bool PAGED>
__global__ void __launch_bounds__(ds_threads<W, CPL, PAGED>(), 1) decode_stream_kernel(
    const uint32_t* __restrict__ bits, const float* __restrict__ norms, const uint32_t* __restrict__ codes,
    const uint16_t* __restrict__ scale, const uint16_t* __restrict__ zero, const float* __restrict__ sq, int64_t G,
    int64_t N, int NS, float est_scale, float logit_scale, float* __restrict__ ws, int* __restrict__ err,
    PagedRead pr) {
  using namespace qjl_sync;
  constexpr int d = 32 * CPL;
  constexpr int kDsConsumers = ds_consumers<W, CPL, PAGED>();
  constexpr int kDsStage = ds_stage<W, CPL, PAGED>();
  constexpr int CW = d / 16;  // code words per token
  constexpr int GW = d / 32;  // scale / zero halves per token
  constexpr int KT = 4;       // 16-token tiles per warp per stage
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* s_inv = reinterpret_cast<float*>(smem_raw);
  float* s_mul = s_inv + 64;
  int* s_qsum = reinterpret_cast<int*>(s_mul + 64);
  uint2* Btab = reinterpret_cast<uint2*>(smem_raw + 3 * 64 * 4);
  float* s_red = reinterpret_cast<float*>(Btab + W * 32);                      // [kDsConsumers][d + 2]
  unsigned char* ring = reinterpret_cast<unsigned char*>(s_red + kDsConsumers * (d + 2));
  const DsLayout L = ds_layout(W, d, kDsStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)NS * L.bytes);
  uint64_t* empty = full + NS;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // this CTA's slice of the flattened (group, 16-token tile) space, cut into one segment per group
  const StreamPlan plan = stream_plan(G, N);
  const int64_t tb = stream_tile0(plan, blockIdx.x), te = stream_tile0(plan, blockIdx.x + 1);
  const int64_t g_first = tb / plan.ntg, g_last = (te - 1) / plan.ntg;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDsConsumers);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kDsConsumers) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      bool stop = false;
      for (int64_t gi = g_first; gi <= g_last && !stop; ++gi) {
        const int64_t t0 = 16 * (max(tb, gi * plan.ntg) - gi * plan.ntg);
        int64_t t1 = min(N, 16 * (min(te, (gi + 1) * plan.ntg) - gi * plan.ntg));
        if (PAGED) t1 = min(t1, min(max((int64_t)__ldg(pr.seq_lens + gi), (int64_t)0), N));
        const int64_t nst = t1 > t0 ? (t1 - t0 + kDsStage - 1) / kDsStage : 0;
        for (int64_t k = 0; k < nst; ++k, ++issued) {
          if (!mbar_wait(&empty[s], ph ^ 1u)) { atomicOr(err, 1); stop = true; break; }
          const int64_t n0 = t0 + k * kDsStage;
          const uint32_t cnt = (uint32_t)(t1 - n0 < kDsStage ? t1 - n0 : kDsStage);
          unsigned char* st = ring + (size_t)s * L.bytes;
          const uint32_t off[5] = {L.bits, L.norms, L.codes, L.scale, L.zero};
          const uint32_t per_tok[5] = {W * 4, 4, CW * 4, GW * 2, GW * 2};
          if constexpr (PAGED) {
            const int T = pr.page_tokens;
            uint32_t tx = 0;
            for (int pass = 0; pass < 2; ++pass) {
              if (pass == 1) mbar_expect_tx(&full[s], tx);
              for (int64_t lo = n0; lo < n0 + cnt;) {
                const int64_t pi = lo / T;
                const int64_t hi = min(n0 + (int64_t)cnt, (pi + 1) * T);
                const uint32_t len4 = (uint32_t)((hi - lo + 3) & ~3);
                const int pg = pi < pr.max_pages ? __ldg(pr.table + gi * (int64_t)pr.max_pages + pi) : -1;
                if (pg >= 0 && (int64_t)pg < pr.num_pages) {
                  const int64_t prow = (int64_t)pg * T + (lo - pi * T);
                  const void* src[5] = {bits + prow * W, norms + prow, codes + prow * CW, scale + prow * GW,
                                        zero + prow * GW};
                  for (int a = 0; a < 5; ++a) {
                    if (pass == 0) tx += len4 * per_tok[a];
                    else bulk_g2s(st + off[a] + (lo - n0) * per_tok[a], src[a], len4 * per_tok[a], &full[s]);
                  }
                } else if (pass == 0) {
                  atomicOr(err, QJL_DEVERR_PAGE);  // a bad page id: its tokens keep stale stage data
                }
                lo = hi;
              }
            }
          } else {
            const int64_t row = gi * N + n0;
            const void* src[5] = {bits + row * W, norms + row, codes + row * CW, scale + row * GW, zero + row * GW};
            uint32_t nb[5];
            for (int a = 0; a < 5; ++a) nb[a] = cnt * per_tok[a];
            uint32_t tx = 0;
            for (int a = 0; a < 5; ++a)
              if (bulk_ok(src[a], nb[a])) tx += nb[a];
            mbar_expect_tx(&full[s], tx);
            for (int a = 0; a < 5; ++a)
              if (bulk_ok(src[a], nb[a])) bulk_g2s(st + off[a], src[a], nb[a], &full[s]);
          }
          if (++s == NS) { s = 0; ph ^= 1u; }
        }
      }
      // do not leave while copies are in flight
      const int used = issued < NS ? (int)issued : NS;
      for (int j = 0; j < used; ++j) {
        int stg = s - 1 - j;
        uint32_t p = ph;
        if (stg < 0) { stg += NS; p ^= 1u; }
        if (!mbar_wait(&full[stg], p)) atomicOr(err, 2);
      }
    }
    return;
  }

  // consumers: one segment (one group) at a time; the ring carries on across segments
  int s = 0;
  uint32_t ph = 0;
  bool dead = false;  // a timed-out wait: keep the loop's barriers, skip the work
  for (int64_t gi = g_first; gi <= g_last; ++gi) {
  const int64_t t0 = 16 * (max(tb, gi * plan.ntg) - gi * plan.ntg);
  int64_t t1 = min(N, 16 * (min(te, (gi + 1) * plan.ntg) - gi * plan.ntg));
  if (PAGED) t1 = min(t1, min(max((int64_t)__ldg(pr.seq_lens + gi), (int64_t)0), N));
  const int64_t nst = t1 > t0 ? (t1 - t0 + kDsStage - 1) / kDsStage : 0;
  build_tables_dig<W>(sq + gi * (int64_t)(32 * W), 1, 1, true, est_scale, s_inv, s_mul, s_qsum, Btab, kDsConsumers,
                      1);
  uint2 breg[W];
#pragma unroll
  for (int mu = 0; mu < W; ++mu) breg[mu] = Btab[mu * 32 + lane];
  const float xmul = s_mul[0] * logit_scale * 1.4426950408889634f;  // to log2-domain logits
  const uint32_t qsum = (uint32_t)s_qsum[0];
  const int gq = lane >> 2, q = lane & 3;
  // value accumulation: lane = 8 tg + cs takes channels c0 = cs PL .. c0 + PL - 1 of the tokens
  // of group tg. At step j a warp covers four consecutive rows 4 (j & 3) + tg of its tile j / 4,
  // so the four groups read adjacent tokens (conflict-free) and all fetch their probability from
  // the same register (p0 for rows < 8, p1 above) of the MMA-layout lanes.
  constexpr int PL = d / 8;
  const int tg = lane >> 3, cs = lane & 7;
  const int c0 = cs * PL;
  const int grp = c0 >> 5, cwi = c0 >> 4;

  float m_run = -INFINITY, l_lane = 0.f, accz = 0.f, acc[PL];
#pragma unroll
  for (int c = 0; c < PL; ++c) acc[c] = 0.f;
  for (int64_t k = 0; k < nst; ++k) {
    const int64_t n0 = t0 + k * kDsStage;
    const int cnt = (int)(t1 - n0 < kDsStage ? t1 - n0 : kDsStage);
    const int64_t row0 = gi * N + n0;
    if (!dead && !__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) { atomicOr(err, 4); dead = true; }
    if (!dead) {
    const unsigned char* st = ring + (size_t)s * L.bytes;
    const uint32_t* sb = reinterpret_cast<const uint32_t*>(st + L.bits);
    const bool nb_norm = PAGED || bulk_ok(norms + row0, (uint32_t)cnt * 4);
    const bool nb_codes = PAGED || bulk_ok(codes + row0 * CW, (uint32_t)cnt * CW * 4);
    const bool nb_scale = PAGED || bulk_ok(scale + row0 * GW, (uint32_t)cnt * GW * 2);
    const bool nb_zero = PAGED || bulk_ok(zero + row0 * GW, (uint32_t)cnt * GW * 2);
    const float* snorm = reinterpret_cast<const float*>(st + L.norms);
    const uint32_t* scodes = reinterpret_cast<const uint32_t*>(st + L.codes);
    const uint16_t* sscale = reinterpret_cast<const uint16_t*>(st + L.scale);
    const uint16_t* szero = reinterpret_cast<const uint16_t*>(st + L.zero);

    // ---- estimates of this warp's KT tiles (tiles warp + 8 t2)
    uint32_t w0[KT][W / 4], w1[KT][W / 4];
#pragma unroll
    for (int t2 = 0; t2 < KT; ++t2) {
      const int rA = (warp + t2 * kDsConsumers) * 16 + gq;
#pragma unroll
      for (int kk = 0; kk < W / 8; ++kk) {
        const uint2 a = *reinterpret_cast<const uint2*>(sb + rA * W + q * (W / 4) + 2 * kk);
        const uint2 b = *reinterpret_cast<const uint2*>(sb + (rA + 8) * W + q * (W / 4) + 2 * kk);
        w0[t2][2 * kk] = a.x; w0[t2][2 * kk + 1] = a.y;
        w1[t2][2 * kk] = b.x; w1[t2][2 * kk + 1] = b.y;
      }
    }
    // shift-window sign sums (build_tables_dig): the A fragments are the words shifted right by
    // s = 0..7, unmasked; both B column halves carry the query's four digits
    int accm[KT][4];
#pragma unroll
    for (int p = 0; p < W / 8; ++p) {
#pragma unroll
      for (int sh = 0; sh < 8; ++sh) {
        const uint2 bb = breg[8 * p + sh];
#pragma unroll
        for (int t2 = 0; t2 < KT; ++t2) {
          const uint32_t a0 = w0[t2][2 * p] >> sh, a1 = w1[t2][2 * p] >> sh;
          const uint32_t a2 = w0[t2][2 * p + 1] >> sh, a3 = w1[t2][2 * p + 1] >> sh;
          if (p == 0 && sh == 0) mma_u8s8_zero(accm[t2], a0, a1, a2, a3, bb.x, bb.y);
          else mma_u8s8_acc(accm[t2], a0, a1, a2, a3, bb.x, bb.y);
        }
      }
    }
    // lane (gq, q = 2 half + par) holds digits (2 par, 2 par + 1) of rows gq and gq + 8. The pair
    // (q, q ^ 1) completes row gq + 8 par of tile 2k + half: x[k], k = 0, 1.
    const int par = q & 1, half = q >> 1;
    const uint32_t hm = par ? 65536u : 1u;
    float x[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      int cc[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) cc[j] = half ? accm[2 * k + 1][j] : accm[2 * k][j];
      const uint32_t P0 = (uint32_t)cc[0] * hm + (uint32_t)cc[1] * (hm << 8);
      const uint32_t P1 = (uint32_t)cc[2] * hm + (uint32_t)cc[3] * (hm << 8);
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, par ? P0 : P1, 1);
      const uint32_t tot = (par ? P1 : P0) + recv;
      const int row = (warp + (2 * k + half) * kDsConsumers) * 16 + gq + 8 * par;
      if (row < cnt) {
        const float nrm = nb_norm ? snorm[row] : __ldg(norms + row0 + row);
        x[k] = xmul * nrm * (float)(int)(2u * tot - qsum);
      } else {
        x[k] = -INFINITY;
      }
    }
    // ---- online softmax over the warp's 64 tokens
    float mt = fmaxf(x[0], x[1]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
    const float mn = fmaxf(m_run, mt);
    if (mn != -INFINITY) {
      const float corr = exp2f(m_run - mn);
      m_run = mn;
      l_lane *= corr;
      accz *= corr;
#pragma unroll
      for (int c = 0; c < PL; ++c) acc[c] *= corr;
      const float p0 = exp2f(x[0] - mn), p1 = exp2f(x[1] - mn);
      l_lane += p0 + p1;
      // ---- p * v_hat: the token at (tile t2, row) has its p in lane 4 (row % 8) + 2 (t2 % 2) + row / 8,
      // register t2 / 2
      if (cnt == kDsStage && nb_codes && nb_scale && nb_zero) {
        // whole stage in shared memory: no per-token bounds or source selection
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t2 = j >> 2, row = 4 * (j & 3) + tg;
          const int tok = (warp + t2 * kDsConsumers) * 16 + row;
          const float pt = __shfl_sync(0xffffffffu, (t2 >> 1) ? p1 : p0, 4 * (row & 7) + 2 * (t2 & 1) + (row >> 3));
          pv_accum<PL>(scodes + tok * CW + cwi, c0, sscale[tok * GW + grp], szero[tok * GW + grp], pt, acc, accz);
        }
      } else {
#pragma unroll 1
        for (int j = 0; j < 16; ++j) {
          const int t2 = j >> 2, row = 4 * (j & 3) + tg;
          const int tok = (warp + t2 * kDsConsumers) * 16 + row;
          const float pt = __shfl_sync(0xffffffffu, (t2 >> 1) ? p1 : p0, 4 * (row & 7) + 2 * (t2 & 1) + (row >> 3));
          if (tok >= cnt) continue;
          uint32_t cwd[PL < 16 ? 1 : PL / 16];
#pragma unroll
          for (int i = 0; i < (PL < 16 ? 1 : PL / 16); ++i)
            cwd[i] = nb_codes ? scodes[tok * CW + cwi + i] : __ldg(codes + (row0 + tok) * CW + cwi + i);
          const uint16_t sr = nb_scale ? sscale[tok * GW + grp] : __ldg(scale + (row0 + tok) * GW + grp);
          const uint16_t zr = nb_zero ? szero[tok * GW + grp] : __ldg(zero + (row0 + tok) * GW + grp);
          pv_accum<PL>(cwd, c0, sr, zr, pt, acc, accz);
        }
      }
    }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == NS) { s = 0; ph ^= 1u; }
  }

  // ---- merge the consumer warps: (m, l, acc[d]) per warp, then one partial per CTA
  float l_w = l_lane;
#pragma unroll
  for (int o = 16; o; o >>= 1) l_w += __shfl_xor_sync(0xffffffffu, l_w, o);
  // the four token groups hold the same channels: add them (lanes cs, cs + 8, cs + 16, cs + 24)
#pragma unroll
  for (int c = 0; c < PL; ++c) {
    acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 8);
    acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], 16);
  }
  accz += __shfl_xor_sync(0xffffffffu, accz, 8);
  accz += __shfl_xor_sync(0xffffffffu, accz, 16);
  float* red = s_red + warp * (d + 2);
  if (tg == 0) {
#pragma unroll
    for (int c = 0; c < PL; ++c) red[2 + c0 + c] = acc[c] * (1.0f / (float)(1 << (2 * (c & 7)))) + accz;
  }
  if (lane == 0) {
    red[0] = m_run;
    red[1] = l_w;
  }
  named_sync(1, kDsConsumers * 32);
  const int64_t slot = (int64_t)blockIdx.x * plan.maxseg + (gi - g_first);
  for (int idx = threadIdx.x; idx < d + 2; idx += kDsConsumers * 32) {
    float M = -INFINITY;
    for (int w = 0; w < kDsConsumers; ++w) M = fmaxf(M, s_red[w * (d + 2)]);
    float v = 0.f;
    if (idx == 0) {
      v = M;
    } else {
      for (int w = 0; w < kDsConsumers; ++w) {
        const float mw = s_red[w * (d + 2)];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        v += f * s_red[w * (d + 2) + idx];
      }
    }
    ws[slot * (d + 2) + idx] = v;
  }
  }  // segments
}

// The one-query partials of group g: the CTAs whose tile ranges meet g's tiles, each in slot
// (c, g - first group of c). out[g][c] = sum acc 2^(m - M) / sum l 2^(m - M).
__global__ void __launch_bounds__(128) decode_combine_stream_kernel(const float* __restrict__ ws, int64_t G, int64_t N,
                                                                    int d, float* __restrict__ out) {
  const int64_t g = blockIdx.x;
  if (g >= G) return;
  const StreamPlan plan = stream_plan(G, N);
  const int64_t c_lo = stream_cta_of(plan, g * plan.ntg), c_hi = stream_cta_of(plan, (g + 1) * plan.ntg - 1);
  auto entry = [&](int64_t c) {
    return ws + (c * plan.maxseg + (g - stream_tile0(plan, c) / plan.ntg)) * (d + 2);
  };
  float M = -INFINITY;
  for (int64_t c = c_lo; c <= c_hi; ++c) M = fmaxf(M, entry(c)[0]);
  float Lsum = 0.f;
  for (int64_t c = c_lo; c <= c_hi; ++c) {
    const float* e = entry(c);
    Lsum += (e[0] == -INFINITY) ? 0.f : e[1] * exp2f(e[0] - M);
  }
  const float invL = Lsum > 0.f ? 1.f / Lsum : 0.f;  // a group with no tokens (paged, seq_lens 0) gives 0
  for (int ch = threadIdx.x; ch < d; ch += blockDim.x) {
    float v = 0.f;
    for (int64_t c = c_lo; c <= c_hi; ++c) {
      const float* e = entry(c);
      if (e[0] != -INFINITY) v += e[2 + ch] * exp2f(e[0] - M);
    }
    out[g * d + ch] = v * invL;
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

template <int W, int CPL, bool PAGED = false>
qjl_status launch_stream(const qjl_projection* P, const uint32_t* bits, const float* norms, const uint32_t* codes,
                         const uint16_t* scale, const uint16_t* zero, int64_t G, int64_t N, const float* sq,
                         float softmax_scale, float* out, float* ws, cudaStream_t st,
                         const PagedRead& pr = PagedRead()) {
  constexpr int d = 32 * CPL;
  constexpr int kDsConsumers = ds_consumers<W, CPL, PAGED>();
  constexpr int kDsThreads = ds_threads<W, CPL, PAGED>();
  const DsLayout L = ds_layout(W, d, ds_stage<W, CPL, PAGED>());
  int NS = 4;  // one CTA per SM: three 768-token stages (194 KB) at d = 128, m = 256
  while (NS > 2 && 3 * 64 * 4 + (size_t)W * 32 * sizeof(uint2) + (size_t)kDsConsumers * (d + 2) * 4 +
                       (size_t)NS * L.bytes + (size_t)2 * NS * 8 > 220 * 1024)
    --NS;
  const size_t smem = 3 * 64 * 4 + (size_t)W * 32 * sizeof(uint2) + (size_t)kDsConsumers * (d + 2) * 4 +
                      (size_t)NS * L.bytes + (size_t)2 * NS * 8;
  auto kern = decode_stream_kernel<W, CPL, PAGED>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return qjl_check_launch("decode_stream_kernel smem attribute");
  int* err = qjl_error_flag(P->device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  const StreamPlan plan = stream_plan(G, N);
  qjl_log_launch("decode_stream_kernel", plan.ncta, kDsThreads, smem, 1);
  kern<<<(unsigned)plan.ncta, kDsThreads, smem, st>>>(bits, norms, codes, scale, zero, sq, G, N, NS, P->est_scale,
                                                      softmax_scale, ws, err, pr);
  qjl_status s = qjl_check_launch("decode_stream_kernel");
  if (s != QJL_OK) return s;
  decode_combine_stream_kernel<<<(unsigned)G, 128, 0, st>>>(ws, G, N, d, out);
  return qjl_check_launch("decode_combine_stream_kernel");
}

template <int W>
qjl_status launch_w(const qjl_projection* P, const uint32_t* bits, const float* norms,
                    const uint32_t* codes, const uint16_t* scale, const uint16_t* zero, int64_t G,
                    int64_t N, const float* sq, int J, float softmax_scale, float* out, float* ws,
                    cudaStream_t st) {
  if (J == 1) {
    switch (P->d) {
      case 32: return launch_stream<W, 1>(P, bits, norms, codes, scale, zero, G, N, sq, softmax_scale, out, ws, st);
      case 64: return launch_stream<W, 2>(P, bits, norms, codes, scale, zero, G, N, sq, softmax_scale, out, ws, st);
      case 128: return launch_stream<W, 4>(P, bits, norms, codes, scale, zero, G, N, sq, softmax_scale, out, ws, st);
      case 256: return launch_stream<W, 8>(P, bits, norms, codes, scale, zero, G, N, sq, softmax_scale, out, ws, st);
    }
  }
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
  if (J == 1) {
    // the one-query kernel: maxseg partial slots per persistent CTA
    const StreamPlan p = stream_plan(G, N);
    return (size_t)p.ncta * (size_t)p.maxseg * (size_t)(d + 2) * sizeof(float);
  }
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

size_t decode_paged_workspace_bytes(int64_t groups, int64_t max_len, int d) {
  return decode_workspace_bytes(groups, 1, max_len, d);
}

qjl_status launch_decode_paged(const qjl_projection* P, const uint32_t* bits_pool, const float* norms_pool,
                               const uint32_t* codes_pool, const uint16_t* scale_pool, const uint16_t* zero_pool,
                               const PagedRead& pr, int64_t G, int64_t max_len, const float* sq,
                               float softmax_scale, float* out, void* ws, cudaStream_t st) {
  if (P->m != 256 || P->d != 128)
    return qjl_set_error(QJL_ERR_UNSUPPORTED, "paged decode attention supports d = 128 and m = 256");
  return launch_stream<8, 4, true>(P, bits_pool, norms_pool, codes_pool, scale_pool, zero_pool, G, max_len, sq,
                                   softmax_scale, out, reinterpret_cast<float*>(ws), st, pr);
}
