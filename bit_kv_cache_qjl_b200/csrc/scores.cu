// Asymmetric QJL estimator over packed sign bits (QJL abstract, "Majid
// Daliri" page): est = c * alpha * ||k|| * sum_i (2 b_i - 1) * Sq_i.
//
// Decode reads every key's bits once per query step (KIVI abstract: the
// whole cache is loaded per generated token), so the kernel must stay at the
// HBM roof, where each SM has under two clocks per 40-byte key. A plain
// bit-serial sign-dot costs several instructions per bit, and on sm_100a the
// 1-bit and 4-bit mma.sync forms are emulated, so the sign sums run on the
// u8 x s8 tensor-core path (mma.sync m16n8k32). A u8 A element carries at
// most one new bit per byte against arbitrary weights, so a 32-bit sign word
// needs eight A registers (32 k-slots); two ways of building them are used:
//
//   * Shift windows (one or two queries per group, build_tables_dig in
//     sign_mma.cuh): the eight registers are the word shifted right by
//     s = 0..7, unmasked, and B holds Q times the inverse of the windows'
//     unit-triangular weight matrix, modulo 2^32, as four int8 digits in four
//     columns. Seven shifts per word, and Sq keeps 31 - log2(m) bits.
//   * Weight classes (three or four queries, build_tables): Sq is rounded to
//     16-bit fixed point and split into int8 hi/lo columns, so one n8 tile
//     serves four queries. A register is (word >> s) & (0x01010101 << 2c):
//     four bits worth 4^c, one AND per 4 bits. Four accumulators (c = 0..3)
//     are merged exactly in int32. Its only error is the 16-bit rounding of
//     Sq, at most m * max|Sq| / 65278 before scaling.
// In both, the sign sums are exact integers; the estimate is
// (2 sum b Q - sum Q) times the scale, converted to fp32 once.
//
// Layout: bits [G][N][W] uint32, norms [G][N], sq [G][J][m], scores [G][J][N].
// Keys stream through a shared-memory ring filled by cp.async.bulk from one
// producer lane; persistent CTAs each take a contiguous range of (group,
// stage) items.

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <algorithm>
#include <type_traits>

#include "qjl_internal.h"
#include "mbarrier.cuh"
#include "sign_mma.cuh"

namespace {

using namespace qjl_sign;

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
// Decode fast path: at most 4 queries per group (one n8 column tile), so each
// consumer thread keeps its B fragments in registers (2 W of them), loaded
// from the shared table once per group. The first MMA of each accumulator
// takes a zero C operand. Stages are 512 keys (16 KB of bits at m = 256) and
// two tiles' MMAs are interleaved per consumer warp.
constexpr int kDecStageKeys = 512;
constexpr int kDecConsumers = 8;                                         // consumer warps
constexpr int kDecThreads = (kDecConsumers + 1) * 32;
constexpr int kDecTilesPerWarp = kDecStageKeys / 16 / kDecConsumers;    // 4

__device__ __forceinline__ void mma_u8s8_zc(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

template <int W>
__global__ void __launch_bounds__(kDecThreads, 2) scores_decode_kernel(
    const uint32_t* __restrict__ bits, const float* __restrict__ norms, const float* __restrict__ sq,
    int64_t G, int64_t N, int J, int NS, float est_scale, int64_t items_per_cta, float* __restrict__ scores,
    int* __restrict__ err) {
  using namespace qjl_sync;
  constexpr int SK = kDecStageKeys;
  constexpr int KT = 2;   // tiles whose MMA chains are interleaved per warp
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* s_inv = reinterpret_cast<float*>(smem_raw);
  float* s_mul = s_inv + 64;
  int* s_qsum = reinterpret_cast<int*>(s_mul + 64);
  uint2* Btab = reinterpret_cast<uint2*>(smem_raw + 3 * 64 * 4);
  uint32_t* sbits = reinterpret_cast<uint32_t*>(Btab + (size_t)W * 32);     // [NS][SK * W]
  float* snorm = reinterpret_cast<float*>(sbits + (size_t)NS * SK * W);    // [NS][SK]
  uint64_t* full = reinterpret_cast<uint64_t*>(snorm + (size_t)NS * SK);
  uint64_t* empty = full + NS;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t cpg = (N + SK - 1) / SK;
  const int64_t total = G * cpg;
  const int64_t i0 = (int64_t)blockIdx.x * items_per_cta;
  const int64_t i1 = min(total, i0 + items_per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecConsumers);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kDecConsumers) {
    if (lane == 0) {
      int64_t g = i0 / cpg, c = i0 - (i0 / cpg) * cpg;
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t it = i0; it < i1; ++it, ++issued) {
        if (!mbar_wait(&empty[s], ph ^ 1u)) { atomicOr(err, 1); break; }
        const int64_t n0 = c * SK;
        const int cnt = (int)(N - n0 < SK ? N - n0 : SK);
        const float* nsrc = norms + g * N + n0;
        const bool nbulk = (((uintptr_t)nsrc & 15u) == 0) && (cnt % 4 == 0);
        const uint32_t bbytes = (uint32_t)cnt * W * 4;
        mbar_expect_tx(&full[s], bbytes + (nbulk ? (uint32_t)cnt * 4 : 0u));
        bulk_g2s(sbits + (size_t)s * SK * W, bits + (g * N + n0) * W, bbytes, &full[s]);
        if (nbulk) bulk_g2s(snorm + (size_t)s * SK, nsrc, (uint32_t)cnt * 4, &full[s]);
        if (++c == cpg) { c = 0; ++g; }
        if (++s == NS) { s = 0; ph ^= 1u; }
      }
      const int used = issued < NS ? (int)issued : NS;
      for (int j = 0; j < used; ++j) {
        int st = s - 1 - j;
        uint32_t p = ph;
        if (st < 0) { st += NS; p ^= 1u; }
        if (!mbar_wait(&full[st], p)) atomicOr(err, 2);
      }
    }
    return;
  }

  const int gq = lane >> 2, q = lane & 3;
  int64_t g = i0 / cpg, c = i0 - (i0 / cpg) * cpg;
  int64_t cur_g = -1;
  int s = 0;
  uint32_t ph = 0;
  uint2 breg[W];
  float mul = 0.f;
  int qs32 = 0;
  bool dead = false;  // a timed-out wait: keep the loop's barriers, skip the work
  for (int64_t it = i0; it < i1; ++it) {
    const int64_t n0 = c * SK;
    const int cnt = (int)(N - n0 < SK ? N - n0 : SK);
    if (g != cur_g) {
      named_sync(1, kDecConsumers * 32);
      build_tables<W>(sq + g * (int64_t)J * (32 * W), J, 1, est_scale, s_inv, s_mul, s_qsum, Btab, kDecConsumers,
                      1);
#pragma unroll
      for (int mu = 0; mu < W; ++mu) breg[mu] = Btab[mu * 32 + lane];
      mul = q < J ? s_mul[q] * 0.03125f : 0.f;
      qs32 = q < J ? 32 * s_qsum[q] : 0;
      cur_g = g;
    }
    if (!dead && !__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) { atomicOr(err, 4); dead = true; }
    if (!dead) {
    const float* nsrc = norms + g * N + n0;
    const bool nbulk = (((uintptr_t)nsrc & 15u) == 0) && (cnt % 4 == 0);
    const uint32_t* sb = sbits + (size_t)s * SK * W;
    const float* sn = snorm + (size_t)s * SK;
    float* gout = scores + (g * J + q) * N + n0;
#pragma unroll 1
    for (int i = 0; i < kDecTilesPerWarp; i += KT) {
      const int tile0 = warp + i * kDecConsumers;
      if (tile0 * 16 >= cnt) break;
      int rr[KT][2];
      uint32_t w0[KT][W / 4], w1[KT][W / 4];
#pragma unroll
      for (int t2 = 0; t2 < KT; ++t2) {
        rr[t2][0] = (tile0 + t2 * kDecConsumers) * 16 + gq;
        rr[t2][1] = rr[t2][0] + 8;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          // rows past cnt (always < SK) read stale stage data; their results are never stored
          const uint32_t* src = sb + rr[t2][r] * W + q * (W / 4);
#pragma unroll
          for (int kk = 0; kk < W / 8; ++kk) {
            const uint2 v = *reinterpret_cast<const uint2*>(src + 2 * kk);
            (r ? w1 : w0)[t2][2 * kk] = v.x;
            (r ? w1 : w0)[t2][2 * kk + 1] = v.y;
          }
        }
      }
      int acc[KT][4][4];
#pragma unroll
      for (int p = 0; p < W / 8; ++p) {
#pragma unroll
        for (int sh = 0; sh < 2; ++sh) {
#pragma unroll
          for (int Ji = 0; Ji < 4; ++Ji) {
            const uint32_t M = 0x01010101u << (2 * Ji);
            const uint2 bb = breg[8 * p + 2 * Ji + sh];
#pragma unroll
            for (int t2 = 0; t2 < KT; ++t2) {
              const uint32_t a0 = (w0[t2][2 * p] >> sh) & M, a1 = (w1[t2][2 * p] >> sh) & M;
              const uint32_t a2 = (w0[t2][2 * p + 1] >> sh) & M, a3 = (w1[t2][2 * p + 1] >> sh) & M;
              if (p == 0 && sh == 0) mma_u8s8_zc(acc[t2][Ji], a0, a1, a2, a3, bb.x, bb.y);
              else mma_u8s8(acc[t2][Ji], a0, a1, a2, a3, bb.x, bb.y);
            }
          }
        }
      }
      if (q < J) {
#pragma unroll
        for (int t2 = 0; t2 < KT; ++t2) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int row = rr[t2][r];
            if (row >= cnt) continue;
            const int hi = ((acc[t2][0][2 * r] * 4 + acc[t2][1][2 * r]) * 4 + acc[t2][2][2 * r]) * 4 + acc[t2][3][2 * r];
            const int lo = ((acc[t2][0][2 * r + 1] * 4 + acc[t2][1][2 * r + 1]) * 4 + acc[t2][2][2 * r + 1]) * 4 +
                           acc[t2][3][2 * r + 1];
            // 32 * sum_i (2 b_i - 1) Q_i, exact in int32 (|.| <= 32 m 32639 < 2^31 for m <= 2048)
            const int Dq = hi * 256 + lo - qs32;
            const float nrm = nbulk ? sn[row] : __ldg(nsrc + row);
            gout[row] = mul * nrm * (float)Dq;
          }
        }
      }
    }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++c == cpg) { c = 0; ++g; }
    if (++s == NS) { s = 0; ph ^= 1u; }
  }
}

// Decode scores with shift-window digit sums (build_tables_dig): the A
// fragments are the sign words shifted right by s = 0..7, unmasked, so a
// 16-key tile costs 7 shifts per word and W MMAs per column tile of two
// queries. The stage ring and producer are those of scores_decode_kernel,
// with SKT keys per stage. With DUP (one query per group) both halves of the
// B tile carry the same digits, and lanes q = 2, 3 finish the odd tiles while
// lanes 0, 1 finish the even ones.

// Finishes KT tiles: lane (gq, q) holds digits (2 par, 2 par + 1) of rows gq and
// gq + 8. P_r is its part of sum b Q for row r, and the pair (q, q ^ 1)
// completes row par. CHECK guards rows past cnt and unaligned norms.
template <int NT, bool DUP, int KT, bool CHECK>
__device__ __forceinline__ void digit_epilogue(const int (&acc)[KT][NT][4], int tile0, int gq, int par, int half,
                                               int cnt, bool nbulk, const float* __restrict__ sn,
                                               const float* __restrict__ nsrc, const float (&mul)[NT],
                                               const uint32_t (&qs)[NT], int J, int64_t N,
                                               float* __restrict__ gout) {
  const uint32_t hm = par ? 65536u : 1u;  // lanes with odd q hold digits 2, 3
  if constexpr (DUP) {
#pragma unroll
    for (int k = 0; k < KT / 2; ++k) {
      int cc[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) cc[j] = half ? acc[2 * k + 1][0][j] : acc[2 * k][0][j];
      const uint32_t P0 = (uint32_t)cc[0] * hm + (uint32_t)cc[1] * (hm << 8);
      const uint32_t P1 = (uint32_t)cc[2] * hm + (uint32_t)cc[3] * (hm << 8);
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, par ? P0 : P1, 1);
      const uint32_t tot = (par ? P1 : P0) + recv;
      const int row = (tile0 + (2 * k + half) * kDecConsumers) * 16 + gq + 8 * par;
      if (!CHECK || row < cnt) {
        const float nrm = (!CHECK || nbulk) ? sn[row] : __ldg(nsrc + row);
        gout[row] = mul[0] * nrm * (float)(int)(2u * tot - qs[0]);
      }
    }
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int jq = 2 * nt + half;
#pragma unroll
      for (int t = 0; t < KT; ++t) {
        const uint32_t P0 = (uint32_t)acc[t][nt][0] * hm + (uint32_t)acc[t][nt][1] * (hm << 8);
        const uint32_t P1 = (uint32_t)acc[t][nt][2] * hm + (uint32_t)acc[t][nt][3] * (hm << 8);
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, par ? P0 : P1, 1);
        const uint32_t tot = (par ? P1 : P0) + recv;
        const int row = (tile0 + t * kDecConsumers) * 16 + gq + 8 * par;
        if (jq < J && (!CHECK || row < cnt)) {
          const float nrm = (!CHECK || nbulk) ? sn[row] : __ldg(nsrc + row);
          gout[jq * N + row] = mul[nt] * nrm * (float)(int)(2u * tot - qs[nt]);
        }
      }
    }
  }
}

// PAGED reads group g's tokens t < seq_lens[g] through the block table
// (PagedRead); N is then the bound max_len, and the row stride of scores.
//
// Shared memory: the per-query constants, the B fragments, NS stages of
// [SK keys x W words] bits and [SK] norms, one slot for a group's Sq rows
// ([J][m] fp32) and the barriers. The producer copies each new group's Sq
// rows into the slot with that group's first stage, once the consumers have
// signalled (slot_free) that the previous group's table is built; the table
// build then reuses the slot for its packed digits and the B fragments'
// space for the quantised Sq.
template <int W, int NT, bool DUP, int KT, int SKT, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, 2) scores_digit_kernel(
    const uint32_t* __restrict__ bits, const float* __restrict__ norms, const float* __restrict__ sq,
    int64_t G, int64_t N, int J, int NS, float est_scale, int64_t items_per_cta, float* __restrict__ scores,
    int* __restrict__ err, PagedRead pr) {
  using namespace qjl_sync;
  constexpr int SK = SKT;
  constexpr int m = 32 * W;
  constexpr int TPW = SK / 16 / kDecConsumers;  // tiles per consumer warp per stage
  static_assert(!DUP || NT == 1, "DUP is the one-query layout");
  static_assert(TPW % KT == 0 && (KT == 2 || KT == 4), "KT tiles per batch");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* s_mul = reinterpret_cast<float*>(smem_raw);
  int* s_qsum = reinterpret_cast<int*>(s_mul + 64);
  uint2* Btab = reinterpret_cast<uint2*>(s_qsum + 64);                       // [NT][W][32]
  uint32_t* sbits = reinterpret_cast<uint32_t*>(Btab + (size_t)NT * W * 32);  // [NS][SK * W]
  float* snorm = reinterpret_cast<float*>(sbits + (size_t)NS * SK * W);     // [NS][SK]
  float* ssq = snorm + (size_t)NS * SK;                                      // [J * m]
  uint64_t* full = reinterpret_cast<uint64_t*>(ssq + (size_t)J * m);
  uint64_t* empty = full + NS;
  uint64_t* slot_free = empty + NS;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t cpg = (N + SK - 1) / SK;
  const int64_t total = G * cpg;
  const int64_t i0 = (int64_t)blockIdx.x * items_per_cta;
  const int64_t i1 = min(total, i0 + items_per_cta);
  const uint32_t sq_bytes = (uint32_t)J * m * 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecConsumers);
    }
    mbar_init(slot_free, 1);
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kDecConsumers) {
    if (lane == 0) {
      int64_t g = i0 / cpg, c = i0 - (i0 / cpg) * cpg;
      int64_t prev_g = -1;
      uint32_t sph = 0;  // parity of the slot's next release
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t it = i0; it < i1; ++it, ++issued) {
        if (!mbar_wait(&empty[s], ph ^ 1u)) { atomicOr(err, 1); break; }
        const int64_t n0 = c * SK;
        // the first stage of each group this CTA visits also brings the group's Sq rows,
        // into the slot the previous group's table build has released
        const bool new_group = g != prev_g;
        prev_g = g;
        if (new_group) {
          if (!mbar_wait(slot_free, sph ^ 1u)) { atomicOr(err, 1); break; }
          sph ^= 1u;
        }
        const uint32_t tx_sq = new_group ? sq_bytes : 0u;
        if constexpr (PAGED) {
          // the stage's tokens [n0, n0 + cnt) of group g, one copy per page segment, each
          // rounded up to 4 tokens (16 bytes of norms; never past the page, which holds a
          // multiple of 16 tokens). An empty stage only arrives.
          const int64_t Lg = min64(max64(__ldg(pr.seq_lens + g), 0), N);
          const int cnt = (int)max64(0, min64(SK, Lg - n0));
          const int T = pr.page_tokens;
          uint32_t tx = tx_sq;
          for (int pass = 0; pass < 2; ++pass) {
            if (pass == 1) {
              mbar_expect_tx(&full[s], tx);
              if (new_group) bulk_g2s(ssq, sq + g * (int64_t)J * m, sq_bytes, &full[s]);
            }
            for (int64_t lo = n0; lo < n0 + cnt;) {
              const int64_t pi = lo / T;
              const int64_t hi = min64(n0 + cnt, (pi + 1) * T);
              const uint32_t len4 = (uint32_t)((hi - lo + 3) & ~3);
              const int pg = pi < pr.max_pages ? __ldg(pr.table + g * (int64_t)pr.max_pages + pi) : -1;
              if (pg >= 0 && (int64_t)pg < pr.num_pages) {
                const int64_t prow = (int64_t)pg * T + (lo - pi * T);
                if (pass == 0) {
                  tx += len4 * (W * 4 + 4);
                } else {
                  bulk_g2s(sbits + (size_t)s * SK * W + (lo - n0) * W, bits + prow * W, len4 * W * 4, &full[s]);
                  bulk_g2s(snorm + (size_t)s * SK + (lo - n0), norms + prow, len4 * 4, &full[s]);
                }
              } else if (pass == 0) {
                atomicOr(err, QJL_DEVERR_PAGE);  // a bad page id: its tokens keep stale stage data
              }
              lo = hi;
            }
          }
        } else {
          const int cnt = (int)(N - n0 < SK ? N - n0 : SK);
          const float* nsrc = norms + g * N + n0;
          const bool nbulk = (((uintptr_t)nsrc & 15u) == 0) && (cnt % 4 == 0);
          const uint32_t bbytes = (uint32_t)cnt * W * 4;
          mbar_expect_tx(&full[s], bbytes + (nbulk ? (uint32_t)cnt * 4 : 0u) + tx_sq);
          bulk_g2s(sbits + (size_t)s * SK * W, bits + (g * N + n0) * W, bbytes, &full[s]);
          if (nbulk) bulk_g2s(snorm + (size_t)s * SK, nsrc, (uint32_t)cnt * 4, &full[s]);
          if (new_group) bulk_g2s(ssq, sq + g * (int64_t)J * m, sq_bytes, &full[s]);
        }
        if (++c == cpg) { c = 0; ++g; }
        if (++s == NS) { s = 0; ph ^= 1u; }
      }
      const int used = issued < NS ? (int)issued : NS;
      for (int j = 0; j < used; ++j) {
        int st = s - 1 - j;
        uint32_t p = ph;
        if (st < 0) { st += NS; p ^= 1u; }
        if (!mbar_wait(&full[st], p)) atomicOr(err, 2);
      }
    }
    return;
  }

  const int gq = lane >> 2, q = lane & 3, par = q & 1, half = q >> 1;
  // Each CTA walks its contiguous range of (group, stage) items in order.
  // Stage bookkeeping is incremental and 32-bit where it can be: chunk c of
  // group g, with the norms and output pointers stepped per stage.
  int64_t g = i0 / cpg;
  int c = (int)(i0 - g * cpg);
  const int cpg32 = (int)cpg;
  const int last_cnt = (int)(N - (cpg - 1) * SK);
  const bool groups_aligned = ((((uintptr_t)norms) & 15u) == 0) && (N % 4 == 0);
  const float* nsrc = norms + g * N + (int64_t)c * SK;
  float* gout = scores + g * (int64_t)J * N + (int64_t)c * SK;
  int64_t cur_g = -1;
  int64_t Lg = N;  // valid tokens of the current group (PAGED)
  int s = 0;
  uint32_t ph = 0;
  uint2 breg[NT == 1 ? W : 1];
  float mul[NT];
  uint32_t qs[NT];
  bool dead = false;  // a timed-out wait: keep the loop's barriers, skip the work
  const int nitems = (int)(i1 - i0);
  for (int item = 0; item < nitems; ++item) {
    if (PAGED && g != cur_g) Lg = min64(max64(__ldg(pr.seq_lens + g), 0), N);
    const int cnt = PAGED ? (int)max64(0, min64(SK, Lg - (int64_t)c * SK))
                          : (c == cpg32 - 1 ? last_cnt : SK);
    if (!dead && !__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) { atomicOr(err, 4); dead = true; }
    if (g != cur_g) {
      // every consumer warp takes part (dead or not), so the named barriers stay matched
      named_sync(1, kDecConsumers * 32);
      // the slot's Sq rows become the digit scratch, Btab's space holds Q until phase 3
      build_tables_dig_smem<W>(ssq, J, NT, DUP, est_scale, s_mul, s_qsum, reinterpret_cast<int*>(Btab),
                               reinterpret_cast<uint32_t*>(ssq), Btab, kDecConsumers, 1);
      if (threadIdx.x == 0) mbar_arrive(slot_free);  // the build's last barrier: nobody reads the slot now
      if constexpr (NT == 1) {
#pragma unroll
        for (int mu = 0; mu < W; ++mu) breg[mu] = Btab[mu * 32 + lane];
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int jq = DUP ? 0 : 2 * nt + half;
        mul[nt] = jq < J ? s_mul[jq] : 0.f;
        qs[nt] = jq < J ? (uint32_t)s_qsum[jq] : 0u;
      }
      cur_g = g;
    }
    if (!dead) {
      // the producer bulk-copied the norms exactly when they were 16-byte aligned
      // and a multiple of 4; otherwise they are read from global memory
      const bool nbulk = PAGED || ((((uintptr_t)nsrc & 15u) == 0) && (cnt % 4 == 0));
      const bool whole = (PAGED || groups_aligned) && cnt == SK;
      const uint32_t* sb = sbits + (size_t)s * SK * W;
      const float* sn = snorm + (size_t)s * SK;
      // one batch of KT tiles from tile0: loads, shift-window MMAs, epilogue (CHECK: bounds and
      // norm source checks for a partial or unaligned stage)
      auto batch = [&](int tile0, auto check) {
        constexpr bool CHECK = decltype(check)::value;
        uint32_t w0[KT][W / 4], w1[KT][W / 4];
#pragma unroll
        for (int t = 0; t < KT; ++t) {
          // rows past cnt (always < SK) read stale stage data; their results are never stored
          const int r0 = (tile0 + t * kDecConsumers) * 16 + gq;
#pragma unroll
          for (int kk = 0; kk < W / 8; ++kk) {
            const uint2 a = *reinterpret_cast<const uint2*>(sb + r0 * W + q * (W / 4) + 2 * kk);
            const uint2 b = *reinterpret_cast<const uint2*>(sb + (r0 + 8) * W + q * (W / 4) + 2 * kk);
            w0[t][2 * kk] = a.x; w0[t][2 * kk + 1] = a.y;
            w1[t][2 * kk] = b.x; w1[t][2 * kk + 1] = b.y;
          }
        }
        int acc[KT][NT][4];
#pragma unroll
        for (int p = 0; p < W / 8; ++p) {
#pragma unroll
          for (int sh = 0; sh < 8; ++sh) {
            uint32_t x[KT][4];
#pragma unroll
            for (int t = 0; t < KT; ++t) {
              x[t][0] = w0[t][2 * p] >> sh;
              x[t][1] = w1[t][2 * p] >> sh;
              x[t][2] = w0[t][2 * p + 1] >> sh;
              x[t][3] = w1[t][2 * p + 1] >> sh;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint2 bb = NT == 1 ? breg[(8 * p + sh) % (NT == 1 ? W : 1)]
                                       : Btab[(nt * W + 8 * p + sh) * 32 + lane];
#pragma unroll
              for (int t = 0; t < KT; ++t) {
                if (p == 0 && sh == 0) mma_u8s8_zc(acc[t][nt], x[t][0], x[t][1], x[t][2], x[t][3], bb.x, bb.y);
                else mma_u8s8(acc[t][nt], x[t][0], x[t][1], x[t][2], x[t][3], bb.x, bb.y);
              }
            }
          }
        }
        digit_epilogue<NT, DUP, KT, CHECK>(acc, tile0, gq, par, half, cnt, nbulk, sn, nsrc, mul, qs, J, N, gout);
      };
      if (whole) {
        // a whole stage: at m = 256 the batches are unrolled, so one batch's epilogue can overlap the
        // next one's MMAs (-3 % time for one query per group, -10 % for two); at m = 512 the
        // registers would spill
        if constexpr (W == 8) {
#pragma unroll
          for (int i = 0; i < TPW; i += KT) batch(warp + i * kDecConsumers, std::false_type());
        } else {
#pragma unroll 1
          for (int i = 0; i < TPW; i += KT) batch(warp + i * kDecConsumers, std::false_type());
        }
      } else {
#pragma unroll 1
        for (int i = 0; i < TPW; i += KT) {
          const int tile0 = warp + i * kDecConsumers;
          if (tile0 * 16 >= cnt) break;
          batch(tile0, std::true_type());
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++c == cpg32) {
      c = 0;
      ++g;
      nsrc = norms + g * N;
      gout = scores + g * (int64_t)J * N;
    } else {
      nsrc += SK;
      gout += SK;
    }
    if (++s == NS) { s = 0; ph ^= 1u; }
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

template <int W>
qjl_status launch_decode_fast(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G,
                              int64_t N, const float* sq, int J, float* scores, cudaStream_t st) {
  const int NS = W == 8 ? 4 : 3;
  const size_t smem = 3 * 64 * 4 + (size_t)W * 32 * sizeof(uint2) + (size_t)NS * kDecStageKeys * (W + 1) * 4 +
                      (size_t)2 * NS * 8;
  static_assert(kDecTilesPerWarp % 4 == 0, "tiles are consumed in groups of 2 or 4");
  auto kern = scores_decode_kernel<W>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return qjl_check_launch("scores_decode_kernel smem attribute");
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return qjl_check_launch("scores_decode_kernel attributes");
  const int regs_per_cta = ((fa.numRegs * 32 + 255) / 256) * 256 * (kDecThreads / 32);
  const int per_sm = std::max(1, std::min(65536 / std::max(regs_per_cta, 1), (int)((228u * 1024u) / (smem + 1024))));
  int* err = qjl_error_flag(P->device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  const int64_t total = G * ((N + kDecStageKeys - 1) / kDecStageKeys);
  const int64_t slots = (int64_t)qjl_num_sms(P->device) * per_sm;
  const int64_t grid = std::min<int64_t>(total, slots);
  const int64_t ipc = (total + grid - 1) / grid;
  const int64_t nblk = (total + ipc - 1) / ipc;
  qjl_log_launch("scores_decode_kernel", nblk, kDecThreads, smem, per_sm);
  kern<<<(unsigned)nblk, kDecThreads, smem, st>>>(bits, norms, sq, G, N, J, NS, P->est_scale, ipc, scores, err);
  return qjl_check_launch("scores_decode_kernel");
}

template <int W, int NT, bool DUP, int KT, int SKT, bool PAGED = false>
qjl_status launch_digit(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G, int64_t N,
                        const float* sq, int J, float* scores, cudaStream_t st, const PagedRead& pr = PagedRead()) {
  // ring depth: as many stages as keep two CTAs per SM within shared memory
  const size_t stage = (size_t)SKT * (W + 1) * 4;  // bits and norms
  const int NS = stage * 4 <= 80 * 1024 ? 4 : (stage * 3 <= 110 * 1024 ? 3 : 2);
  const size_t smem = 2 * 64 * 4 + (size_t)NT * W * 32 * sizeof(uint2) + (size_t)NS * stage +
                      (size_t)J * 32 * W * 4 + (size_t)(2 * NS + 1) * 8;
  static_assert((size_t)NT * W * 32 * sizeof(uint2) >= (size_t)2 * 32 * W * 4, "Q scratch fits in Btab (J <= 2)");
  auto kern = scores_digit_kernel<W, NT, DUP, KT, SKT, PAGED>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return qjl_check_launch("scores_digit_kernel smem attribute");
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, smem) != cudaSuccess || per_sm < 1)
    return qjl_check_launch("scores_digit_kernel occupancy");
  int* err = qjl_error_flag(P->device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  const int64_t total = G * ((N + SKT - 1) / SKT);
  const int64_t slots = (int64_t)qjl_num_sms(P->device) * per_sm;
  const int64_t grid = std::min<int64_t>(total, slots);
  const int64_t ipc = (total + grid - 1) / grid;
  const int64_t nblk = (total + ipc - 1) / ipc;
  qjl_log_launch("scores_digit_kernel", nblk, kDecThreads, smem, per_sm);
  kern<<<(unsigned)nblk, kDecThreads, smem, st>>>(bits, norms, sq, G, N, J, NS, P->est_scale, ipc, scores, err, pr);
  return qjl_check_launch("scores_digit_kernel");
}

// One or two queries per group: 1024-key stages; four tiles per batch at
// m = 256, two at m = 512 (registers).
template <int W, bool PAGED = false>
qjl_status launch_digit_w(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G, int64_t N,
                          const float* sq, int J, float* scores, cudaStream_t st, const PagedRead& pr = PagedRead()) {
  constexpr int KT = W == 8 ? 4 : 2;
  return J == 1 ? launch_digit<W, 1, true, KT, 1024, PAGED>(P, bits, norms, G, N, sq, J, scores, st, pr)
                : launch_digit<W, 1, false, KT, 1024, PAGED>(P, bits, norms, G, N, sq, J, scores, st, pr);
}

}  // namespace

qjl_status launch_scores(const qjl_projection* P, const uint32_t* bits, const float* norms,
                         int64_t G, int64_t N, const float* sq, int J, float* scores, cudaStream_t st) {
  // At m = 256 or 512, one or two queries per group take the shift-window
  // digit kernel and three or four the class kernel (half the MMAs of two
  // digit column tiles). More queries, or m = 1024, are a contraction for the
  // tcgen05 kernel (scores_many.cu). Other m, and one group of more than 2^31
  // keys, take the SIMT kernel.
  if (J <= 2 && (P->m == 256 || P->m == 512))
    return P->m == 256 ? launch_digit_w<8>(P, bits, norms, G, N, sq, J, scores, st)
                       : launch_digit_w<16>(P, bits, norms, G, N, sq, J, scores, st);
  if (J <= 4 && (P->m == 256 || P->m == 512))
    return P->m == 256 ? launch_decode_fast<8>(P, bits, norms, G, N, sq, J, scores, st)
                       : launch_decode_fast<16>(P, bits, norms, G, N, sq, J, scores, st);
  if (scores_many_supported(P->m, N)) return launch_scores_many(P, bits, norms, G, N, sq, J, scores, st);
  const int64_t want = (G * N + 7) / 8;
  const int blocks = (int)std::min<int64_t>(want, (int64_t)qjl_num_sms(P->device) * 16);
  scores_simt_kernel<<<blocks, 256, 0, st>>>(bits, norms, sq, G, N, J, P->m / 32, P->est_scale, scores);
  return qjl_check_launch("scores_simt_kernel");
}

qjl_status launch_scores_paged(const qjl_projection* P, const uint32_t* bits_pool, const float* norms_pool,
                               const PagedRead& pr, int64_t G, int64_t max_len, const float* sq, int J,
                               float* scores, cudaStream_t st) {
  if (J > 2 || (P->m != 256 && P->m != 512))
    return qjl_set_error(QJL_ERR_UNSUPPORTED, "paged scores support q_per_group <= 2 and m in {256, 512}");
  return P->m == 256 ? launch_digit_w<8, true>(P, bits_pool, norms_pool, G, max_len, sq, J, scores, st, pr)
                     : launch_digit_w<16, true>(P, bits_pool, norms_pool, G, max_len, sq, J, scores, st, pr);
}
