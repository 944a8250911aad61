// QJL estimator on the 5th-generation tensor cores (tcgen05 kind::i8).
//
// QJL abstract ("Majid Daliri" page): est = c alpha ||k|| sum_i (2 b_i - 1) Sq_i.
// A decode step reads the whole cache once (KIVI abstract), so this kernel
// has under two SM clocks per 40-byte key. With legacy mma.sync fragments
// each key costs about 350 lane-instructions. Here each key costs about 100:
//
//   * one consumer thread owns one key (one TMEM lane). It reads the key's
//     W sign words from a shared-memory stage and expands each word into
//     8 u8 registers (w >> s) & (0x01010101 << 2J), s in {0,1},
//     J in {0..3}. Byte e of a register is bit 8e+2J+s, worth 4^J. That is
//     one AND per 4 bits. tcgen05.st moves them to TMEM as the A operand
//     (128 keys x 32 W bytes);
//   * Sq is rounded per (group, query) to 16-bit fixed point,
//     Q = rint(Sq * 32639 / max|Sq|) = 256 hi + lo with int8 halves. The B
//     table (one 32-byte K slice per word, in shared memory) has one column
//     per (query, weight class J, half). A byte of class J meets only that
//     class's columns, so the four power-of-4 weights never mix;
//   * one elected lane issues W MMAs (M=128, K=32, N=8 per query) with D in
//     TMEM (s32, exact). The consumers read D back (one tcgen05.ld per key),
//     form 64 sum b Q with three multiply-adds per half, and write one fp32
//     score per key: coalesced along N.
// The sign sums are exact. The only error is the 16-bit rounding of Sq:
// at most m max|Sq| / 65278 before scaling.
//
// Warps: 0-3 consumers (TMEM lane quarters), 4 bulk-copy producer (one lane),
// 5 TMEM allocator and MMA issuer (one lane). Persistent CTAs each take a
// contiguous, g-major range of (group, 128-key tile) items. A and D are
// triple-buffered in TMEM, so the epilogue of tile i-2 overlaps the MMAs of
// tiles i-1 and i. B tables are double-buffered by group. Every wait is bounded.

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "mbarrier.cuh"
#include "qjl_internal.h"

namespace {

using namespace qjl_sync;

constexpr int kTileKeys = 128;
constexpr int kThreads = 192;
constexpr int kQmax = 32639;  // 127 * 256 + 127: both int8 halves stay in range

__host__ __device__ constexpr int ncol_for(int JT) { return JT == 1 ? 8 : (JT == 2 ? 16 : 32); }
constexpr int kNB = 3;   // TMEM buffers for A and D: the epilogue lags the MMAs by two tiles
__host__ __device__ constexpr int dstride_for(int JT) { return ncol_for(JT) < 16 ? 16 : ncol_for(JT); }
__host__ __device__ constexpr int tmem_cols_for(int W, int JT) {
  // kNB A buffers of 8W columns + kNB D buffers, rounded up to a power of two
  return (kNB * 8 * W + kNB * dstride_for(JT)) <= 256 ? 256 : 512;
}

// Instruction descriptor, kind::i8: A u8 (K-major, from TMEM), B s8 (K-major), D s32, M=128.
__host__ __device__ constexpr uint32_t idesc_i8(int N) {
  return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// No-swizzle K-major descriptor: 8-row x 16-byte core matrices, K-chunks 128 B
// apart (LBO), 8-row groups 256 B apart (SBO).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) {
  uint64_t desc = (uint64_t)((saddr >> 4) & 0x3FFFu);
  desc |= (uint64_t)(128u >> 4) << 16;
  desc |= (uint64_t)(256u >> 4) << 32;
  desc |= (uint64_t)1u << 46;
  return desc;
}

// Byte offset of B element (column n, k) inside one word's K slice.
__device__ __forceinline__ int bofs(int n, int k) {
  return (n >> 3) * 256 + (k >> 4) * 128 + (n & 7) * 16 + (k & 15);
}

__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

template <int NC>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[NC]);

template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ int quant16(float v, float inv) {
  const float q = rintf(v * inv);
  return (int)fminf(fmaxf(q, (float)-kQmax), (float)kQmax);
}

// B table and per-query constants for group g (run by the 128 consumer threads).
template <int W, int JT>
__device__ void build_group(const float* __restrict__ sqg, int J, float est_scale, unsigned char* tab,
                            float* s_inv, float* s_mul, float* s_qs) {
  constexpr int m = 32 * W;
  constexpr int NC = ncol_for(JT);
  constexpr int SLICE = NC * 32;  // bytes per word's B slice
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (warp < J) {
    const float* row = sqg + (int64_t)warp * m;
    float mx = 0.f;
    for (int i = lane; i < m; i += 32) mx = fmaxf(mx, fabsf(row[i]));
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float inv = mx > 0.f ? (float)kQmax / mx : 0.f;
    int qs = 0;
    for (int i = lane; i < m; i += 32) qs += quant16(row[i], inv);
#pragma unroll
    for (int o = 16; o; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
    if (lane == 0) {
      s_inv[warp] = inv;
      s_mul[warp] = est_scale * (mx > 0.f ? mx / (float)kQmax : 0.f) * 0.015625f;  // the D sums carry 64x
      s_qs[warp] = 64.f * (float)qs;
    }
  }
  named_sync(1, 128);
  // one 32-bit word of B per (word t, column n, 4 consecutive k): W * NC * 8 entries
  const int entries = W * NC * 8;
  for (int idx = tid; idx < entries; idx += 128) {
    const int t = idx / (NC * 8);
    const int rem = idx - t * (NC * 8);
    const int n = rem >> 3, ri = rem & 7;  // k = 4 ri .. 4 ri + 3
    const int jq = n >> 3, Jc = (n >> 1) & 3, half = n & 1;
    const int Ji = ri >> 1, s = ri & 1;
    uint32_t v = 0;
    if (jq < J && Jc == Ji) {
      const float* row = sqg + (int64_t)jq * m;
      const float inv = s_inv[jq];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int Q = quant16(row[32 * t + 8 * e + 2 * Ji + s], inv);
        const int lo = (int)(int8_t)(Q & 0xFF);
        const int hi = (Q - lo) >> 8;
        v |= ((uint32_t)(half ? lo : hi) & 0xFFu) << (8 * e);
      }
    }
    *reinterpret_cast<uint32_t*>(tab + t * SLICE + bofs(n, 4 * ri)) = v;
  }
  // the MMA reads the table through the async proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  named_sync(1, 128);
}

template <int W, int JT>
__global__ void __launch_bounds__(kThreads, 1) scores_tc_kernel(
    const uint32_t* __restrict__ bits, const float* __restrict__ norms, const float* __restrict__ sq, int64_t G,
    int64_t N, int J, int NS, float est_scale, int64_t items_per_cta, float* __restrict__ scores,
    int* __restrict__ err) {
  constexpr int NC = ncol_for(JT);
  constexpr int SLICE = NC * 32;
  constexpr int TAB = W * SLICE;
  constexpr int ACOLS = 8 * W;
  constexpr int TCOLS = tmem_cols_for(W, JT);
  constexpr int DS = dstride_for(JT);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* tabs = smem_raw;                                         // 2 x TAB
  float* s_inv = reinterpret_cast<float*>(tabs + 2 * TAB);               // 2 x 4
  float* s_mul = s_inv + 8;
  float* s_qs = s_mul + 8;
  uint32_t* sbits = reinterpret_cast<uint32_t*>(s_qs + 8);               // NS x 128 x W
  float* snorm = reinterpret_cast<float*>(sbits + (size_t)NS * kTileKeys * W);  // NS x 128
  uint64_t* full = reinterpret_cast<uint64_t*>(snorm + (size_t)NS * kTileKeys);
  uint64_t* empty = full + NS;
  uint64_t* afull = empty + NS;     // kNB
  uint64_t* dfull = afull + kNB;    // kNB
  uint64_t* dempty = dfull + kNB;   // kNB
  uint64_t* dbar = dempty + kNB;    // 1
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tpg = (N + kTileKeys - 1) / kTileKeys;
  const int64_t total = G * tpg;
  const int64_t i0 = (int64_t)blockIdx.x * items_per_cta;
  const int64_t i1 = min(total, i0 + items_per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    for (int b = 0; b < kNB; ++b) {
      mbar_init(&afull[b], 4);
      mbar_init(&dfull[b], 1);
      mbar_init(&dempty[b], 4);
    }
    mbar_init(dbar, 1);
    mbar_fence_init();
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(TCOLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t a_col0 = 0, d_col0 = kNB * ACOLS;

  if (warp == 4) {
    // ---------------- producer: bits and norms of one 128-key tile per stage
    if (lane == 0) {
      int64_t g = i0 / tpg, c = i0 - (i0 / tpg) * tpg;
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t it = i0; it < i1; ++it, ++issued) {
        if (!mbar_wait(&empty[s], ph ^ 1u)) { atomicOr(err, 1); break; }
        const int64_t n0 = c * kTileKeys;
        const int cnt = (int)(N - n0 < kTileKeys ? N - n0 : kTileKeys);
        const float* nsrc = norms + g * N + n0;
        const bool nbulk = (((uintptr_t)nsrc & 15u) == 0) && (cnt % 4 == 0);
        const uint32_t bbytes = (uint32_t)cnt * W * 4;
        mbar_expect_tx(&full[s], bbytes + (nbulk ? (uint32_t)cnt * 4 : 0u));
        bulk_g2s(sbits + (size_t)s * kTileKeys * W, bits + (g * N + n0) * W, bbytes, &full[s]);
        if (nbulk) bulk_g2s(snorm + (size_t)s * kTileKeys, nsrc, (uint32_t)cnt * 4, &full[s]);
        if (++c == tpg) { c = 0; ++g; }
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
  } else if (warp == 5) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int64_t g = i0 / tpg, c = i0 - (i0 / tpg) * tpg;
      int64_t cur_g = g;
      int tb = 0;  // table buffer of the current group
      int buf = 0;
      uint32_t par = 0;
      const uint32_t idesc = idesc_i8(NC);
      for (int64_t it = i0; it < i1; ++it) {
        if (g != cur_g) { cur_g = g; tb ^= 1; }
        if (!mbar_wait(&afull[buf], par)) { atomicOr(err, 4); break; }
        if (!mbar_wait(&dempty[buf], par ^ 1u)) { atomicOr(err, 4); break; }
        tc_fence_after();
        const uint32_t a_tm = tmem_base + a_col0 + (uint32_t)(buf * ACOLS);
        const uint32_t d_tm = tmem_base + d_col0 + (uint32_t)(buf * DS);
        const uint32_t tab = smem_u32(tabs + tb * TAB);
#pragma unroll
        for (int t = 0; t < W; ++t)
          mma_i8_ts(d_tm, a_tm + (uint32_t)(8 * t), kmajor_desc(tab + (uint32_t)(t * SLICE)), idesc, t > 0 ? 1u : 0u);
        mma_commit(&dfull[buf]);
        if (++c == tpg) { c = 0; ++g; }
        if (++buf == kNB) { buf = 0; par ^= 1u; }
      }
      mma_commit(dbar);
      if (!mbar_wait(dbar, 0)) atomicOr(err, 8);
    }
  } else {
    // ---------------- consumers: thread r owns key r of each tile (TMEM lane r)
    const int r = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    int64_t g = i0 / tpg, c = i0 - (i0 / tpg) * tpg;
    int64_t cur_g = -1;
    int tb = 1;
    int s = 0;
    uint32_t ph = 0;
    int ab = 0;          // TMEM buffer of the tile being expanded
    uint32_t apar = 0;   // its phase parity
    bool ok = true;
    // up to kNB - 1 tiles whose MMAs are in flight and whose epilogue is pending (FIFO)
    struct Pend {
      int64_t out;
      float norm;
      int valid, tb, buf;
      uint32_t par;
    };
    Pend p0{}, p1{};
    int npend = 0;

    auto epilogue = [&](const Pend& p) {
      if (!__all_sync(0xffffffffu, mbar_wait(&dfull[p.buf], p.par))) { atomicOr(err, 16); ok = false; return; }
      tc_fence_after();
      uint32_t dv[NC];
      tmem_ld<NC>(tmem_base + lane_off + d_col0 + (uint32_t)(p.buf * DS), dv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[p.buf]);
      if (p.valid) {
#pragma unroll
        for (int jq = 0; jq < JT; ++jq) {
          if (jq >= J) break;
          int hl[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int* dd = reinterpret_cast<const int*>(dv) + 8 * jq + h;
            hl[h] = ((dd[0] * 4 + dd[2]) * 4 + dd[4]) * 4 + dd[6];  // 64 * sum b (hi or lo)
          }
          const float D = fmaf((float)hl[0], 512.f, 2.f * (float)hl[1]) - s_qs[p.tb * 4 + jq];
          scores[p.out + (int64_t)jq * N] = s_mul[p.tb * 4 + jq] * p.norm * D;
        }
      }
    };
    auto drain = [&]() {
      if (npend > 0 && ok) epilogue(p0);
      if (npend > 1 && ok) epilogue(p1);
      npend = 0;
    };

    for (int64_t it = i0; it < i1 && ok; ++it) {
      const int64_t n0 = c * kTileKeys;
      const int cnt = (int)(N - n0 < kTileKeys ? N - n0 : kTileKeys);
      if (g != cur_g) {
        // a new group: the pending tiles' MMAs read the table buffer and the
        // constants that may now be rebuilt, so finish them first
        drain();
        if (!ok) break;
        tb ^= 1;
        build_group<W, JT>(sq + g * (int64_t)J * (32 * W), J, est_scale, tabs + tb * TAB, s_inv + 4 * tb,
                           s_mul + 4 * tb, s_qs + 4 * tb);
        cur_g = g;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) { atomicOr(err, 32); break; }
      const uint32_t* sb = sbits + (size_t)s * kTileKeys * W + (size_t)r * W;
      uint32_t words[W];
#pragma unroll
      for (int k = 0; k < W; k += 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(sb + k);
        words[k] = v.x; words[k + 1] = v.y; words[k + 2] = v.z; words[k + 3] = v.w;
      }
      const float* nsrc = norms + g * N + n0;
      const bool nbulk = (((uintptr_t)nsrc & 15u) == 0) && (cnt % 4 == 0);
      const float nrm = r < cnt ? (nbulk ? snorm[(size_t)s * kTileKeys + r] : __ldg(nsrc + r)) : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == NS) { s = 0; ph ^= 1u; }
      // expand into A[ab]: its last reader, the MMA of the tile kNB earlier,
      // completed before that tile's epilogue returned
      const uint32_t a_addr = tmem_base + lane_off + a_col0 + (uint32_t)(ab * ACOLS);
#pragma unroll
      for (int t = 0; t < W; ++t) {
        const uint32_t w0 = words[t], w1 = words[t] >> 1;
        uint32_t a[8];
#pragma unroll
        for (int Ji = 0; Ji < 4; ++Ji) {
          const uint32_t M = 0x01010101u << (2 * Ji);
          a[2 * Ji] = w0 & M;
          a[2 * Ji + 1] = w1 & M;
        }
        tmem_st8(a_addr + (uint32_t)(8 * t), a);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[ab]);
      const Pend cur{(g * J) * N + n0 + r, nrm, r < cnt ? 1 : 0, tb, ab, apar};
      if (++ab == kNB) { ab = 0; apar ^= 1u; }
      // the oldest pending tile's epilogue overlaps the newer tiles' MMAs
      if (npend == kNB - 1) {
        epilogue(p0);
        p0 = p1;
        p1 = cur;
      } else if (npend == 0) {
        p0 = cur;
        ++npend;
      } else {
        p1 = cur;
        ++npend;
      }
      if (++c == tpg) { c = 0; ++g; }
    }
    if (ok) drain();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TCOLS));
}

size_t tc_smem(int W, int JT, int NS) {
  const int NC = ncol_for(JT);
  return 2 * (size_t)W * NC * 32 + 24 * 4 + (size_t)NS * kTileKeys * (W + 1) * 4 + (size_t)(2 * NS + 3 * kNB + 1) * 8 +
         16;
}

template <int W, int JT>
qjl_status launch_tc(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G, int64_t N,
                     const float* sq, int J, float* scores, cudaStream_t st) {
  const int NS = W == 8 ? 8 : 6;
  const size_t smem = tc_smem(W, JT, NS);
  auto kern = scores_tc_kernel<W, JT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return qjl_check_launch("scores_tc_kernel smem attribute");
  // CTAs per SM from registers, shared memory and TMEM (512 columns per SM)
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return qjl_check_launch("scores_tc_kernel attributes");
  const int regs_per_cta = ((fa.numRegs * 32 + 255) / 256) * 256 * (kThreads / 32);
  int per_sm = std::min({65536 / std::max(regs_per_cta, 1), (int)((228u * 1024u) / (smem + 1024)),
                         512 / tmem_cols_for(W, JT)});
  per_sm = std::max(per_sm, 1);
  int api = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&api, kern, kThreads, smem);
  cudaGetLastError();
  qjl_log_launch("scores_tc_kernel (occupancy api)", api, kThreads, smem, per_sm);
  int* err = qjl_error_flag(P->device);
  if (!err) return qjl_set_error(QJL_ERR_OOM, "cannot allocate the kernel error flag");
  const int64_t total = G * ((N + kTileKeys - 1) / kTileKeys);
  const int64_t slots = (int64_t)qjl_num_sms(P->device) * per_sm;
  const int64_t grid = std::min<int64_t>(total, slots);
  const int64_t ipc = (total + grid - 1) / grid;
  const int64_t nblk = (total + ipc - 1) / ipc;
  qjl_log_launch("scores_tc_kernel", nblk, kThreads, smem, per_sm);
  kern<<<(unsigned)nblk, kThreads, smem, st>>>(bits, norms, sq, G, N, J, NS, P->est_scale, ipc, scores, err);
  return qjl_check_launch("scores_tc_kernel");
}

}  // namespace

bool scores_tc_supported(int m, int J) { return (m == 256 || m == 512) && J >= 1 && J <= 4; }

qjl_status launch_scores_tc(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G, int64_t N,
                            const float* sq, int J, float* scores, cudaStream_t st) {
  if (P->m == 256) {
    switch (J) {
      case 1: return launch_tc<8, 1>(P, bits, norms, G, N, sq, J, scores, st);
      case 2: return launch_tc<8, 2>(P, bits, norms, G, N, sq, J, scores, st);
      default: return launch_tc<8, 4>(P, bits, norms, G, N, sq, J, scores, st);
    }
  }
  switch (J) {
    case 1: return launch_tc<16, 1>(P, bits, norms, G, N, sq, J, scores, st);
    case 2: return launch_tc<16, 2>(P, bits, norms, G, N, sq, J, scores, st);
    default: return launch_tc<16, 4>(P, bits, norms, G, N, sq, J, scores, st);
  }
}
