// Many-query QJL scores on the 5th-generation tensor cores (tcgen05 kind::i8).
//
// With many queries per key group ("Fast Quantized Johnson - Lindenstrauss
// Transforms", "Key concepts": bulk scoring of sketched keys against a batch
// of queries) the estimator est = c * alpha * ||k|| * sum_i (2 b_i - 1) Sq_i
// is a true contraction: [keys x m] sign bits times [m x J] projected
// queries. It runs as an integer MMA into TMEM:
//
//   * B (shared memory, s8): each query's Sq rounded to 16-bit fixed point,
//     Q = rint(Sq * 32639 / max|Sq|), split exactly as Q = 256 hi + lo with
//     int8 hi and lo. Columns [0, JP) hold hi and [JP, 2 JP) lo, so one MMA of
//     N = 2 JP columns serves JP queries.
//   * A (TMEM, u8): the sign bits as bytes 0 or 1. A key's word w becomes
//     eight 32-bit A columns a_s = (w >> s) & 0x01010101, s = 0..7, so column
//     s carries bits s, s + 8, s + 16, s + 24 in its four bytes. B uses the same
//     order along K: K position 4 s + e of word w holds the digit of bit
//     8 e + s. The order of a sum does not matter, so D = sum_i b_i digit_i.
//   * D (TMEM, s32, exact): sum b Q = 256 D_hi + D_lo, and the estimate is
//     mul * ||k|| * (2 sum b Q - sum Q), mul = c alpha max|Sq| / 32639. The
//     16-bit rounding of Sq is the only error, as in the class tables of the
//     decode score kernel: at most m max|Sq| / 65278 before scaling.
//
// A lives in TMEM rather than shared memory: expanding m bits into m bytes
// per key and reading them back through shared memory would take more
// shared-memory bandwidth than the MMAs leave. Persistent kernel, one CTA
// per SM, 22 warps:
//   warp 0      bulk-copy producer: each 128-key tile's sign words into a
//               ring of shared-memory stages.
//   warp 1      allocates TMEM (two D buffers of 128 columns, then A
//               buffers); one lane issues M = 128, N = 2 JP, K = 32 MMAs, one
//               per sign word, and commits their completion to mbarriers.
//   warps 2-5   expanders: thread r of lane quarter r / 32 owns key row r; it
//               turns its words into A columns with tcgen05.st, KC words per
//               A buffer.
//   warps 6-21  epilogue: four warps per lane quarter, each a quarter of the
//               queries; tcgen05.ld of D, the estimate (pairs of queries in
//               packed f32x2 arithmetic), coalesced stores of
//               scores[g][j][n]. They also build each group's B table: a
//               group's table goes into a buffer once the last tile that read
//               that buffer has left the epilogue (so its MMAs are complete).
// The producer loads each tile with a 2-D TMA copy whose swizzle matches the
// row width (32, 64 or 128 bytes), so that the expanders' per-row 16-byte
// reads, at an XOR-ed address, hit distinct banks.
// Every wait is bounded; on expiry a role records an error bit and stops,
// the MMA issuer drains what it issued, and TMEM is freed.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <type_traits>

#include "cache_hint.cuh"
#include "mbarrier.cuh"
#include "qjl_internal.h"
#include "tcgen05.cuh"

namespace {

using namespace qjl_sync;

constexpr int kTile = 128;             // keys per MMA tile (M)
constexpr int kExpWarps = 4;
constexpr int kEpiWarps = 16;
constexpr int kThreads = (2 + kExpWarps + kEpiWarps) * 32;
constexpr int kTmemCols = 512;
constexpr int kDStride = 128;          // columns per D buffer
constexpr int kAcol0 = 2 * kDStride;   // first A column
constexpr int kQmax = 32639;           // 127 * 256 + 127: both int8 digits stay in range

// Words per A buffer (8 TMEM columns per word) and the number of A buffers.
__host__ __device__ constexpr int kc_words(int W) { return W < 16 ? W : 16; }
__host__ __device__ constexpr int n_abuf(int W) { return (kTmemCols - kAcol0) / (8 * kc_words(W)); }

struct ManyParams {
  const uint32_t* bits;
  const float* norms;
  const float* sq;
  float* scores;
  int* err;
  int64_t G, N, items_per_cta;
  int J, NS, ntab;
  float est_scale;
};

// Table of one group into `tab` (2 JP rows x m bytes, K-major slices of 32
// bytes per sign word) and its per-query constants. Run by the epilogue
// warps (kEpiWarps * 32 threads, named barrier 1). A warp takes whole query
// rows: lane l holds coordinate 32 k + l of the row for every word k, loaded
// at once, so one pass finds max |Sq| and a second quantises and writes the
// two digit bytes of each coordinate to its K position (4 s + e for bit
// 8 e + s of the word). Rows j >= J are zero.
template <int W, int JP>
__device__ void build_table(const float* __restrict__ sqg, int J, float est_scale, unsigned char* tab,
                            float2* s_cst, int tid) {
  constexpr int m = 32 * W;
  constexpr int nthr = kEpiWarps * 32;
  constexpr int N = 2 * JP;
  const int lane = tid & 31, wq = tid >> 5;
  const int kpos = 4 * (lane & 7) + (lane >> 3);  // K position of bit `lane` within its word's slice
  // every epilogue warp is done with the buffer's previous constants
  named_sync(1, nthr);
  for (int j = wq; j < JP; j += kEpiWarps) {
    float v[W];
#pragma unroll
    for (int k = 0; k < W; ++k) v[k] = j < J ? __ldg(sqg + (int64_t)j * m + 32 * k + lane) : 0.f;
    float mx = 0.f;
#pragma unroll
    for (int k = 0; k < W; ++k) mx = fmaxf(mx, fabsf(v[k]));
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float inv = mx > 0.f ? (float)kQmax / mx : 0.f;
    int qs = 0;
    unsigned char* hi_row = tab + qjl_tc::kmajor_ofs(j, kpos);
    unsigned char* lo_row = tab + qjl_tc::kmajor_ofs(JP + j, kpos);
#pragma unroll
    for (int k = 0; k < W; ++k) {
      const int Q = (int)fminf(fmaxf(rintf(v[k] * inv), (float)-kQmax), (float)kQmax);
      qs += Q;
      const int l = (int)(int8_t)(Q & 0xFF);
      hi_row[k * N * 32] = (unsigned char)((Q - l) >> 8);
      lo_row[k * N * 32] = (unsigned char)l;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
    if (lane == 0) {
      // the estimate is c1 * (sum b Q) + c0, times ||k||
      const float mul = est_scale * (mx > 0.f ? mx / (float)kQmax : 0.f);
      s_cst[j] = make_float2(2.f * mul, -mul * (float)qs);
    }
  }
  // the MMAs read the table through the async proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  named_sync(1, nthr);
}

// TMEM loads of NC consecutive columns (NC = 2, 4, 8, 16 or 32) of this thread's lane, no wait.
template <int NC>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t* r) {
  if constexpr (NC == 32) {
    qjl_tc::ld32(taddr, r);
  } else if constexpr (NC == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else if constexpr (NC == 8) {
    qjl_tc::ld8(taddr, r);
  } else if constexpr (NC == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else {
    static_assert(NC == 2, "2, 4, 8, 16 or 32 columns");
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Byte offset of 16-byte piece k of row r in a stage written by the swizzled
// TMA copy: rows of W words (32, 64 or 128 bytes, the swizzle span), piece
// bits [4, 7) XOR-ed with address bits [7, 10) as far as the span allows.
template <int W>
__device__ __forceinline__ uint32_t swz_ofs(int r, int k) {
  constexpr uint32_t M = W == 32 ? 7u : (W == 16 ? 3u : 1u);
  const uint32_t off = (uint32_t)(r * W * 4 + 16 * k);
  return off ^ (((off >> 7) & M) << 4);
}

template <int W, int JP>
__global__ void __launch_bounds__(kThreads, 1) scores_many_kernel(const __grid_constant__ CUtensorMap tmB,
                                                                  const ManyParams P) {
  constexpr int m = 32 * W;
  constexpr int NCOL = 2 * JP;            // MMA N: hi digits, then lo digits
  constexpr int KC = kc_words(W);         // sign words per A buffer
  constexpr int NCH = W / KC;             // A buffers per tile
  constexpr int NA = n_abuf(W);
  constexpr int ND = 2;  // D buffers
  constexpr int JH = JP / (kEpiWarps / 4);  // queries per epilogue warp (even)
  static_assert(JH % 2 == 0, "query pairs");
  constexpr uint32_t TAB = (uint32_t)NCOL * 32 * W;
  constexpr uint32_t STAGE = (uint32_t)kTile * W * 4;
  static_assert(W % KC == 0 && NA >= 2, "A buffers");
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  // 1024-byte alignment for the swizzled stages
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_dyn + 1023) & ~(uintptr_t)1023);
  unsigned char* sbits = base;                                                // [NS] stages
  unsigned char* tabs = sbits + (size_t)P.NS * STAGE;                         // [ntab] tables
  float2* s_cst = reinterpret_cast<float2*>(tabs + (size_t)P.ntab * TAB);   // [2][64] per-query (c1, c0)
  uint64_t* full = reinterpret_cast<uint64_t*>(s_cst + 128);
  uint64_t* empty = full + P.NS;
  uint64_t* afull = empty + P.NS;    // [NA]
  uint64_t* aempty = afull + NA;     // [NA]
  uint64_t* dfull = aempty + NA;     // [ND]
  uint64_t* dempty = dfull + ND;     // [ND]
  uint64_t* tfull = dempty + ND;     // [2]
  uint64_t* dbar = tfull + 2;        // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NS = P.NS, ntab = P.ntab;
  const int64_t N = P.N;
  const int64_t tpg = (N + kTile - 1) / kTile;
  const int64_t total = P.G * tpg;
  const int64_t i0 = (int64_t)blockIdx.x * P.items_per_cta;
  const int64_t i1 = min(total, i0 + P.items_per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kExpWarps);
    }
    for (int a = 0; a < NA; ++a) {
      mbar_init(&afull[a], kExpWarps);
      mbar_init(&aempty[a], 1);
    }
    for (int b = 0; b < ND; ++b) {
      mbar_init(&dfull[b], 1);
      mbar_init(&dempty[b], kEpiWarps);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&tfull[b], 1);
    mbar_init(dbar, 1);
    mbar_fence_init();
  }
  if (warp == 1) qjl_tc::alloc(tmem_holder, kTmemCols);
  qjl_tc::fence_before();
  __syncthreads();
  qjl_tc::fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ---------------- producer: one 128-row box of sign words per stage (rows past the
    // group's end belong to the next group or are zero-filled; their results are not stored)
    if (lane == 0) {
      int64_t g = i0 / tpg, c = i0 - (i0 / tpg) * tpg;
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t it = i0; it < i1; ++it, ++issued) {
        if (!mbar_wait(&empty[s], ph ^ 1u)) { atomicOr(P.err, 1); break; }
        mbar_expect_tx(&full[s], STAGE);
        tma_load_2d(sbits + (size_t)s * STAGE, &tmB, &full[s], 0, (int)(g * N + c * kTile));
        if (++c == tpg) { c = 0; ++g; }
        if (++s == NS) { s = 0; ph ^= 1u; }
      }
      const int used = issued < NS ? (int)issued : NS;
      for (int j = 0; j < used; ++j) {
        int st = s - 1 - j;
        uint32_t p = ph;
        if (st < 0) { st += NS; p ^= 1u; }
        if (!mbar_wait(&full[st], p)) atomicOr(P.err, 2);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = qjl_tc::idesc_u8s8(NCOL);
      int64_t g = i0 / tpg, c = i0 - (i0 / tpg) * tpg;
      int64_t cur_g = -1;
      int gi = -1, tb = 0;
      int ab = 0, db = 0;
      uint32_t apar = 0, dpar = 0;
      bool ok = true;
      for (int64_t it = i0; it < i1 && ok; ++it) {
        if (g != cur_g) {
          cur_g = g;
          ++gi;
          tb = gi % ntab;
          if (!mbar_wait(&tfull[tb], (uint32_t)((gi / ntab) & 1))) { atomicOr(P.err, 8); break; }
        }
        if (!mbar_wait(&dempty[db], dpar ^ 1u)) { atomicOr(P.err, 8); break; }
        qjl_tc::fence_after();
        const uint32_t d_tm = tmem_base + (uint32_t)(db * kDStride);
        const uint32_t tab = smem_u32(tabs + (size_t)tb * TAB);
        for (int ch = 0; ch < NCH; ++ch) {
          if (!mbar_wait(&afull[ab], apar)) { atomicOr(P.err, 8); ok = false; break; }
          qjl_tc::fence_after();
          const uint32_t a_tm = tmem_base + (uint32_t)(kAcol0 + ab * 8 * KC);
#pragma unroll
          for (int t = 0; t < KC; ++t)
            qjl_tc::mma_i8_ts(d_tm, a_tm + (uint32_t)(8 * t),
                              qjl_tc::kmajor_desc(tab + (uint32_t)((ch * KC + t) * NCOL * 32)), idesc,
                              (ch | t) != 0 ? 1u : 0u);
          qjl_tc::commit(&aempty[ab]);
          if (++ab == NA) { ab = 0; apar ^= 1u; }
        }
        if (!ok) break;
        qjl_tc::commit(&dfull[db]);
        if (++db == ND) { db = 0; dpar ^= 1u; }
        if (++c == tpg) { c = 0; ++g; }
      }
      // every MMA issued has completed before TMEM is freed
      qjl_tc::commit(dbar);
      if (!mbar_wait(dbar, 0)) atomicOr(P.err, 8);
    }
  } else if (warp < 2 + kExpWarps) {
    // ---------------- expanders: thread r owns key row r (TMEM lane r)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    int s = 0, ab = 0;
    uint32_t ph = 0, apar = 0;
    for (int64_t it = i0; it < i1; ++it) {
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) { atomicOr(P.err, 4); break; }
      const unsigned char* stg = sbits + (size_t)s * STAGE;
      bool ok = true;
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        // this chunk's KC words of row r (16-byte pieces at their swizzled offsets)
        uint32_t words[KC];
#pragma unroll
        for (int k = 0; k < KC / 4; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(stg + swz_ofs<W>(r, ch * (KC / 4) + k));
          words[4 * k] = v.x; words[4 * k + 1] = v.y; words[4 * k + 2] = v.z; words[4 * k + 3] = v.w;
        }
        if (ch == NCH - 1) {
          // the stage is read: hand it back to the producer
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&aempty[ab], apar ^ 1u))) { atomicOr(P.err, 4); ok = false; break; }
        qjl_tc::fence_after();
        const uint32_t a_addr = tmem_base + lane_off + (uint32_t)(kAcol0 + ab * 8 * KC);
        // column 8 t + s' of word t: byte e is bit 8 e + s' of the word (0 or 1)
#pragma unroll
        for (int t4 = 0; t4 < KC; t4 += 4) {
          uint32_t a[32];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t w = words[t4 + u];
#pragma unroll
            for (int sh = 0; sh < 8; ++sh) a[8 * u + sh] = (w >> sh) & 0x01010101u;
          }
          qjl_tc::st32(a_addr + (uint32_t)(8 * t4), a);
        }
        qjl_tc::wait_st();
        qjl_tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[ab]);
        if (++ab == NA) { ab = 0; apar ^= 1u; }
      }
      if (++s == NS) { s = 0; ph ^= 1u; }
      if (!ok) break;
    }
  } else {
    // ---------------- epilogue and table builder
    const int ew = warp - 2 - kExpWarps;   // 0..7
    const int tid = ew * 32 + lane;        // 0..255, named barrier 1
    const int quarter = warp & 3;
    const int hq = ew >> 2;                // which share of the queries
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int J = P.J;
    const int64_t g_first = i0 / tpg;
    const int64_t ngroups = i1 > i0 ? (i1 - 1) / tpg - g_first + 1 : 0;
    for (int k = 0; k < ntab && k < ngroups; ++k) {
      build_table<W, JP>(P.sq + (g_first + k) * (int64_t)J * m, J, P.est_scale, tabs + (size_t)k * TAB,
                         s_cst + 64 * k, tid);
      if (tid == 0) mbar_arrive(&tfull[k]);
    }
    const uint64_t pol = qjl_hint::evict_first();
    int64_t g = g_first, c = i0 - g_first * tpg;
    int64_t cur_g = g;
    int gi = 0, tb = 0, db = 0;
    uint32_t dpar = 0;
    bool dead = false;  // a timed-out wait: keep the builds' barriers, skip the work
    // A tile's norms come from HBM, and the epilogue is the stage that releases the D buffers,
    // so they are fetched one tile ahead: the load for tile it + 1 is issued while tile it's
    // accumulator is awaited and stored.
    auto norm_of = [&](int64_t gg, int64_t cc) {
      const int64_t nn = cc * kTile + r;
      return nn < N ? __ldg(P.norms + gg * N + nn) : 0.f;
    };
    float nrm_next = i0 < i1 ? norm_of(g, c) : 0.f;
    for (int64_t it = i0; it < i1; ++it) {
      if (g != cur_g) {
        cur_g = g;
        ++gi;
        tb = gi % ntab;
      }
      const int64_t n0 = c * kTile;
      const int cnt = (int)(N - n0 < kTile ? N - n0 : kTile);
      const float nrm = nrm_next;
      if (it + 1 < i1) nrm_next = c + 1 == tpg ? norm_of(g + 1, 0) : norm_of(g, c + 1);
      if (!dead && !__all_sync(0xffffffffu, mbar_wait(&dfull[db], dpar))) { atomicOr(P.err, 16); dead = true; }
      if (!dead) {
        qjl_tc::fence_after();
        uint32_t hi[JH], lo[JH];
        const uint32_t dt = tmem_base + lane_off + (uint32_t)(db * kDStride + hq * JH);
        tmem_ld<JH>(dt, hi);
        tmem_ld<JH>(dt + JP, lo);
        qjl_tc::wait_ld();
        qjl_tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[db]);
        if (r < cnt) {
          const int64_t n = n0 + r;
          float* out = P.scores + (g * J + hq * JH) * N + n;
          const float2* cst = s_cst + 64 * tb + hq * JH;
          // ALL: every query of this warp's share exists, so the stores need no per-query branch
          // (each guarded store of the other form is a branch around the store instruction)
          auto write = [&](auto all_c) {
            constexpr bool ALL = decltype(all_c)::value;
#pragma unroll
            for (int jj = 0; jj < JH; jj += 2) {
              // sum b Q = 256 D_hi + D_lo, exact in int32 (|.| <= m * 32639 < 2^31); two queries at once
              const float4 cc = *reinterpret_cast<const float4*>(cst + jj);  // (c1, c0) of queries jj, jj + 1
              const float d0 = (float)((int)hi[jj] * 256 + (int)lo[jj]);
              const float d1 = (float)((int)hi[jj + 1] * 256 + (int)lo[jj + 1]);
              float e0, e1;
              asm("{\n\t.reg .b64 a, b, c;\n\t"
                  "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
                  "fma.rn.f32x2 a, a, b, c;\n\tmov.b64 b, {%8, %8};\n\tmul.rn.f32x2 a, a, b;\n\t"
                  "mov.b64 {%0, %1}, a;\n\t}"
                  : "=f"(e0), "=f"(e1)
                  : "f"(cc.x), "f"(cc.z), "f"(d0), "f"(d1), "f"(cc.y), "f"(cc.w), "f"(nrm));
              if (ALL || hq * JH + jj < J) qjl_hint::st_f32(out + (int64_t)jj * N, e0, pol);
              if (ALL || hq * JH + jj + 1 < J) qjl_hint::st_f32(out + (int64_t)(jj + 1) * N, e1, pol);
            }
          };
          if (hq * JH + JH <= J) write(std::true_type());
          else write(std::false_type());
        }
      }
      if (++db == ND) { db = 0; dpar ^= 1u; }
      // after the last tile of this group in the range, the MMAs that read its table are
      // complete: the buffer takes the table of the group ntab places further on
      const bool last = (c + 1 == tpg) || (it + 1 == i1);
      if (last && gi + ntab < ngroups) {
        build_table<W, JP>(P.sq + (g_first + gi + ntab) * (int64_t)J * m, J, P.est_scale, tabs + (size_t)tb * TAB,
                           s_cst + 64 * tb, tid);
        if (tid == 0) mbar_arrive(&tfull[tb]);
      }
      if (++c == tpg) { c = 0; ++g; }
    }
  }
  qjl_tc::fence_before();
  __syncthreads();
  qjl_tc::fence_after();
  if (warp == 1) qjl_tc::dealloc(tmem_base, kTmemCols);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
    return (EncodeTiledFn) nullptr;
  }();
  return fn;
}

// 2-D map over the sign words: rows of W uint32, boxes of 128 rows, swizzle of the row width.
bool bits_map(CUtensorMap* map, const uint32_t* bits, uint64_t rows, int W) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)W, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)W * 4};
  const cuuint32_t box[2] = {(cuuint32_t)W, (cuuint32_t)kTile};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = W == 32 ? CU_TENSOR_MAP_SWIZZLE_128B
                                        : (W == 16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(bits), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int W, int JP>
qjl_status launch_many_t(const qjl_projection* Pj, const uint32_t* bits, const float* norms, int64_t G, int64_t N,
                         const float* sq, int J, float* scores, cudaStream_t st) {
  constexpr size_t TAB = (size_t)2 * JP * 32 * W;
  constexpr size_t STAGE = (size_t)kTile * W * 4;
  constexpr int NA = n_abuf(W);
  const int NS = 4;
  const int ntab = 2 * TAB + NS * STAGE <= 200 * 1024 ? 2 : 1;
  size_t smem = 1024 + NS * STAGE + ntab * TAB + 2 * 128 * 4 + (size_t)(2 * NS + 2 * NA + 7) * 8 + 16;
  smem = std::max<size_t>(smem, 120 * 1024);  // one CTA per SM: it holds all 512 TMEM columns
  // the map (keyed on pointer and rows; one cache per instantiation, so per W) is cached per thread
  struct MapCache {
    const uint32_t* bits = nullptr;
    uint64_t rows = 0;
    CUtensorMap map;
  };
  static thread_local MapCache mc;
  const uint64_t rows = (uint64_t)G * (uint64_t)N;
  if (mc.bits != bits || mc.rows != rows) {
    mc.bits = nullptr;
    if (!bits_map(&mc.map, bits, rows, W))
      return qjl_set_error(QJL_ERR_CUDA, "cuTensorMapEncodeTiled failed for the sign words");
    mc.bits = bits;
    mc.rows = rows;
  }
  int* err = qjl_error_flag(Pj->device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  auto kern = scores_many_kernel<W, JP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return qjl_check_launch("scores_many_kernel smem attribute");
  const int64_t total = G * ((N + kTile - 1) / kTile);
  const int64_t grid = std::min<int64_t>(total, qjl_num_sms(Pj->device));
  const int64_t ipc = (total + grid - 1) / grid;
  const int64_t nblk = (total + ipc - 1) / ipc;
  ManyParams prm{bits, norms, sq, scores, err, G, N, ipc, J, NS, ntab, Pj->est_scale};
  qjl_log_launch("scores_many_kernel", nblk, kThreads, smem, 1);
  kern<<<(unsigned)nblk, kThreads, smem, st>>>(mc.map, prm);
  return qjl_check_launch("scores_many_kernel");
}

template <int W>
qjl_status launch_many_w(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G, int64_t N,
                         const float* sq, int J, float* scores, cudaStream_t st) {
  if (J <= 8) return launch_many_t<W, 8>(P, bits, norms, G, N, sq, J, scores, st);
  if (J <= 16) return launch_many_t<W, 16>(P, bits, norms, G, N, sq, J, scores, st);
  if (J <= 32) return launch_many_t<W, 32>(P, bits, norms, G, N, sq, J, scores, st);
  return launch_many_t<W, 64>(P, bits, norms, G, N, sq, J, scores, st);
}

}  // namespace

// Rows of one launch: the TMA row coordinate is a signed 32-bit int.
constexpr int64_t kMaxRows = 2147483647LL - 2 * kTile;

bool scores_many_supported(int m, int64_t N) { return (m == 256 || m == 512 || m == 1024) && N <= kMaxRows; }

qjl_status launch_scores_many(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G,
                              int64_t N, const float* sq, int J, float* scores, cudaStream_t st) {
  const int W = P->m / 32;
  if ((W != 8 && W != 16 && W != 32) || N > kMaxRows)
    return qjl_set_error(QJL_ERR_UNSUPPORTED, "many-query scores need m in {256, 512, 1024} and N < 2^31");
  // one launch per run of groups whose rows fit the map's 32-bit coordinates
  const int64_t gmax = std::max<int64_t>(1, kMaxRows / N);
  for (int64_t g0 = 0; g0 < G; g0 += gmax) {
    const int64_t gc = std::min(gmax, G - g0);
    const uint32_t* b = bits + g0 * N * W;
    const float* nr = norms + g0 * N;
    const float* q = sq + g0 * (int64_t)J * P->m;
    float* out = scores + g0 * (int64_t)J * N;
    qjl_status s = W == 8 ? launch_many_w<8>(P, b, nr, gc, N, q, J, out, st)
                          : (W == 16 ? launch_many_w<16>(P, b, nr, gc, N, q, J, out, st)
                                     : launch_many_w<32>(P, b, nr, gc, N, q, J, out, st));
    if (s != QJL_OK) return s;
  }
  return QJL_OK;
}
