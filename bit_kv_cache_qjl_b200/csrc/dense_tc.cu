// Dense QJL key sketch on the 5th-generation tensor cores (tcgen05 + TMA).
//
// QJL abstract ("Majid Daliri" page): a key is stored as sign(S k) plus
// ||k||. For a batch of keys K [n][d] this is a dense contraction K S^T
// followed by a sign. "Fast Quantized Johnson - Lindenstrauss Transforms"
// ("Transcript: The paper's improvements") notes that the dense projection
// is the slow one to apply, so it runs on the tensor cores: bf16 operands
// with fp32 accumulators in TMEM.
//
// Persistent kernel, one CTA per SM, 12 warps:
//   warp 0     TMA producer. S_eff [m][d] is loaded once into shared memory.
//              Then 128-key tiles stream through an NS-stage ring, each
//              stage 128 rows x d bf16 in 128-byte swizzled atoms of 64
//              columns.
//   warp 1     allocates 512 TMEM columns (two 128 x 256 fp32 accumulators).
//              One elected lane issues tcgen05.mma M=128, N<=256, K=16 over
//              d/16 steps per work unit. A work unit is (tile, 256-column
//              chunk of m). Completion goes to mbarriers via tcgen05.commit.
//   warps 2-9  epilogue. Warp w reads TMEM lanes 32*(w%4)..+31, so each
//              thread owns one key row. The two warps on a lane quarter take
//              half of the accumulator columns each: four tcgen05.ld of 32
//              columns with one wait, and eight independent funnel-shift
//              chains per 64 values gather the sign bits (bit = 1 iff y >= 0).
//              Words leave as 16-byte stores.
//   warps 10-11 ||k|| from the swizzled key tile already in shared memory:
//              two rows per thread, sm_100 mixed-precision FMA (bf16 in, fp32
//              accumulate, 4 accumulators per row). These warps, not the epilogue,
//              release the key stage together with the MMAs' commit.
// Every mbarrier wait is bounded. On expiry the kernel records an error
// flag, drains what it issued, frees TMEM and returns.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string.h>

#include <mutex>

#include "cache_hint.cuh"
#include "key_math.cuh"
#include "qjl_internal.h"

namespace {

using qjl_km::sq_acc_bf16x2;

constexpr int BM = 128;            // keys per tile (MMA M)
constexpr int kEpiWarps = 8;
constexpr int kNormWarps = 2;
constexpr int kThreads = (2 + kEpiWarps + kNormWarps) * 32;  // producer, MMA, epilogue, norms
constexpr int kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s

struct TcParams {
  int64_t n;
  int m;
  int ns;        // pipeline stages
  int nchunk;    // ceil(m / 256)
  uint32_t* bits;
  float* norms;
  int* err;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase with the given parity: gives up after
// kWaitLimitNs of wall time and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if ((it & 255u) == 255u) {
      const uint64_t now = global_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > kWaitLimitNs) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), LBO unused for swizzled K-major (encoded as 1),
// descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t desc = (uint64_t)((saddr >> 4) & 0x3FFFu);
  desc |= (uint64_t)1u << 16;
  desc |= (uint64_t)(1024u >> 4) << 32;
  desc |= (uint64_t)1u << 46;
  desc |= (uint64_t)2u << 61;
  return desc;
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M=128, N.
__host__ __device__ constexpr uint32_t idesc_bf16(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Two back-to-back 32-column TMEM loads (64 columns of this thread's row), no wait.
__device__ __forceinline__ void tmem_ld64_nowait(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr + 32u));
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld64_nowait(taddr, r);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 64 fp32 accumulators -> 2 sign words (bit i of word k = 1 iff value 32k+i >= 0
// as a sign bit). Eight independent 8-step funnel-shift chains keep the
// dependency depth at 8 instead of 32.
__device__ __forceinline__ void sign_words2(const uint32_t (&r)[64], uint32_t& w0, uint32_t& w1) {
  uint32_t c[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) c[k] = 0u;
#pragma unroll
  for (int i = 7; i >= 0; --i) {
#pragma unroll
    for (int k = 0; k < 8; ++k) c[k] = __funnelshift_l(r[8 * k + i], c[k], 1);
  }
  w0 = ~(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24));
  w1 = ~(c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// 128 columns (four 32-column loads issued back to back, one wait) -> 4 sign words.
__device__ __forceinline__ void tmem_ld128_pack(uint32_t taddr, uint32_t (&w)[4]) {
  uint32_t v0[64], v1[64];
  tmem_ld64_nowait(taddr, v0);
  tmem_ld64_nowait(taddr + 64u, v1);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  sign_words2(v0, w[0], w[1]);
  sign_words2(v1, w[2], w[3]);
}

__device__ __forceinline__ void tmem_ld64_pack(uint32_t taddr, uint32_t& w0, uint32_t& w1) {
  uint32_t v[64];
  tmem_ld64(taddr, v);
  sign_words2(v, w0, w1);
}

__device__ __forceinline__ void flag_error(int* err, int code) { atomicOr(err, code); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1) dense_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                             const __grid_constant__ CUtensorMap tmS,
                                                             const TcParams prm) {
  constexpr int KA = D / 64;                    // 64-column swizzle atoms per row
  constexpr uint32_t kStageBytes = KA * BM * 128;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  // 1024-byte alignment for the swizzled operands
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_dyn + 1023) & ~(uintptr_t)1023);
  const int m = prm.m;
  const int NS = prm.ns;
  unsigned char* sS = base;                                   // KA atoms x m rows x 128 B
  unsigned char* sK = sS + (size_t)KA * m * 128;              // NS stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + (size_t)NS * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + NS;
  uint64_t* tfull = empty + NS;
  uint64_t* tempty = tfull + 2;
  uint64_t* sbar = tempty + 2;
  uint64_t* dbar = sbar + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(dbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (prm.n + BM - 1) / BM;
  const int nchunk = prm.nchunk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kNormWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(sbar, 1);
    mbar_init(dbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // S_eff once: KA atoms x ceil(m/256) row blocks
      const int sblocks = (m + 255) / 256;
      mbar_expect_tx(sbar, (uint32_t)(KA * m * 128));
      for (int a = 0; a < KA; ++a)
        for (int rb = 0; rb < sblocks; ++rb)
          tma_load_2d(sS + ((size_t)a * m + rb * 256) * 128, &tmS, sbar, a * 64, rb * 256);
      int64_t issued = 0;
      int s = 0;
      uint32_t ph = 0;
      for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++issued) {
        if (!mbar_wait(&empty[s], ph ^ 1u)) { flag_error(prm.err, 1); break; }
        mbar_expect_tx(&full[s], kStageBytes);
        unsigned char* dst = sK + (size_t)s * kStageBytes;
        for (int a = 0; a < KA; ++a) tma_load_2d(dst + a * BM * 128, &tmK, &full[s], a * 64, (int)(t * BM));
        if (++s == NS) { s = 0; ph ^= 1u; }
      }
      // drain: the most recent phase of every used stage must have landed before exit
      const int used = issued < NS ? (int)issued : NS;
      for (int j = 0; j < used; ++j) {
        int st = s - 1 - j;
        uint32_t p = ph;
        if (st < 0) { st += NS; p ^= 1u; }
        if (!mbar_wait(&full[st], p)) flag_error(prm.err, 2);
      }
      if (!mbar_wait(sbar, 0)) flag_error(prm.err, 2);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(sbar, 0);
      if (!ok) flag_error(prm.err, 4);
      uint32_t u = 0;
      int s = 0;
      uint32_t ph = 0;
      for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        if (!mbar_wait(&full[s], ph)) { flag_error(prm.err, 4); ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sK + (size_t)s * kStageBytes);
        for (int c = 0; c < nchunk && ok; ++c, ++u) {
          const int buf = (int)(u & 1u);
          if (!mbar_wait(&tempty[buf], ((u >> 1) & 1u) ^ 1u)) { flag_error(prm.err, 4); ok = false; break; }
          tc_fence_after();
          const int N = min(256, m - 256 * c);
          const uint32_t idesc = idesc_bf16(N);
          const uint32_t dcol = tmem_base + (uint32_t)(buf * 256);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int a = kk >> 2;
            const uint32_t koff = (uint32_t)((kk & 3) * 32);
            const uint64_t adesc = sw128_desc(a_base + (uint32_t)(a * BM * 128) + koff);
            const uint64_t bdesc = sw128_desc(smem_u32(sS) + (uint32_t)(((size_t)a * m + 256 * c) * 128) + koff);
            mma_bf16(dcol, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&tfull[buf]);
        }
        mma_commit(&empty[s]);
        if (++s == NS) { s = 0; ph ^= 1u; }
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(dbar);
      if (!mbar_wait(dbar, 0)) flag_error(prm.err, 8);
    }
  } else if (warp < 2 + kEpiWarps) {
    // epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (the hardware ties a warp
    // to its lane quarter), so each thread owns one key row; the two warps on a
    // quarter take half of the accumulator columns each
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int W = m >> 5;
    uint32_t u = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const int64_t row = t * BM + r;
      for (int c = 0; c < nchunk; ++c, ++u) {
        const int buf = (int)(u & 1u);
        if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (u >> 1) & 1u))) { flag_error(prm.err, 16); ok = false; break; }
        tc_fence_after();
        const int N = min(256, m - 256 * c);
        const int hc = N >> 1;  // columns per half: 128 or 64
        const uint32_t taddr =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * 256 + half * hc);
        if (hc == 128) {
          uint32_t wq[4];
          tmem_ld128_pack(taddr, wq);
          if (row < prm.n)
            qjl_hint::st_v4(prm.bits + row * W + c * 8 + half * 4, wq[0], wq[1], wq[2], wq[3], qjl_hint::evict_first());
        } else {
          uint32_t w0, w1;
          tmem_ld64_pack(taddr, w0, w1);
          if (row < prm.n) qjl_hint::st_v2(prm.bits + row * W + c * 8 + half * 2, w0, w1, qjl_hint::evict_first());
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
      }
    }
  } else {
    // norm warps: ||k|| of rows 32*nw + lane and 32*nw + lane + 64 from the swizzled key tile
    // (16-byte chunk c of row r sits at chunk c ^ (r % 8)); then the stage is
    // released together with the MMAs' commit
    const int r0 = (warp - 2 - kEpiWarps) * 32 + lane;  // rows r0 and r0 + 64
    int s = 0;
    uint32_t ph = 0;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) { flag_error(prm.err, 32); break; }
      const unsigned char* tile = sK + (size_t)s * kStageBytes;
      float acc[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[j][k] = 0.f;
#pragma unroll
      for (int a = 0; a < KA; ++a) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int r = r0 + 64 * j;
            const uint4 v = *reinterpret_cast<const uint4*>(tile + a * BM * 128 + r * 128 + ((c ^ (r & 7)) << 4));
            sq_acc_bf16x2(v.x, acc[j][0]);
            sq_acc_bf16x2(v.y, acc[j][1]);
            sq_acc_bf16x2(v.z, acc[j][2]);
            sq_acc_bf16x2(v.w, acc[j][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int64_t row = t * BM + r0 + 64 * j;
        if (row < prm.n)
          qjl_hint::st_f32(prm.norms + row, sqrtf((acc[j][0] + acc[j][1]) + (acc[j][2] + acc[j][3])),
                           qjl_hint::evict_first());
      }
      if (++s == NS) { s = 0; ph ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2D bf16 map: rows x cols (inner), row stride ld elements, box 64 cols x box_rows, 128B swizzle.
bool make_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kSmemLimit = 227 * 1024;

size_t smem_bytes(int d, int m, int ns) {
  return 1024 + (size_t)(d / 64) * m * 128 + (size_t)ns * (d / 64) * BM * 128 + (2 * ns + 6) * 8 + 16;
}

int pick_stages(int d, int m) {
  for (int ns = 6; ns >= 2; --ns)
    if (smem_bytes(d, m, ns) <= kSmemLimit) return ns;
  return 0;
}

}  // namespace

bool dense_tc_supported(const qjl_projection* P, int dtype, const void* keys, int64_t ld) {
  if (dtype != QJL_BF16 || !P->S_bf16 || !P->opt.s_bf16) return false;
  if (P->d % 64 || P->d > 256) return false;
  if (P->m % 256 && P->m != 128) return false;  // S loads in 256-row boxes
  if (((uintptr_t)keys & 15u) || (ld * 2) % 16) return false;
  return pick_stages(P->d, P->m) >= 2 && get_encode() != nullptr;
}

static_assert(sizeof(CUtensorMap) == sizeof(qjl_projection::s_map), "CUtensorMap size");

bool qjl_make_bf16_map(void* map, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  return make_map(reinterpret_cast<CUtensorMap*>(map), ptr, rows, cols, ld, box_rows);
}

void dense_tc_prepare(qjl_projection* P) {
  P->s_map_ok = P->S_bf16 && make_map(reinterpret_cast<CUtensorMap*>(P->s_map), P->S_bf16, (uint64_t)P->m,
                                      (uint64_t)P->d, (uint64_t)P->d, (uint32_t)std::min(P->m, 256));
}

qjl_status launch_dense_tc(const qjl_projection* P, const void* keys, int64_t n, int64_t ld, uint32_t* bits,
                           float* norms, cudaStream_t st) {
  // The keys' map is cached per thread for the last (pointer, rows, ld, d): a
  // caller that quantises the same buffer every step encodes it once. S's map
  // was encoded with the projection.
  struct KeyMapCache {
    const void* ptr = nullptr;
    int64_t n = -1, ld = -1;
    int d = -1;
    CUtensorMap map;
  };
  static thread_local KeyMapCache kc;
  if (kc.ptr != keys || kc.n != n || kc.ld != ld || kc.d != P->d) {
    kc.ptr = nullptr;
    if (!make_map(&kc.map, keys, (uint64_t)n, (uint64_t)P->d, (uint64_t)ld, BM))
      return qjl_set_error(QJL_ERR_CUDA, "cuTensorMapEncodeTiled failed for the keys");
    kc.ptr = keys;
    kc.n = n;
    kc.ld = ld;
    kc.d = P->d;
  }
  const CUtensorMap tmK = kc.map;
  CUtensorMap tmS;
  if (P->s_map_ok) {
    memcpy(&tmS, P->s_map, sizeof(tmS));
  } else if (!make_map(&tmS, P->S_bf16, (uint64_t)P->m, (uint64_t)P->d, (uint64_t)P->d,
                       (uint32_t)std::min(P->m, 256))) {
    return qjl_set_error(QJL_ERR_CUDA, "cuTensorMapEncodeTiled failed for S");
  }
  int* err = qjl_error_flag(P->device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  const int ns = pick_stages(P->d, P->m);
  const size_t smem = smem_bytes(P->d, P->m, ns);
  TcParams prm{n, P->m, ns, (P->m + 255) / 256, bits, norms, err};
  const int64_t ntiles = (n + BM - 1) / BM;
  const int grid = (int)std::min<int64_t>(ntiles, qjl_num_sms(P->device));
  void (*kern)(CUtensorMap, CUtensorMap, TcParams) = nullptr;
  switch (P->d) {
    case 64: kern = dense_tc_kernel<64>; break;
    case 128: kern = dense_tc_kernel<128>; break;
    case 192: kern = dense_tc_kernel<192>; break;
    case 256: kern = dense_tc_kernel<256>; break;
    default: return qjl_set_error(QJL_ERR_UNSUPPORTED, "tensor-core path needs d in {64,128,192,256}");
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return qjl_check_launch("dense_tc_kernel smem attribute");
  qjl_log_launch("dense_tc_kernel", grid, kThreads, smem, 1);
  kern<<<grid, kThreads, smem, st>>>(tmK, tmS, prm);
  return qjl_check_launch("dense_tc_kernel");
}
