// FQJL key sketch with the first randomized Hadamard transform on the
// 5th-generation tensor cores (tcgen05 + TMA).
//
// "Fast Quantized Johnson - Lindenstrauss Transforms" ("Key concepts", "The
// paper" abstract): block b of the sketch is z = H D_g Pi H D_r x, up to a
// positive factor, with H the unnormalised Sylvester matrix and Pi the
// gather u'[i] = u[pi(i)]. Its first factor S1 = Pi H D_r has entries +-1:
// row i is row pi(i) of H with its columns signed by D_r. With bf16 keys
// every product k_c S1[i][c] is exact, so u' = S1 x is a dense contraction
// with exact operands and fp32 sums, run like the dense sketch: S1 resident
// in shared memory, keys streamed by TMA, tcgen05 MMAs into TMEM. The second
// factor H D_g is not exact in bf16 and stays on the FP32 lanes: epilogue
// warps read accumulator rows from TMEM (one key per thread), scale them by
// D_g and run the Walsh-Hadamard butterflies in registers. The top butterfly,
// which pairs the two halves of a block, is fused with D_g as the rows are
// read, and each warp transforms one output half. The D-FQJL dither (d = 128)
// follows the transform in the same warps.
//
// Persistent kernel, one CTA per SM:
//   warp 0     TMA producer: this pass's 256 rows of S1 once, then the keys as
//              128-row x 64-column bf16 boxes (one 128-byte swizzle atom
//              each) through an NS-slot ring, d/64 slots per 128-key tile.
//   warp 1     allocates 512 TMEM columns (two 128 x 256 fp32 accumulators);
//              one lane issues M=128, N=256, K=16 MMAs, four per slot.
//   warps 2-3  ||x|| from the swizzled key slots (as in the dense sketch).
//   warps 4-   epilogue. Warp w reads TMEM lanes 32 (w % 4) .. + 31, so each
//              thread owns one key.
//              d = 256: 8 warps; the two on a lane quarter form both output
//              halves of the block for 64 input pairs each and write them
//              back to TMEM, then take 128 outputs each (a 128-point
//              transform).
//              d = 128: 16 warps; four per lane quarter, two per block. Each
//              reads its block's row and forms one output half of 64 (a
//              64-point transform, its dither and two sign words), so that
//              four of them share an SM sub-partition and hide each other's
//              latencies.
// A pass covers 256 output coordinates (one block of d = 256 or two of
// d = 128). For m > 256 one launch runs m/256 groups of CTAs, one per pass,
// that walk the same tiles in step: each key tile comes from HBM once and is
// an L2 hit for the other passes.
//
// No output bit comes from a -0. D_g is applied in the sweep as
// fma(g, a, fma(+-g', b, +0)), so an exact zero is +0. Sums of values that are not -0 are not -0, so the stored bit is exactly
// [z >= 0].
//
// Every mbarrier wait is bounded. On expiry the kernel records an error flag,
// drains what it issued, frees TMEM and returns.

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "cache_hint.cuh"
#include "key_math.cuh"
#include "mbarrier.cuh"
#include "qjl_internal.h"
#include "tcgen05.cuh"

namespace {

using namespace qjl_km;
using qjl_sync::mbar_arrive;
using qjl_sync::mbar_expect_tx;
using qjl_sync::mbar_fence_init;
using qjl_sync::mbar_init;
using qjl_sync::mbar_wait;
using qjl_sync::smem_u32;

constexpr int BM = 128;                   // keys per tile (MMA M)
constexpr int kPass = 256;                // output coordinates per pass (MMA N)
constexpr int kNormWarps = 2;
// epilogue warps and threads per CTA
template <int D>
__host__ __device__ constexpr int epi_warps() { return D == 128 ? 16 : 8; }
template <int D>
__host__ __device__ constexpr int ftc_threads() { return (2 + kNormWarps + epi_warps<D>()) * 32; }
// Register split by warpgroup (setmaxnreg, d = 128 only: it measured slower for d = 256). The
// launch of 640 threads gets 96 registers a thread (65536 / 640, rounded down to a multiple of
// 8); the producer, MMA and norm warps give theirs up for the epilogue: 128 x 56 + 512 x 104 =
// 60416 <= 640 x 96.
constexpr int kRegsLaunch = 96;
constexpr int kRegsLow = 56;
constexpr int kRegsHigh = 104;
static_assert(128 * kRegsLow + 512 * kRegsHigh <= ftc_threads<128>() * kRegsLaunch, "register split exceeds the launch");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotBytes = BM * 128;  // 128 keys x 64 bf16 channels
constexpr size_t kSmemLimit = 227 * 1024;

struct FtcParams {
  int64_t n;
  int W;                 // sign words per key row
  int npass;             // m / 256: CTA c takes pass c % npass (coordinates 256 pass ..
                         // 256 pass + 255) and every (gridDim / npass)-th tile from c / npass
  int ns;                // ring slots
  const float* D_g;      // [m], all blocks
  float sigma;           // D-FQJL dither sigma_rel (the dithered instantiation)
  uint32_t k0, k1;       // the seed as the Philox key
  uint64_t first_token;  // token index of row 0 (the dither's counter)
  uint32_t rk[20];       // Philox round keys of (k0, k1)
  uint32_t* bits;
  float* norms;          // written by the CTAs of pass 0
  int* err;
};

__device__ __forceinline__ void flag_error(int* err, int code) { atomicOr(err, code); }

// 2 NP-point unnormalised Walsh-Hadamard transform in place, V[t] = (v_2t, v_2t+1): the pair
// stage within registers, then log2(NP) stages of packed butterflies.
template <int NP>
__device__ __forceinline__ void fwht(float2 (&V)[NP]) {
#pragma unroll
  for (int t = 0; t < NP; ++t) {
    const float a = V[t].x, b = V[t].y;
    V[t].x = a + b;
    V[t].y = a - b;
  }
#pragma unroll
  for (int h = 1; h < NP; h <<= 1) {
#pragma unroll
    for (int t = 0; t < NP; ++t)
      if (!(t & h)) bfly2(V[t], V[t + h]);
  }
}

// Sign words of 2 NP values: bit k of word j is 1 iff element 32 j + k >= 0. NP / 8 independent
// funnel-shift chains of 16 elements each.
template <int NP>
__device__ __forceinline__ void sign_words(const float2 (&V)[NP], uint32_t (&w)[NP / 16]) {
  constexpr int NC = NP / 8;
  uint32_t c[NC];
#pragma unroll
  for (int k = 0; k < NC; ++k) c[k] = 0u;
#pragma unroll
  for (int i = 7; i >= 0; --i) {
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      c[k] = __funnelshift_l(__float_as_uint(V[8 * k + i].y), c[k], 1);
      c[k] = __funnelshift_l(__float_as_uint(V[8 * k + i].x), c[k], 1);
    }
  }
#pragma unroll
  for (int j = 0; j < NP / 16; ++j) w[j] = ~(c[2 * j] | (c[2 * j + 1] << 16));
}

// D-FQJL dither of coordinates e0 .. e0 + 2 NP - 1 of token tok, scaled by amp, added to V: the
// register kernel's draw (fqjl_keys.cu). Coordinate e comes from the Philox4x32-10 block at
// counter (e/8, tok_lo, tok_hi, dither stream): word w gives coordinates 8c + 2w and
// 8c + 2w + 1, the pair V[4c + w], by Box-Muller on its two 16-bit halves. Four blocks at a
// time, their rounds interleaved.
template <int NP>
__device__ __forceinline__ void add_dither(float2 (&V)[NP], uint32_t e0, uint64_t tok, float amp,
                                           const uint32_t (&rk)[20]) {
  static_assert(NP % 16 == 0, "whole groups of four Philox blocks");
  const uint32_t cb = e0 >> 3, tlo = (uint32_t)tok, thi = (uint32_t)(tok >> 32);
#pragma unroll
  for (int c = 0; c < NP / 4; c += 4) {
    qjl::U32x4 w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) w[j] = qjl::U32x4{cb + c + j, tlo, thi, qjl::kStreamDither};
    philox_xn_rk<4>(w, rk);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = 4 * (c + j);
      add_box_muller16(V[q], w[j].x, amp);
      add_box_muller16(V[q + 1], w[j].y, amp);
      add_box_muller16(V[q + 2], w[j].z, amp);
      add_box_muller16(V[q + 3], w[j].w, amp);
    }
  }
}

__device__ __forceinline__ float2 as_f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}

// First sweep of the top butterfly fused with D_g over 32 columns: with a = A[k], b = B[k],
// A[k] <- g[k] a + gp[k] b and B[k] <- g[k] a + gn[k] b (gn = -gp), each as
// fma(g, a, fma(+-g', b, +0)) so that an exact zero is +0.
__device__ __forceinline__ void sweep32(uint32_t (&A)[32], uint32_t (&B)[32], const float* g, const float* gp,
                                        const float* gn) {
#pragma unroll
  for (int q = 0; q < 32; q += 4) {
    const float4 ga = *reinterpret_cast<const float4*>(g + q);
    const float4 gpp = *reinterpret_cast<const float4*>(gp + q);
    const float4 gnn = *reinterpret_cast<const float4*>(gn + q);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 g0 = e ? make_float2(ga.z, ga.w) : make_float2(ga.x, ga.y);
      const float2 g1 = e ? make_float2(gpp.z, gpp.w) : make_float2(gpp.x, gpp.y);
      const float2 g2 = e ? make_float2(gnn.z, gnn.w) : make_float2(gnn.x, gnn.y);
      const int k = q + 2 * e;
      const float2 a = as_f2(A[k], A[k + 1]), b = as_f2(B[k], B[k + 1]);
      float2 p = b, n = b, v0 = a, v1 = a;
      mulz2(p, g1);
      mulz2(n, g2);
      fma2(v0, g0, p);
      fma2(v1, g0, n);
      A[k] = __float_as_uint(v0.x);
      A[k + 1] = __float_as_uint(v0.y);
      B[k] = __float_as_uint(v1.x);
      B[k + 1] = __float_as_uint(v1.y);
    }
  }
}

// The epilogue warp is done reading accumulator buffer `bar`'s TMEM columns.
__device__ __forceinline__ void release_tmem(uint64_t* bar, int lane) {
  qjl_tc::fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

template <int D, bool DITHER>
__global__ void __launch_bounds__(ftc_threads<D>(), 1) fqjl_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                            const __grid_constant__ CUtensorMap tmS,
                                                            const FtcParams prm) {
  static_assert(D == 128 || D == 256, "d in {128, 256}");
  static_assert(!DITHER || D == 128, "the dithered instantiation is d = 128");
  constexpr int KA = D / 64;  // key slots (64-column atoms) per tile
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_dyn + 1023) & ~(uintptr_t)1023);
  const int NS = prm.ns;
  unsigned char* sS = base;                                     // KA atoms x 256 rows x 128 B
  unsigned char* ring = sS + (size_t)KA * kPass * 128;          // NS slots
  float* sG = reinterpret_cast<float*>(ring + (size_t)NS * kSlotBytes);  // [2][256]
  float* sNrm = sG + 2 * kPass;  // [2][128]: ||x||^2 of the keys of the tiles in the two TMEM buffers
  uint64_t* full = reinterpret_cast<uint64_t*>(sNrm + 2 * BM);
  uint64_t* empty = full + NS;
  uint64_t* tfull = empty + NS;
  uint64_t* tempty = tfull + 2;
  uint64_t* sbar = tempty + 2;
  uint64_t* dbar = sbar + 1;
  uint64_t* xbar = dbar + 1;  // [4], d = 256: the two epilogue warps of a lane quarter, first sweep done
  uint64_t* nfull = xbar + 4;    // [2], dither: the norm warps wrote sNrm[b]
  uint64_t* nempty = nfull + 2;  // [2], dither: the epilogue warps read it
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(nempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (prm.n + BM - 1) / BM;
  // the npass CTAs of a group walk the same tiles in step, so a key tile read from HBM by one
  // of them is an L2 hit for the others
  const int pass = (int)(blockIdx.x % (unsigned)prm.npass);
  const int cta0 = (int)(blockIdx.x / (unsigned)prm.npass), ncta = (int)(gridDim.x / (unsigned)prm.npass);

  // D_g of this pass's coordinates. Row h scales the upper half of each block by (+1, -1)[h]: the
  // fused top butterfly reads row h for output half h.
  for (int i = threadIdx.x; i < 2 * kPass; i += blockDim.x) {
    const int h = i / kPass, c = i % kPass;
    const float g = __ldg(prm.D_g + (size_t)kPass * pass + c);
    sG[i] = (h == 1 && (c & (D / 2))) ? -g : g;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kNormWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], epi_warps<D>());
    }
    mbar_init(sbar, 1);
    mbar_init(dbar, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&xbar[q], 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&nfull[b], kNormWarps);
      mbar_init(&nempty[b], epi_warps<D>());
    }
    mbar_fence_init();
  }
  if (warp == 1) qjl_tc::alloc(tmem_holder, kTmemCols);
  qjl_tc::fence_before();
  __syncthreads();
  qjl_tc::fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp < 4) {
    if constexpr (D == 128) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
      if (lane == 0) {
        mbar_expect_tx(sbar, (uint32_t)(KA * kPass * 128));
        for (int a = 0; a < KA; ++a) qjl_tc::tma_load_2d(sS + (size_t)a * kPass * 128, &tmS, sbar, a * 64, kPass * pass);
        int64_t issued = 0;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int64_t t = cta0; t < ntiles && ok; t += ncta) {
          for (int a = 0; a < KA; ++a, ++issued) {
            if (!mbar_wait(&empty[s], ph ^ 1u)) { flag_error(prm.err, 1); ok = false; break; }
            mbar_expect_tx(&full[s], kSlotBytes);
            qjl_tc::tma_load_2d(ring + (size_t)s * kSlotBytes, &tmK, &full[s], a * 64, (int)(t * BM));
            if (++s == NS) { s = 0; ph ^= 1u; }
          }
        }
        // drain: the most recent phase of every used slot must have landed before exit
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
        const uint32_t idesc = qjl_tc::idesc_bf16(kPass);
        const uint32_t sS_addr = smem_u32(sS);
        uint32_t u = 0;
        int s = 0;
        uint32_t ph = 0;
        for (int64_t t = cta0; t < ntiles && ok; t += ncta, ++u) {
          const int buf = (int)(u & 1u);
          if (!mbar_wait(&tempty[buf], ((u >> 1) & 1u) ^ 1u)) { flag_error(prm.err, 4); break; }
          qjl_tc::fence_after();
          const uint32_t dcol = tmem_base + (uint32_t)(buf * 256);
          for (int a = 0; a < KA; ++a) {
            if (!mbar_wait(&full[s], ph)) { flag_error(prm.err, 4); ok = false; break; }
            qjl_tc::fence_after();
            const uint32_t a_addr = smem_u32(ring + (size_t)s * kSlotBytes);
            const uint32_t b_addr = sS_addr + (uint32_t)(a * kPass * 128);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              qjl_tc::mma_bf16_ss(dcol, qjl_tc::sw128_desc(a_addr + 32u * kk), qjl_tc::sw128_desc(b_addr + 32u * kk),
                                  idesc, (a | kk) ? 1u : 0u);
            qjl_tc::commit(&empty[s]);
            if (++s == NS) { s = 0; ph ^= 1u; }
          }
          if (!ok) break;
          qjl_tc::commit(&tfull[buf]);
        }
        // every MMA this thread issued has completed before TMEM is released
        qjl_tc::commit(dbar);
        if (!mbar_wait(dbar, 0)) flag_error(prm.err, 8);
      }
    } else {
      // norm warps: ||x|| of rows r0 and r0 + 64 of each tile from the swizzled key slots
      // (16-byte chunk c of row r sits at chunk c ^ (r % 8)), then the slot is released
      // together with the MMAs' commit. For the dither they also hand ||x||^2 to the
      // epilogue through sNrm, double-buffered like the TMEM accumulators.
      const int r0 = (warp - 2) * 32 + lane;
      int s = 0;
      uint32_t ph = 0, u = 0;
      bool ok = true;
      for (int64_t t = cta0; t < ntiles && ok; t += ncta, ++u) {
        float acc[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[j][k] = 0.f;
        for (int a = 0; a < KA; ++a) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) { flag_error(prm.err, 32); ok = false; break; }
          const unsigned char* slot = ring + (size_t)s * kSlotBytes;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int rr = r0 + 64 * j;
              const uint4 v = *reinterpret_cast<const uint4*>(slot + rr * 128 + ((c ^ (rr & 7)) << 4));
              sq_acc_bf16x2(v.x, acc[j][0]);
              sq_acc_bf16x2(v.y, acc[j][1]);
              sq_acc_bf16x2(v.z, acc[j][2]);
              sq_acc_bf16x2(v.w, acc[j][3]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
          if (++s == NS) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        float x2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) x2[j] = (acc[j][0] + acc[j][1]) + (acc[j][2] + acc[j][3]);
        if constexpr (DITHER) {
          const int nb = (int)(u & 1u);
          if (!__all_sync(0xffffffffu, mbar_wait(&nempty[nb], ((u >> 1) & 1u) ^ 1u))) {
            flag_error(prm.err, 32);
            break;
          }
          sNrm[nb * BM + r0] = x2[0];
          sNrm[nb * BM + r0 + 64] = x2[1];
          __syncwarp();
          if (lane == 0) mbar_arrive(&nfull[nb]);
        }
        if (pass != 0) continue;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int64_t row = t * BM + r0 + 64 * j;
          if (row < prm.n) qjl_hint::st_f32(prm.norms + row, sqrtf(x2[j]), qjl_hint::evict_first());
        }
      }
    }
  } else {
    if constexpr (D == 128) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int quarter = warp & 3;
    const int part = ((warp - 4) >> 2) & 1;  // d = 256: output half; d = 128: block of the pass
    const int half = (warp - 4) >> 3;        // d = 128: output half of the block
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint64_t pol = qjl_hint::evict_first();
    uint32_t u = 0;
    for (int64_t t = cta0; t < ntiles; t += ncta, ++u) {
      const int buf = (int)(u & 1u);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (u >> 1) & 1u))) { flag_error(prm.err, 16); break; }
      qjl_tc::fence_after();
      const int64_t row = t * BM + r;
      const uint32_t tb = lane_base + (uint32_t)(buf * 256);
      if constexpr (D == 256) {
        // One block of 256: output half h is the 128-point transform of
        // v_h,i = g_i u'_i + (+-1)[h] g_{i+128} u'_{i+128}, i < 128. First sweep: this warp forms
        // both halves for i in [64 part, 64 part + 64) and writes them back in place, v_0 over
        // u'[0, 128) and v_1 over u'[128, 256), 32 columns at a time. Once the other warp of the
        // quarter has done the same, it reads its half back whole.
#pragma unroll 1
        for (int rr = 0; rr < 2; ++rr) {
          const int i0 = 64 * part + 32 * rr;
          uint32_t A[32], B[32];
          qjl_tc::ld32(tb + i0, A);
          qjl_tc::ld32(tb + 128u + i0, B);
          qjl_tc::wait_ld();
          sweep32(A, B, sG + i0, sG + 128 + i0, sG + kPass + 128 + i0);
          qjl_tc::st32(tb + i0, A);
          qjl_tc::st32(tb + 128u + i0, B);
        }
        qjl_tc::wait_st();
        qjl_tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xbar[quarter]);
        if (!__all_sync(0xffffffffu, mbar_wait(&xbar[quarter], u & 1u))) { flag_error(prm.err, 16); break; }
        qjl_tc::fence_after();
        // this warp's 128 outputs: columns 128 part .. 128 part + 127, formed by the sweep
        uint32_t R[128];
#pragma unroll
        for (int j = 0; j < 4; ++j) qjl_tc::ld32(tb + 128u * part + 32u * j, R + 32 * j);
        qjl_tc::wait_ld();
        release_tmem(&tempty[buf], lane);
        float2 V[64];
#pragma unroll
        for (int q = 0; q < 64; ++q) V[q] = as_f2(R[2 * q], R[2 * q + 1]);
        fwht(V);
        uint32_t w[4];
        sign_words(V, w);
        if (row < prm.n) qjl_hint::st_v4(prm.bits + row * (int64_t)prm.W + 8 * pass + 4 * part, w[0], w[1], w[2], w[3], pol);
      } else {
        // One block of 128 in columns 128 part ..: output half h is the 64-point transform of
        // v_h,i = g_i u'_i + (+-1)[h] g_{i+64} u'_{i+64}, i < 64. This warp reads the whole
        // block, 16 column pairs (i, i + 64) at a time, and forms its half.
        const uint32_t cb = tb + 128u * (uint32_t)part;
        const float* g_lo = sG + 128 * part;
        const float* g_hi = sG + kPass * half + 128 * part + 64;  // (+-1)[h] g_{i+64}
        float2 V[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t A[16], B[16];
          qjl_tc::ld16(cb + 16u * c, A);
          qjl_tc::ld16(cb + 64u + 16u * c, B);
          qjl_tc::wait_ld();
#pragma unroll
          for (int k = 0; k < 16; k += 4) {
            const float4 gl = *reinterpret_cast<const float4*>(g_lo + 16 * c + k);
            const float4 gh = *reinterpret_cast<const float4*>(g_hi + 16 * c + k);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = k + 2 * e;
              const float2 a = as_f2(A[j], A[j + 1]), b = as_f2(B[j], B[j + 1]);
              float2 p = b, v = a;
              mulz2(p, e ? make_float2(gh.z, gh.w) : make_float2(gh.x, gh.y));
              fma2(v, e ? make_float2(gl.z, gl.w) : make_float2(gl.x, gl.y), p);
              V[8 * c + j / 2] = v;
            }
          }
        }
        release_tmem(&tempty[buf], lane);

        fwht(V);
        if constexpr (DITHER) {
          // sigma of the unnormalised transform: sqrt(d) sigma_rel ||x|| (||S1 x|| = sqrt(d) ||x||),
          // with ||x||^2 from the norm warps
          if (!__all_sync(0xffffffffu, mbar_wait(&nfull[buf], (u >> 1) & 1u))) { flag_error(prm.err, 16); break; }
          const float x2 = sNrm[buf * BM + r];
          __syncwarp();
          if (lane == 0) mbar_arrive(&nempty[buf]);
          const float amp = prm.sigma * sqrtf((float)D * x2);
          if (amp != 0.f)
            add_dither(V, (uint32_t)(kPass * pass + 128 * part + 64 * half), prm.first_token + (uint64_t)row, amp,
                       prm.rk);
        }
        uint32_t w[2];
        sign_words(V, w);
        if (row < prm.n)
          qjl_hint::st_v2(prm.bits + row * (int64_t)prm.W + 8 * pass + 4 * part + 2 * half, w[0], w[1], pol);
      }
    }
  }
  qjl_tc::fence_before();
  __syncthreads();
  qjl_tc::fence_after();
  if (warp == 1) qjl_tc::dealloc(tmem_base, kTmemCols);
}

size_t smem_bytes(int d, int ns) {
  return 1024 + (size_t)(d / 64) * kPass * 128 + (size_t)ns * kSlotBytes + 2 * kPass * 4 + 2 * BM * 4 +
         (2 * ns + 14) * 8 + 16;
}

int pick_slots(int d) {
  for (int ns = 8; ns >= 3; --ns)
    if (smem_bytes(d, ns) <= kSmemLimit) return ns;
  return 0;
}

}  // namespace

bool fqjl_tc_shape(int d, int m, bool dg_outer) {
  return (d == 128 || d == 256) && m % kPass == 0 && !dg_outer && pick_slots(d) > 0;
}

// S1 [m][d] as bf16 bit patterns: row b d + i is row pi_b(i) of H, column c times D_r^b[c];
// H[p][c] = (-1)^popcount(p & c) (Sylvester order).
std::vector<uint16_t> fqjl_tc_matrix(int d, int m, const float* D_r, const int32_t* perm) {
  std::vector<uint16_t> s1((size_t)m * d);
  for (int b = 0; b < m / d; ++b)
    for (int i = 0; i < d; ++i) {
      const int p = perm[(size_t)b * d + i];
      uint16_t* row = s1.data() + ((size_t)b * d + i) * d;
      for (int c = 0; c < d; ++c) {
        const bool neg = (__builtin_popcount((unsigned)(p & c)) & 1) != (D_r[(size_t)b * d + c] < 0.f);
        row[c] = neg ? 0xBF80u : 0x3F80u;
      }
    }
  return s1;
}

void fqjl_tc_prepare(qjl_projection* P) {
  P->s_map_ok = P->S1_bf16 && qjl_make_bf16_map(P->s_map, P->S1_bf16, (uint64_t)P->m, (uint64_t)P->d,
                                                (uint64_t)P->d, (uint32_t)kPass);
}

bool fqjl_tc_supported(const qjl_projection* P, int dtype, int64_t n) {
  // the D-FQJL dither runs here for d = 128 only
  const bool dither = P->kind == QJL_DFQJL && P->dither_sigma != 0.f;
  return P->kind != QJL_DENSE && (!dither || P->d == 128) && P->S1_bf16 && P->s_map_ok && dtype == QJL_BF16 &&
         fqjl_tc_shape(P->d, P->m, P->opt.dg_outer != 0) && n <= (int64_t)INT32_MAX - BM;
}

qjl_status launch_fqjl_tc(const qjl_projection* P, const void* keys, int64_t n, int64_t ld, uint64_t first_token,
                          uint32_t* bits, float* norms, cudaStream_t st) {
  if (n <= 0) return QJL_OK;
  // the keys' map is cached per thread for the last (pointer, rows, ld, d), as in the dense sketch
  struct KeyMapCache {
    const void* ptr = nullptr;
    int64_t n = -1, ld = -1;
    int d = -1;
    alignas(64) unsigned char map[128];
  };
  static thread_local KeyMapCache kc;
  if (kc.ptr != keys || kc.n != n || kc.ld != ld || kc.d != P->d) {
    kc.ptr = nullptr;
    if (!qjl_make_bf16_map(kc.map, keys, (uint64_t)n, (uint64_t)P->d, (uint64_t)ld, BM))
      return qjl_set_error(QJL_ERR_CUDA, "cuTensorMapEncodeTiled failed for the keys");
    kc.ptr = keys;
    kc.n = n;
    kc.ld = ld;
    kc.d = P->d;
  }
  CUtensorMap tmK, tmS;
  memcpy(&tmK, kc.map, sizeof(tmK));
  memcpy(&tmS, P->s_map, sizeof(tmS));
  int* err = qjl_error_flag(P->device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  const int ns = pick_slots(P->d);
  const size_t smem = smem_bytes(P->d, ns);
  const bool dither = P->kind == QJL_DFQJL && P->dither_sigma != 0.f;
  void (*kern)(CUtensorMap, CUtensorMap, FtcParams) =
      P->d == 256 ? fqjl_tc_kernel<256, false> : (dither ? fqjl_tc_kernel<128, true> : fqjl_tc_kernel<128, false>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return qjl_check_launch("fqjl_tc_kernel smem attribute");
  // one launch: npass groups of CTAs, one per 256 coordinates, each walking all tiles
  const int npass = P->m / kPass;
  const int64_t ntiles = (n + BM - 1) / BM;
  const int64_t per = std::min<int64_t>(ntiles, std::max(1, qjl_num_sms(P->device) / npass));
  const int grid = (int)(per * npass);
  FtcParams prm{n, P->m / 32, npass, ns, P->D_g, P->dither_sigma, (uint32_t)P->seed, (uint32_t)(P->seed >> 32),
                first_token, {}, bits, norms, err};
  philox_round_keys(prm.k0, prm.k1, prm.rk);
  const int threads = P->d == 256 ? ftc_threads<256>() : ftc_threads<128>();
  if (P->d == 128) {
    // the register split asks setmaxnreg for 128 x 56 + 512 x 104 registers of the launch's pool
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return qjl_check_launch("fqjl_tc_kernel attributes");
    if (fa.numRegs < kRegsLaunch)
      return qjl_set_error(QJL_ERR_CUDA, "fqjl_tc_kernel<128> was built with fewer registers than its split needs");
  }
  qjl_log_launch("fqjl_tc_kernel", grid, threads, smem, 1);
  kern<<<grid, threads, smem, st>>>(tmK, tmS, prm);
  return qjl_check_launch("fqjl_tc_kernel");
}
