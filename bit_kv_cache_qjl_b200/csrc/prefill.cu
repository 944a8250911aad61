// Causal prefill attention over sketched keys and 2-bit values, on the
// 5th-generation tensor cores (tcgen05).
//
// At prefill every position is a query that attends to the keys at or before
// it. The scores are the QJL estimator (QJL abstract, "Majid Daliri" page)
// over the packed sign bits, the values the KIVI per-token 2-bit codes (KIVI
// abstract, "Vladimir Braverman" page):
//   out[g][i] = sum_{j <= i} softmax_j(scale * est(q_i, k_j)) * v_hat[g][j].
//
// One CTA per (key head, tile of 128 queries), longest tiles launched first.
// It walks the key axis in tiles of 128 up to its diagonal. Per key tile:
//   * S = Q . K on kind::i8: A is the tile's queries as 16-bit fixed-point Sq
//     (Q = rint(Sq * 32639 / max|Sq|) per query), split into int8 hi and lo
//     digit tiles in shared memory and built once; B is the key tile's sign
//     bits as bytes 0 or 1, in the K order of the digits (K position 4 s + e
//     of a word holds bit 8 e + s). Two MMA chains give S_hi and S_lo in
//     TMEM, exact int32 sums, and sum b Q = 256 S_hi + S_lo.
//   * softmax: four warps, thread i owns query row i. The estimate is
//     mul_i * ||k_j|| * (2 sum b Q - sum Q), in log2 units with the softmax
//     scale folded into mul_i; keys after the query (or past L) are masked.
//     A first pass over the row finds the tile's max; the running max moves
//     only when the tile's exceeds it by more than 2^8 (the output
//     accumulator is then rescaled in TMEM), so p = 2^(s - m) <= 256 stays
//     exact enough in fp16. The second pass writes p as fp16 pairs into a
//     TMEM P buffer (two, alternating) and adds it to the row sum.
//   * O += P . V on kind::f16: A is P from TMEM, B the key tile's values
//     dequantised to fp16 (code * scale + zero in one fp16 FMA, so each value
//     is the correctly rounded v_hat) and stored transposed, [channel][key],
//     in shared memory. O (fp32, 128 x 128) stays in TMEM.
// Expander warps fill the next key tile's operands (read from global memory:
// a head's keys are re-read by each of its query tiles and stay in L2) while
// the current one is in the MMAs. The MMA thread issues S(t + 1) before
// P.V(t), so the score MMAs of one tile overlap the softmax of the previous.
// Roles: warps 0-3 softmax (lane quarter = warp), warp 4 MMA (and TMEM),
// warps 5-8 expanders. Every wait is bounded; on expiry a role records an
// error bit and stops, and TMEM is freed after the MMAs drain.
//
// P and v_hat are rounded to binary16 (relative 2^-11 each); the P.V sums run
// in fp32. The score sums are exact integers; the 16-bit rounding of Sq is the
// scores' only error, as in the class tables of the decode kernels.

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "mbarrier.cuh"
#include "qjl_internal.h"
#include "tcgen05.cuh"

namespace {

using namespace qjl_sync;

constexpr int kT = 128;              // queries per CTA, keys per tile
constexpr int kW = 8;                // sign words per key (m = 256)
constexpr int kM = 32 * kW;
constexpr int kD = 128;              // head dim
constexpr int kCW = kD / 16;         // code words per token
constexpr int kGW = kD / 32;         // scale / zero halves per token
constexpr int kSoftWarps = 4;
constexpr int kExpWarps = 4;
constexpr int kMmaWarp = kSoftWarps;
constexpr int kThreads = (kSoftWarps + 1 + kExpWarps) * 32;
constexpr int kQmax = 32639;
constexpr float kTau = 8.f;          // lazy rescale threshold, log2 units

// TMEM columns
constexpr uint32_t kColShi = 0, kColSlo = 128, kColO = 256, kColP = 384;  // P: two buffers of 64
constexpr uint32_t kTmemCols = 512;

// shared memory (bytes, 1024-aligned base)
constexpr uint32_t kAbytes = kT * kM;            // one digit tile (hi or lo): 32 KB
constexpr uint32_t kKbytes = kT * kM;            // key bits as bytes: 32 KB
constexpr uint32_t kVbytes = kD * kT * 2;        // V^T fp16: 32 KB
constexpr uint32_t kOffAhi = 0;
constexpr uint32_t kOffAlo = kOffAhi + kAbytes;
constexpr uint32_t kOffK = kOffAlo + kAbytes;            // [2]
constexpr uint32_t kOffV = kOffK + 2 * kKbytes;          // [2]
constexpr uint32_t kOffNorm = kOffV + 2 * kVbytes;       // [2][128] fp32
constexpr uint32_t kOffBar = kOffNorm + 2 * kT * 4;
constexpr uint32_t kSmemBytes = kOffBar + 16 * 8 + 16 + 1024;  // barriers, TMEM holder, alignment slack

struct PrefillParams {
  const uint32_t* bits;
  const float* norms;
  const uint32_t* codes;
  const uint16_t* scale;
  const uint16_t* zero;
  const float* sq;
  float* out;
  int* err;
  int64_t G, L, nqt;
  float est_scale, logit_scale;   // logit_scale = softmax scale * log2(e)
};

// idesc kind::i8: A s8 (query digits), B u8 (key bits), D s32, M = N = 128
constexpr uint32_t kIdescS = (2u << 4) | (1u << 7) | (0u << 10) | ((uint32_t)(kT >> 3) << 17) |
                             ((uint32_t)(kT >> 4) << 24);
// idesc kind::f16: A and B fp16, D fp32, M = 128, N = 128 channels
constexpr uint32_t kIdescPV = (1u << 4) | ((uint32_t)(kD >> 3) << 17) | ((uint32_t)(kT >> 4) << 24);

__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// 16 consecutive columns of this thread's lane
__device__ __forceinline__ void st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]));
}

// Query row r of the tile (thread r of the softmax warps): its Sq row quantised to the
// 16-bit grid, written as hi and lo digits into the A tiles (row r, K order of the key
// bytes), and the row's constants. A row past L is zero.
__device__ __forceinline__ void build_query_row(const float* __restrict__ sqrow, bool valid, unsigned char* Ahi,
                                                unsigned char* Alo, float est_scale, float logit_scale, int r,
                                                float& mul, int& qsum) {
  float mx = 0.f;
  if (valid) {
#pragma unroll 8
    for (int i = 0; i < kM; i += 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(sqrow + i));
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
  }
  const float inv = mx > 0.f ? (float)kQmax / mx : 0.f;
  int qs = 0;
#pragma unroll 1
  for (int w = 0; w < kW; ++w) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 x = valid ? __ldg(reinterpret_cast<const float4*>(sqrow + 32 * w + i)) : make_float4(0, 0, 0, 0);
      v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
    }
    unsigned char* sh = Ahi + (size_t)w * kT * 32;
    unsigned char* sl = Alo + (size_t)w * kT * 32;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      uint32_t hi = 0u, lo = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int Q = (int)fminf(fmaxf(rintf(v[8 * e + s] * inv), (float)-kQmax), (float)kQmax);
        qs += Q;
        const int l = (int)(int8_t)(Q & 0xFF);
        hi |= ((uint32_t)((Q - l) >> 8) & 0xFFu) << (8 * e);
        lo |= ((uint32_t)l & 0xFFu) << (8 * e);
      }
      *reinterpret_cast<uint32_t*>(sh + qjl_tc::kmajor_ofs(r, 4 * s)) = hi;
      *reinterpret_cast<uint32_t*>(sl + qjl_tc::kmajor_ofs(r, 4 * s)) = lo;
    }
  }
  qsum = qs;
  mul = est_scale * (mx > 0.f ? mx / (float)kQmax : 0.f) * logit_scale;
}

__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const PrefillParams P) {
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_dyn + 1023) & ~(uintptr_t)1023);
  unsigned char* Ahi = base + kOffAhi;
  unsigned char* Alo = base + kOffAlo;
  unsigned char* Kb = base + kOffK;                       // [2][kKbytes]
  unsigned char* Vb = base + kOffV;                       // [2][kVbytes]
  float* snorm = reinterpret_cast<float*>(base + kOffNorm);  // [2][kT]
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffBar);
  uint64_t* kready = bars;       // [2] expander warps: key tile operands written
  uint64_t* kfree = bars + 2;    // [2] commit: the MMAs that read them are done
  uint64_t* sfull = bars + 4;    // commit: S_hi, S_lo of the current tile
  uint64_t* sfree = bars + 5;    // softmax warps: S read
  uint64_t* pfull = bars + 6;    // [2] softmax warps: P written
  uint64_t* pfree = bars + 8;    // [2] commit: the P.V that read P (and updated O) is done
  uint64_t* aready = bars + 10;  // softmax warps: the query digit tiles are built
  uint64_t* ofull = bars + 11;   // commit: every MMA is done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // longest tiles first: items walk the query tiles from the last one down
  const int64_t item = blockIdx.x;
  const int64_t qt = P.nqt - 1 - item / P.G;
  const int64_t g = item % P.G;
  const int64_t q0 = qt * kT;
  const int nkt = (int)qt + 1;  // key tiles 0 .. qt; tile qt holds the diagonal
  const int64_t L = P.L;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&kready[b], kExpWarps);
      mbar_init(&kfree[b], 1);
      mbar_init(&pfull[b], kSoftWarps);
      mbar_init(&pfree[b], 1);
    }
    mbar_init(sfull, 1);
    mbar_init(sfree, kSoftWarps);
    mbar_init(aready, kSoftWarps);
    mbar_init(ofull, 1);
    mbar_fence_init();
  }
  if (warp == kMmaWarp) qjl_tc::alloc(tmem_holder, kTmemCols);
  qjl_tc::fence_before();
  __syncthreads();
  qjl_tc::fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < kSoftWarps) {
    // ---------------- softmax: thread r owns query row r (TMEM lane r)
    const int r = threadIdx.x;
    const int64_t qi = q0 + r;  // this row's position
    const bool qvalid = qi < L;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float mul;
    int qsum;
    build_query_row(P.sq + (g * L + (qvalid ? qi : 0)) * kM, qvalid, Ahi, Alo, P.est_scale, P.logit_scale, r, mul,
                    qsum);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(aready);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int kt = 0; kt < nkt && ok; ++kt) {
      const int kb = kt & 1, pb = kt & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(sfull, (uint32_t)(kt & 1)))) { atomicOr(P.err, 16); ok = false; break; }
      // the expanders' norms for this tile (already complete: orders their writes before our reads)
      if (!__all_sync(0xffffffffu, mbar_wait(&kready[kb], (uint32_t)((kt >> 1) & 1)))) { atomicOr(P.err, 16); ok = false; break; }
      qjl_tc::fence_after();
      const float* nb = snorm + kb * kT;
      const int64_t k0 = (int64_t)kt * kT;
      // key j of the tile is visible to this row iff k0 + j <= qi and k0 + j < L; only the last
      // tile (the diagonal one, the only one that can reach past L) needs the check
      const int64_t jmax = min(qi, L - 1) - k0;  // last visible j (< 0: none)
      const bool masked = kt == nkt - 1;
      // one pass over the row: the scores, their max, and (unless the max must be found first)
      // p = 2^(s - m) against the running max, written as fp16 pairs into P buffer pb
      auto pass = [&](auto mask_c, auto write_c, float mref, float& mt, float& lt) {
        constexpr bool MASK = decltype(mask_c)::value;
        constexpr bool WRITE = decltype(write_c)::value;
#pragma unroll 1
        for (int ch = 0; ch < kT / 32; ++ch) {
          uint32_t hi[32], lo[32];
          qjl_tc::ld32(tmem + lane_off + kColShi + 32 * ch, hi);
          qjl_tc::ld32(tmem + lane_off + kColSlo + 32 * ch, lo);
          qjl_tc::wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int jj = 0; jj < 32; jj += 2) {
            float p2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int j = 32 * ch + jj + u;
              const int t = 2 * ((int)hi[jj + u] * 256 + (int)lo[jj + u]) - qsum;
              float sc = mul * nb[j] * (float)t;
              if (MASK && j > jmax) sc = -INFINITY;
              mt = fmaxf(mt, sc);
              p2[u] = WRITE ? exp2f(sc - mref) : 0.f;
              lt += p2[u];
            }
            if (WRITE) {
              const __half2 h = __floats2half2_rn(p2[0], p2[1]);
              pk[jj / 2] = *reinterpret_cast<const uint32_t*>(&h);
            }
          }
          if (WRITE) st16(tmem + lane_off + kColP + 64 * pb + 16 * ch, pk);
        }
      };
      // P buffer pb is free once the P.V two tiles back has read it
      if (!__all_sync(0xffffffffu, mbar_wait(&pfree[pb], (uint32_t)(((kt >> 1) & 1) ^ 1))))
        { atomicOr(P.err, 16); ok = false; break; }
      qjl_tc::fence_after();
      const bool fresh = __any_sync(0xffffffffu, m_run == -INFINITY);  // the first visible tile
      float mt = -INFINITY, lt = 0.f;
      if (fresh) {
        if (masked) pass(std::true_type(), std::false_type(), 0.f, mt, lt);
        else pass(std::false_type(), std::false_type(), 0.f, mt, lt);
      } else {
        if (masked) pass(std::true_type(), std::true_type(), m_run, mt, lt);
        else pass(std::false_type(), std::true_type(), m_run, mt, lt);
      }
      // ---- lazy rescale: a row's running max moves only when the tile's exceeds it by more than
      // 2^kTau (or on its first visible key). Rows decide on their own; the O rescale in TMEM is
      // warp-wide (tcgen05.ld / st are warp-collective), with factor 1 for rows that keep their max.
      const bool move = (mt > m_run + kTau) || (m_run == -INFINITY && mt != -INFINITY);
      const bool scale_o = move && m_run != -INFINITY;  // this row's O holds earlier tiles
      float f = 1.f;
      if (move) {
        if (scale_o) f = exp2f(m_run - mt);
        m_run = mt;
      }
      if (__any_sync(0xffffffffu, scale_o)) {
        // O holds P.V of tiles < kt: wait for the last of them, then scale the rows in TMEM
        const int pt = kt - 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&pfree[pt & 1], (uint32_t)((pt >> 1) & 1))))
          { atomicOr(P.err, 16); ok = false; break; }
        qjl_tc::fence_after();
#pragma unroll 1
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t o[32];
          qjl_tc::ld32(tmem + lane_off + kColO + 32 * ch, o);
          qjl_tc::wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
          qjl_tc::st32(tmem + lane_off + kColO + 32 * ch, o);
        }
      }
      if (fresh || __any_sync(0xffffffffu, move)) {
        // p against the final max (rows that kept theirs get the same values again); the first
        // pass's P stores complete before these overwrite them
        qjl_tc::wait_st();
        const float mref = m_run == -INFINITY ? 0.f : m_run;
        float mt2 = -INFINITY;
        lt = 0.f;
        if (masked) pass(std::true_type(), std::true_type(), mref, mt2, lt);
        else pass(std::false_type(), std::true_type(), mref, mt2, lt);
      }
      l_run = l_run * f + lt;
      qjl_tc::wait_st();
      qjl_tc::fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sfree);
        mbar_arrive(&pfull[pb]);
      }
    }
    // ---------------- output: O / l for this row
    if (ok && __all_sync(0xffffffffu, mbar_wait(ofull, 0))) {
      qjl_tc::fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      float* orow = P.out + (g * L + qi) * kD;
#pragma unroll 1
      for (int ch = 0; ch < kD / 32; ++ch) {
        uint32_t o[32];
        qjl_tc::ld32(tmem + lane_off + kColO + 32 * ch, o);
        qjl_tc::wait_ld();
        if (qvalid) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(orow + 32 * ch + c) =
                make_float4(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv,
                            __uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
        }
      }
    } else if (ok) {
      atomicOr(P.err, 16);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer: S(t) then P.V(t - 1)
    if (lane == 0) {
      bool ok = mbar_wait(aready, 0);
      if (!ok) atomicOr(P.err, 8);
      const uint32_t ahi = smem_u32(Ahi), alo = smem_u32(Alo);
      auto pv = [&](int t) -> bool {
        const int pb = t & 1;
        if (!mbar_wait(&pfull[pb], (uint32_t)((t >> 1) & 1))) { atomicOr(P.err, 8); return false; }
        qjl_tc::fence_after();
        const uint32_t vb = smem_u32(Vb + (size_t)(t & 1) * kVbytes);
#pragma unroll
        for (int k = 0; k < kT / 16; ++k)
          mma_f16_ts(tmem + kColO, tmem + kColP + 64 * pb + 8 * k, qjl_tc::kmajor_desc(vb + k * kD * 32), kIdescPV,
                     (t > 0 || k > 0) ? 1u : 0u);
        qjl_tc::commit(&pfree[pb]);
        qjl_tc::commit(&kfree[t & 1]);
        return true;
      };
      for (int kt = 0; kt < nkt && ok; ++kt) {
        const int kb = kt & 1;
        if (!mbar_wait(&kready[kb], (uint32_t)((kt >> 1) & 1))) { atomicOr(P.err, 8); ok = false; break; }
        if (!mbar_wait(sfree, (uint32_t)((kt & 1) ^ 1))) { atomicOr(P.err, 8); ok = false; break; }
        qjl_tc::fence_after();
        const uint32_t kbs = smem_u32(Kb + (size_t)kb * kKbytes);
#pragma unroll
        for (int w = 0; w < kW; ++w)
          mma_i8_ss(tmem + kColShi, qjl_tc::kmajor_desc(ahi + w * kT * 32), qjl_tc::kmajor_desc(kbs + w * kT * 32),
                    kIdescS, w > 0 ? 1u : 0u);
#pragma unroll
        for (int w = 0; w < kW; ++w)
          mma_i8_ss(tmem + kColSlo, qjl_tc::kmajor_desc(alo + w * kT * 32), qjl_tc::kmajor_desc(kbs + w * kT * 32),
                    kIdescS, w > 0 ? 1u : 0u);
        qjl_tc::commit(sfull);
        if (kt > 0 && !pv(kt - 1)) { ok = false; break; }
      }
      if (ok) ok = pv(nkt - 1);
      qjl_tc::commit(ofull);
      // every MMA has completed before TMEM is freed
      if (!mbar_wait(ofull, 0)) atomicOr(P.err, 8);
    }
  } else {
    // ---------------- expanders: thread r builds key row r of each tile's operands
    const int r = threadIdx.x - (kSoftWarps + 1) * 32;
    for (int kt = 0; kt < nkt; ++kt) {
      const int kb = kt & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&kfree[kb], (uint32_t)(((kt >> 1) & 1) ^ 1)))) { atomicOr(P.err, 4); break; }
      const int64_t j = (int64_t)kt * kT + r;
      const bool valid = j < L;
      const int64_t row = g * L + (valid ? j : 0);
      // sign bits -> bytes 0/1: column s of word w holds bits 8 e + s (K positions 4 s + e)
      uint4 b0 = make_uint4(0, 0, 0, 0), b1 = b0;
      if (valid) {
        b0 = __ldg(reinterpret_cast<const uint4*>(P.bits + row * kW));
        b1 = __ldg(reinterpret_cast<const uint4*>(P.bits + row * kW) + 1);
      }
      const uint32_t words[kW] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      unsigned char* kt_s = Kb + (size_t)kb * kKbytes;
#pragma unroll
      for (int w = 0; w < kW; ++w) {
        uint32_t a[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) a[s] = (words[w] >> s) & 0x01010101u;
        unsigned char* sl = kt_s + w * kT * 32;
        *reinterpret_cast<uint4*>(sl + qjl_tc::kmajor_ofs(r, 0)) = make_uint4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<uint4*>(sl + qjl_tc::kmajor_ofs(r, 16)) = make_uint4(a[4], a[5], a[6], a[7]);
      }
      snorm[kb * kT + r] = valid ? __ldg(P.norms + row) : 0.f;
      // values: v_hat = code * scale + zero in one fp16 FMA, stored as V^T [channel][key] in 32-byte K slices
      uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0;
      __half sc[kGW], zr[kGW];
#pragma unroll
      for (int q = 0; q < kGW; ++q) {
        sc[q] = __ushort_as_half(valid ? __ldg(P.scale + row * kGW + q) : (uint16_t)0);
        zr[q] = __ushort_as_half(valid ? __ldg(P.zero + row * kGW + q) : (uint16_t)0);
      }
      if (valid) {
        c0 = __ldg(reinterpret_cast<const uint4*>(P.codes + row * kCW));
        c1 = __ldg(reinterpret_cast<const uint4*>(P.codes + row * kCW) + 1);
      }
      const uint32_t cw[kCW] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      unsigned char* vs = Vb + (size_t)kb * kVbytes + (r >> 4) * (kD * 32);  // the K slice of this key
      const int kbyte = 2 * (r & 15);
      // channels c and c + 8 share a code word and a scale group: one shift and one mask-or give
      // the fp16 pair (1024 + code_c, 1024 + code_c+8), an exact subtract leaves the codes, and one
      // fp16x2 FMA forms both code * scale + zero with a single rounding each
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        const __half2 s2 = __half2half2(sc[w >> 1]), z2 = __half2half2(zr[w >> 1]);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t x = ((cw[w] >> (2 * k)) & 0x00030003u) | 0x64006400u;
          const __half2 v = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&x), __float2half2_rn(1024.f)), s2, z2);
          *reinterpret_cast<__half*>(vs + qjl_tc::kmajor_ofs(16 * w + k, kbyte)) = __low2half(v);
          *reinterpret_cast<__half*>(vs + qjl_tc::kmajor_ofs(16 * w + k + 8, kbyte)) = __high2half(v);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&kready[kb]);
    }
  }
  qjl_tc::fence_before();
  __syncthreads();
  qjl_tc::fence_after();
  if (warp == kMmaWarp) qjl_tc::dealloc(tmem, kTmemCols);
}

qjl_status launch_prefill_tc(const qjl_projection* Pj, const uint32_t* bits, const float* norms, const uint32_t* codes,
                             const uint16_t* scale, const uint16_t* zero, int64_t G, int64_t L, const float* sq,
                             float softmax_scale, float* out, cudaStream_t st) {
  int* err = qjl_error_flag(Pj->device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  const int64_t nqt = (L + kT - 1) / kT;
  if (G * nqt > ((int64_t)1 << 31) - 1) return qjl_set_error(QJL_ERR_UNSUPPORTED, "too many query tiles");
  if (cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
      cudaSuccess)
    return qjl_check_launch("prefill_tc_kernel smem attribute");
  PrefillParams prm{bits, norms, codes, scale, zero, sq, out, err, G, L, nqt, Pj->est_scale,
                    softmax_scale * 1.4426950408889634f};
  qjl_log_launch("prefill_tc_kernel", G * nqt, kThreads, kSmemBytes, 1);
  prefill_tc_kernel<<<(unsigned)(G * nqt), kThreads, kSmemBytes, st>>>(prm);
  return qjl_check_launch("prefill_tc_kernel");
}

}  // namespace

extern "C" qjl_status qjl_prefill_attention(const qjl_projection* P, const uint32_t* bits, const float* norms,
                                            const uint32_t* codes, const uint16_t* scale, const uint16_t* zero,
                                            int64_t groups, int64_t L, const float* sq, float softmax_scale,
                                            float* out, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (groups < 0 || L < 0 || groups > (1 << 20) || L > (1 << 24))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "groups/L out of range");
  if (!isfinite(softmax_scale)) return qjl_set_error(QJL_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (P->d != kD || P->m != kM)
    return qjl_set_error(QJL_ERR_UNSUPPORTED, "prefill attention supports d = 128 and m = 256");
  if (groups == 0 || L == 0) return QJL_OK;
  if (!bits || !norms || !codes || !scale || !zero || !sq || !out) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(bits) || !aligned16(codes) || !aligned16(sq) || !aligned16(out) || ((uintptr_t)norms & 3u) ||
      ((uintptr_t)scale & 1u) || ((uintptr_t)zero & 1u))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "bits, codes, sq and out must be 16-byte aligned; norms, scale, zero naturally");
  DeviceGuard gd(P->device);
  if (!gd.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  return launch_prefill_tc(P, bits, norms, codes, scale, zero, groups, L, sq, softmax_scale, out,
                           (cudaStream_t)stream);
}
