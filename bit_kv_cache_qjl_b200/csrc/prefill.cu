// Causal prefill attention over sketched keys and 2-bit values.
//
// At prefill every position is a query that attends to the keys at or before
// it. The scores are the QJL estimator (QJL abstract, "Majid Daliri" page)
// over the packed sign bits, the values the KIVI per-token 2-bit codes (KIVI
// abstract, "Vladimir Braverman" page):
//   out[g][i] = sum_{j <= i} softmax_j(scale * est(q_i, k_j)) * v_hat[g][j].
//
// One warp per 16 consecutive queries of a key head, four warps (64 queries)
// per CTA. The warps walk the key axis in 16-key steps, each up to its own
// diagonal; the CTA dequantises each step's value tile once for all four.
// At under 170 registers and 73 KB of shared memory three CTAs (12 warps) fit
// on an SM.
// Per warp and step:
//   * scores: shift-window sign sums (build_tables_dig) on the u8 x s8
//     mma.sync, two queries per n8 column tile, so 8 column tiles cover the
//     warp's 16 queries; then the causal and length masks;
//   * an online base-2 softmax: a lane keeps the running max of the eight
//     queries whose scores it holds, and its share of their sums; the
//     rescale factors reach the lanes holding the output rows through
//     shared memory;
//   * P . V on the fp16 tensor-core path (mma.sync m16n8k16, fp32
//     accumulate). P goes through shared memory to ldmatrix as the A
//     fragment; the step's 16 values are dequantised to fp16
//     (code * scale + zero, packed half2 arithmetic) into a shared tile, one code word
//     per thread of the CTA, and read with ldmatrix.trans as the B fragments of
//     16 channel tiles. Each step's key and value data is loaded one step
//     ahead. (Dequantising the values once into an fp16 workspace
//     and streaming tiles of it with cp.async measured slower: 3.35 against
//     3.01 ms for 32 heads x 4096 tokens.)
// P and v_hat are rounded to binary16 (relative 2^-11 each); the sums run in
// fp32. Key data is re-read by every later query tile of the head, so it is
// read straight from global memory and served by L2.

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "qjl_internal.h"
#include "sign_mma.cuh"

namespace {

using namespace qjl_sign;

constexpr int kQ = 16;          // queries per warp (CTA)
constexpr int kWs = 8;          // sign words per key (m = 256)
constexpr int kD = 128;         // head dim
constexpr int kNT = kQ / 2;     // digit column tiles
constexpr int kPS = 24;         // P tile row stride (halves): 48 bytes, 16-byte aligned rows
constexpr int kVS = kD + 8;     // V tile row stride (halves): 272 bytes

constexpr int kWarps = 4;       // warps per CTA: 64 consecutive queries share each value tile

struct WarpSmem {
  uint4 btab[kNT * kWs * 16];  // two shifts' B fragments per lane and entry
  float s_inv[kQ], s_mul[kQ];  // s_mul: then times log2(e) * softmax scale
  int s_qsum[kQ];
  float xq[kQ];  // per-query exchange: the step's rescale factors, then the final sums
  __align__(16) __half P[kQ * kPS];
};

struct PrefillSmem {
  WarpSmem w[kWarps];
  __align__(16) __half V[16 * kVS];  // the step's value tile, shared by the warps
};

__device__ __forceinline__ void ldm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

__device__ __forceinline__ void ldm_x2_trans(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

// d = a . b with a zero accumulator input
__device__ __forceinline__ void mma_u8s8_first(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// 2^x on the special-function unit (PTX ex2.approx.ftz: about 2^-22 relative error, 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__global__ void __launch_bounds__(kWarps * 32, 3) prefill_kernel(const uint32_t* __restrict__ bits,
                                                              const float* __restrict__ norms,
                                                              const uint32_t* __restrict__ codes,
                                                              const uint16_t* __restrict__ scale,
                                                              const uint16_t* __restrict__ zero,
                                                              const float* __restrict__ sq, int64_t G, int64_t L,
                                                              float est_scale, float logit2, float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PrefillSmem& SM = *reinterpret_cast<PrefillSmem*>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  WarpSmem& S = SM.w[warp];
  constexpr int kCQ = kWarps * kQ;
  const int64_t nqt = (L + kCQ - 1) / kCQ;
  // the heaviest query tiles (late in the sequence) first
  const int64_t tile = (nqt - 1) - (int64_t)(blockIdx.x / G);
  const int64_t g = (int64_t)(blockIdx.x % G);
  const int64_t q0c = tile * kCQ;
  const int64_t q0 = q0c + kQ * warp;                        // this warp's first query
  const int nq = (int)max((int64_t)0, min((int64_t)kQ, L - q0));
  // the CTA's key steps run to its last warp with queries
  const int64_t wl = min((int64_t)(kWarps - 1), (L - 1 - q0c) / kQ);
  const int ktiles_cta = (int)((q0c + kQ * wl) / 16 + 1);
  const int ktiles = nq > 0 ? (int)(q0 / 16 + 1) : 0;    // this warp's steps: up to its diagonal

  // every warp's tables, each built by the whole CTA
  for (int w = 0; w < kWarps; ++w) {
    const int64_t qw = q0c + kQ * w;
    const int nw = (int)max((int64_t)0, min((int64_t)kQ, L - qw));
    build_tables_dig<kWs, true>(sq + (g * L + min(qw, L - 1)) * (32 * kWs), nw, kNT, false, est_scale,
                                SM.w[w].s_inv, SM.w[w].s_mul, SM.w[w].s_qsum,
                                reinterpret_cast<uint2*>(SM.w[w].btab), kWarps, 0);
  }
  if (lane < kQ) S.s_mul[lane] *= logit2;
  __syncwarp();

  const int gq = lane >> 2, q = lane & 3, par = q & 1, half = q >> 1;
  const uint32_t hm = par ? 65536u : 1u;
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[n][j] = 0.f;
  // the lane's eight queries 2 ct + half: running max (the same in all 16 lanes of the query) and
  // this lane's share of the running sum
  float m_own[kNT], l_part[kNT];
#pragma unroll
  for (int ct = 0; ct < kNT; ++ct) {
    m_own[ct] = -INFINITY;
    l_part[ct] = 0.f;
  }
  // the sign words and norm of a 16-key step, loaded one step ahead (this lane's words of key rows
  // gq and gq + 8, and the norm of its key row kr), and this thread's share of the value tile: key
  // t / 8, code word t % 8 (16 channels) with its scale and zero
  struct StepData {
    uint2 wa, wb;
    float nrm;
  };
  struct ValData {
    uint32_t cw;
    uint16_t s, z;
  };
  const int kr = gq + 8 * par;
  const int vk = threadIdx.x >> 3, vw = threadIdx.x & 7;
  // 32-bit offsets from this group's and lane's first element (L <= 2^24)
  const int Li = (int)L;
  const uint2* bits_l = reinterpret_cast<const uint2*>(bits + (g * L + gq) * kWs + 2 * q);
  const float* norms_l = norms + g * L + kr;
  const uint32_t* codes_l = codes + (g * L + vk) * (kD / 16) + vw;
  const uint16_t* scale_l = scale + (g * L + vk) * (kD / 32) + (vw >> 1);
  const uint16_t* zero_l = zero + (g * L + vk) * (kD / 32) + (vw >> 1);
  auto load_step = [&](int k0, StepData& sd) {
    sd.wa = k0 + gq < Li ? __ldg(bits_l + k0 * (kWs / 2)) : make_uint2(0, 0);
    sd.wb = k0 + gq + 8 < Li ? __ldg(bits_l + (k0 + 8) * (kWs / 2)) : make_uint2(0, 0);
    sd.nrm = k0 + kr < Li ? __ldg(norms_l + k0) : 0.f;
  };
  auto load_val = [&](int k0, ValData& vd) {
    if (k0 + vk < Li) {
      vd.cw = __ldg(codes_l + k0 * (kD / 16));
      vd.s = __ldg(scale_l + k0 * (kD / 32));
      vd.z = __ldg(zero_l + k0 * (kD / 32));
    } else {
      vd.cw = 0u;  // past the last token: zero values (P is 0 there)
      vd.s = vd.z = 0;
    }
  };
  StepData cur, nxt;
  ValData vcur, vnxt;
  if (ktiles > 0) load_step(0, cur);
  load_val(0, vcur);
  for (int kt = 0; kt < ktiles_cta; ++kt) {
    const int k0 = kt * 16;
    __half* Vt = SM.V;
    // ---- v_hat (fp16) of this thread's 16 channels 16 vw + i into the shared tile [key][position].
    // Within each 16-channel group, channels i and i + 8 sit side by side (positions 2i, 2i + 1), so
    // one shift and one mask put both codes in the halves of a word: 0x6400 | code is 1024 + code in
    // fp16, and (h - 1024) s + z is one packed subtract (exact) and one packed fused multiply-add
    // (one rounding to fp16)
    {
      const __half2 s2 = __half2half2(__ushort_as_half(vcur.s)), z2 = __half2half2(__ushort_as_half(vcur.z));
      const __half2 k1024 = __half2half2(__ushort_as_half((unsigned short)0x6400u));
      uint32_t h[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t x = ((vcur.cw >> (2 * i)) & 0x00030003u) | 0x64006400u;
        const __half2 v = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&x), k1024), s2, z2);
        h[i] = *reinterpret_cast<const uint32_t*>(&v);
      }
      uint4* dst = reinterpret_cast<uint4*>(Vt + vk * kVS + 16 * vw);
      dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
      dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
    if (kt + 1 < ktiles_cta) load_val(k0 + 16, vnxt);
    if (kt + 1 < ktiles) load_step(k0 + 16, nxt);
    // the tile is complete for every warp
    __syncthreads();
    if (kt < ktiles) {
    // ---- scores: rows g and g + 8 of the key tile, words 2q and 2q + 1
    const uint32_t w0[2] = {cur.wa.x, cur.wa.y}, w1[2] = {cur.wb.x, cur.wb.y};
    int acc[kNT][4];
#pragma unroll
    for (int sp = 0; sp < kWs / 2; ++sp) {
      // shifts 2 sp and 2 sp + 1, two column tiles at a time: one 16-byte table load per tile
#pragma unroll
      for (int cg = 0; cg < kNT; cg += 2) {
        uint4 bb[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) bb[c] = S.btab[((cg + c) * (kWs / 2) + sp) * 32 + lane];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int sh = 2 * sp + h;
          const uint32_t a0 = w0[0] >> sh, a1 = w1[0] >> sh, a2 = w0[1] >> sh, a3 = w1[1] >> sh;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (sp == 0 && h == 0)
              mma_u8s8_first(acc[cg + c], a0, a1, a2, a3, bb[c].x, bb[c].y);
            else
              mma_u8s8(acc[cg + c], a0, a1, a2, a3, h ? bb[c].z : bb[c].x, h ? bb[c].w : bb[c].y);
          }
        }
      }
    }
    // lane (gq, q) completes key kr = gq + 8 par for query 2 ct + half of each column tile
    // key kr's offset from the warp's first query; query jq sees it when rel <= jq < nq (which also
    // keeps it below L, since q0 + nq <= L)
    const int rel = k0 - (int)q0 + kr;
    const float nrm = cur.nrm;
    float xv[kNT];
#pragma unroll
    for (int ct = 0; ct < kNT; ++ct) {
      const uint32_t P0 = (uint32_t)acc[ct][0] * hm + (uint32_t)acc[ct][1] * (hm << 8);
      const uint32_t P1 = (uint32_t)acc[ct][2] * hm + (uint32_t)acc[ct][3] * (hm << 8);
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, par ? P0 : P1, 1);
      const uint32_t tot = (par ? P1 : P0) + recv;
      const int jq = 2 * ct + half;
      xv[ct] = (rel <= jq && jq < nq) ? S.s_mul[jq] * nrm * (float)(int)(2u * tot - (uint32_t)S.s_qsum[jq])
                                      : -INFINITY;
    }
    // ---- online softmax of the lane's queries: the step's max over the query's 16 key lanes
    // (lane bits 0, 2, 3, 4)
    float pv[kNT], corr[kNT];
#pragma unroll
    for (int ct = 0; ct < kNT; ++ct) {
      float v = xv[ct];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      const float mnew = fmaxf(m_own[ct], v);
      corr[ct] = mnew == -INFINITY ? 1.f : ex2(m_own[ct] - mnew);
      m_own[ct] = mnew;
      pv[ct] = (xv[ct] == -INFINITY) ? 0.f : ex2(xv[ct] - mnew);
      l_part[ct] = l_part[ct] * corr[ct] + pv[ct];
    }
    // ---- P (fp16) into shared memory as [query][key], and the queries' rescale factors
    __syncwarp();
#pragma unroll
    for (int ct = 0; ct < kNT; ++ct) S.P[(2 * ct + half) * kPS + kr] = __float2half_rn(pv[ct]);
    if ((lane & ~2) == 0) {
#pragma unroll
      for (int ct = 0; ct < kNT; ++ct) S.xq[2 * ct + half] = corr[ct];
    }
    __syncwarp();
    // rescale the accumulator rows (queries gq and gq + 8)
    {
      const float c0 = S.xq[gq], c1 = S.xq[gq + 8];
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= c0; o[n][1] *= c0;
        o[n][2] *= c1; o[n][3] *= c1;
      }
    }
    // ---- o += P . v_hat
    uint32_t afr[4];
    ldm_x4(afr, S.P + (lane & 15) * kPS + 8 * (lane >> 4));
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      uint32_t bfr[2];
      ldm_x2_trans(bfr, Vt + (lane & 15) * kVS + 8 * n);
      mma_f16(o[n], afr, bfr);
    }
    __syncwarp();
    cur = nxt;
    }
    vcur = vnxt;
    // every warp is done with the tile before the next step overwrites it
    __syncthreads();
  }
  // ---- each query's sum over its 16 key lanes (lane bits 0, 2, 3, 4), through shared memory to the
  // lanes that hold its output row
  float l_q[kNT];
#pragma unroll
  for (int ct = 0; ct < kNT; ++ct) {
    float v = l_part[ct];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    l_q[ct] = v;
  }
  __syncwarp();
  if ((lane & ~2) == 0) {
#pragma unroll
    for (int ct = 0; ct < kNT; ++ct) S.xq[2 * ct + half] = l_q[ct];
  }
  __syncwarp();
  // ---- normalise and store rows gq and gq + 8
  const float i0 = 1.f / S.xq[gq], i1 = 1.f / S.xq[gq + 8];
  // accumulator positions 8n + 2q and 8n + 2q + 1 hold channels ch and ch + 8 (the value tile's order)
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int ch = 16 * (n >> 1) + 4 * (n & 1) + q;
    if (gq < nq) {
      float* p = out + (g * L + q0 + gq) * kD + ch;
      p[0] = o[n][0] * i0;
      p[8] = o[n][1] * i0;
    }
    if (gq + 8 < nq) {
      float* p = out + (g * L + q0 + gq + 8) * kD + ch;
      p[0] = o[n][2] * i1;
      p[8] = o[n][3] * i1;
    }
  }
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
  if (P->d != kD || P->m != 32 * kWs)
    return qjl_set_error(QJL_ERR_UNSUPPORTED, "prefill attention supports d = 128 and m = 256");
  if (groups == 0 || L == 0) return QJL_OK;
  if (!bits || !norms || !codes || !scale || !zero || !sq || !out) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(bits) || !aligned16(codes) || !aligned16(sq) || !aligned16(out) || ((uintptr_t)norms & 3u) ||
      ((uintptr_t)scale & 1u) || ((uintptr_t)zero & 1u))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "bits, codes, sq and out must be 16-byte aligned; norms, scale, zero naturally");
  const int64_t nqt = (L + kWarps * kQ - 1) / (kWarps * kQ);
  if (groups * nqt > ((int64_t)1 << 31) - 1) return qjl_set_error(QJL_ERR_UNSUPPORTED, "too many query tiles");
  DeviceGuard gd(P->device);
  if (!gd.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  const size_t smem = sizeof(PrefillSmem);
  if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return qjl_check_launch("prefill_kernel smem attribute");
  prefill_kernel<<<(unsigned)(groups * nqt), kWarps * 32, smem, (cudaStream_t)stream>>>(
      bits, norms, codes, scale, zero, sq, groups, L, P->est_scale, softmax_scale * 1.4426950408889634f, out);
  return qjl_check_launch("prefill_kernel");
}
