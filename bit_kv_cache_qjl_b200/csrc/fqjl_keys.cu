// D-FQJL / P-FQJL key sketch: bits and norms by two fast Walsh-Hadamard
// transforms per block.
//
// "Fast Quantized Johnson - Lindenstrauss Transforms" ("In short", "Key
// concepts", "The paper" abstract): the dense Gaussian projection is replaced
// by two randomized Hadamard transforms with a Gaussian diagonal in the second
// stage, at O(d log d) per vector. P-FQJL puts a uniform random permutation
// between the Hadamard stages. D-FQJL adds Gaussian dither before the sign
// ("Transcript: The paper's improvements"). For block b of the m/d stacked
// blocks, with H the unnormalised Sylvester matrix:
//   y = H D_g Pi H D_r x            (default; sqrt(d) H_n D_g Pi H_n D_r x times sqrt(d))
//   y = D_g H Pi H D_r x            (dg_outer, the literal order)
// and the stored bit is [y + sqrt(d) sigma_rel ||x|| xi >= 0] (the positive
// factor sqrt(d) between y and the normalised map does not move a sign).
// The dither xi for coordinate e = b*d + i of token t comes eight coordinates
// to a Philox4x32-10 block at counter (e/8, t_lo, t_hi, 3): word w gives
// coordinates 8c + 2w and 8c + 2w + 1, the cos and sin outputs of Box-Muller
// on its two 16-bit halves.
//
// Work split. A thread holds E = min(d, 128) elements of one key in registers
// as E/2 packed pairs V[t] = (v_t, v_{t+E/2}), so most butterflies are sm_100
// packed-fp32 add/sub. L = d/E lanes share a key (1 for d <= 128, else 2, 4
// or 8), K = 32/L keys per warp, and lane s of a key holds elements
// i = s*E + r, r = 0..E-1. Butterflies on register bits need no data
// movement. Butterflies on lane bits are one shfl_xor and one packed FMA per
// pair. Each lane thus ends with E consecutive output bits, which
// funnel-shift into whole words. The P-FQJL permutation is a gather through
// a per-warp shared buffer, in which element j of key slot k sits at word
// K*(j + j/E) + k: the writes are conflict-free and the gather reads go to
// precomputed offsets.
//
// Keys reach shared memory by cp.async.bulk (the API requires 16-byte aligned
// rows), one copy per key row segment, into segments padded by 16 bytes so
// that the register loads are conflict-free. Each warp fetches its next batch
// of K keys while other warps compute, one batch in flight per warp. Per-block tables (D_r
// and D_g as register pairs, gather offsets) are staged once per CTA, with the
// lanes' segments 16 bytes apart so that they sit in different banks.
//
// No output bit can come from a -0: D_g is applied as fma(u, g, +0), which
// maps an exact zero product to +0, and sums of values that are not -0 are
// not -0. So the sign bit of y is exactly [y < 0].

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <vector>

#include "mbarrier.cuh"
#include "philox.h"
#include "key_math.cuh"
#include "cache_hint.cuh"
#include "qjl_internal.h"

namespace {

using qjl_sync::bulk_g2s;
using qjl_sync::mbar_expect_tx;
using qjl_sync::mbar_fence_init;
using qjl_sync::mbar_init;
using qjl_sync::mbar_wait;
using qjl_sync::smem_u32;
using namespace qjl_km;

constexpr int kMaxWarps = 8;
constexpr size_t kTableBudget = 24 * 1024;   // shared bytes for the per-block tables of one launch
constexpr size_t kSmemLimit = 227 * 1024;

enum { MODE_P = 0, MODE_D = 1 };

// ---- transform ----------------------------------------------------------------------------------

// Unnormalised Walsh-Hadamard transform over the d elements of each key, whatever the layout:
// register-bit stages (pairs, then within a pair), then lane-bit stages.
template <int E, int L>
__device__ __forceinline__ void fwht(float2 (&V)[E / 2], int lane) {
#pragma unroll
  for (int h = 1; h < E / 2; h <<= 1) {
#pragma unroll
    for (int t = 0; t < E / 2; ++t)
      if (!(t & h)) bfly2(V[t], V[t + h]);
  }
#pragma unroll
  for (int t = 0; t < E / 2; ++t) {
    const float a = V[t].x, b = V[t].y;
    V[t].x = a + b;
    V[t].y = a - b;
  }
#pragma unroll
  for (int g = 1; g < L; g <<= 1) {
    // lower lane: a + b = fma(+1, a, b); upper lane: a - b = fma(-1, b, a)
    const float sg = (lane & g) ? -1.f : 1.f;
#pragma unroll
    for (int t = 0; t < E / 2; ++t) {
      float2 p;
      p.x = __shfl_xor_sync(0xffffffffu, V[t].x, g);
      p.y = __shfl_xor_sync(0xffffffffu, V[t].y, g);
      sfma2(V[t], sg, p);
    }
  }
}

// ---- staging ------------------------------------------------------------------------------------

template <int E, int L, int ES>
struct Geo {
  static constexpr int K = 32 / L;                          // keys per warp
  static constexpr int SEGB = E * ES;                       // bytes of one lane's segment of a key row
  static constexpr int SEGP = SEGB + 16;                    // padded segment pitch
  static constexpr int ROWP = L * SEGP;                     // padded row pitch
  static constexpr int XBUF = K * ROWP;                     // staged keys per warp
  static constexpr int GBUF = (32 * E + 32) * 4;            // gather buffer per warp
  static constexpr int TSEG = E + 4;                        // words per lane segment of a table
  static constexpr int TBLK = 3 * L * TSEG;                 // table words per block
};

struct KeysArgs {
  const void* x;
  int64_t n, ld;
  int d, m, b0, b1;           // this launch covers blocks [b0, b1)
  const float* tab;           // device tables of all blocks, 3d words per block
  float amp_rel;              // sqrt(d) * sigma_rel (D-FQJL), else 0
  int dg_outer;
  uint32_t k0, k1;
  uint64_t first_token;
  uint32_t* bits;
  float* norms;
  int W;                      // words per key row of bits
  int* err;
  PageMap pm;                 // appends to a paged cache: row -> pool row, which also seeds the dither
};

template <int E, int L, int ES>
__device__ __forceinline__ void stage_rows(const KeysArgs& a, int64_t row0, int nvalid, unsigned char* xb,
                                           uint64_t* bar, int lane) {
  using G = Geo<E, L, ES>;
  // order this warp's earlier generic-proxy reads of the buffer before the async-proxy writes
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
  if (lane == 0) mbar_expect_tx(bar, (uint32_t)(nvalid * L * G::SEGB));
  __syncwarp();
  if (lane < nvalid * L) {
    const int k = lane / L, j = lane % L;
    const unsigned char* src = reinterpret_cast<const unsigned char*>(a.x);
    bulk_g2s(xb + k * G::ROWP + j * G::SEGP, src + ((row0 + k) * a.ld) * ES + (int64_t)j * G::SEGB, G::SEGB, bar);
  }
}

// This lane's E elements of its key, from the staged row, as register pairs.
template <int E, int L, int ES>
__device__ __forceinline__ void load_x(const unsigned char* xrow, int s, float2 (&V)[E / 2]) {
  using G = Geo<E, L, ES>;
  const unsigned char* seg = xrow + s * G::SEGP;
  if (ES == 2) {
#pragma unroll
    for (int t = 0; t < E / 2; t += 8) {
      const uint4 a = *reinterpret_cast<const uint4*>(seg + 2 * t);
      const uint4 c = *reinterpret_cast<const uint4*>(seg + 2 * (t + E / 2));
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        V[t + 2 * k].x = __uint_as_float(wa[k] << 16);
        V[t + 2 * k + 1].x = __uint_as_float(wa[k] & 0xffff0000u);
        V[t + 2 * k].y = __uint_as_float(wc[k] << 16);
        V[t + 2 * k + 1].y = __uint_as_float(wc[k] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int t = 0; t < E / 2; t += 4) {
      const float4 a = *reinterpret_cast<const float4*>(seg + 4 * t);
      const float4 c = *reinterpret_cast<const float4*>(seg + 4 * (t + E / 2));
      V[t].x = a.x; V[t + 1].x = a.y; V[t + 2].x = a.z; V[t + 3].x = a.w;
      V[t].y = c.x; V[t + 1].y = c.y; V[t + 2].y = c.z; V[t + 3].y = c.w;
    }
  }
}

// ---- kernel -------------------------------------------------------------------------------------

// PAGED: appends to a paged cache (a.pm maps rows to pool rows); otherwise rows map to themselves
template <int E, int L, int ES, int MODE, bool PAGED>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) fqjl_keys_kernel(const KeysArgs a) {
  using G = Geo<E, L, ES>;
  constexpr int K = G::K;
  constexpr bool BUF = (MODE == MODE_P);
  extern __shared__ __align__(16) unsigned char smem[];
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kp = lane / L, s = lane % L;
  const int d = a.d, nbl = a.b1 - a.b0;
  const size_t tab_bytes = (size_t)nbl * G::TBLK * 4;

  // shared layout: tables | per-warp staged keys | per-warp gather buffers | per-warp barriers
  float* tab = reinterpret_cast<float*>(smem);
  unsigned char* xb = smem + tab_bytes + (size_t)warp * G::XBUF;
  float* gb = reinterpret_cast<float*>(smem + tab_bytes + (size_t)nw * G::XBUF + (BUF ? (size_t)warp * G::GBUF : 0));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + tab_bytes + (size_t)nw * G::XBUF +
                                              (BUF ? (size_t)nw * G::GBUF : 0)) + warp;

  {
    const float4* src = reinterpret_cast<const float4*>(a.tab + (size_t)a.b0 * G::TBLK);
    float4* dst = reinterpret_cast<float4*>(tab);
    for (int i = threadIdx.x; i < nbl * G::TBLK / 4; i += blockDim.x) dst[i] = __ldg(src + i);
  }
  if (lane == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();

  // this warp's batches are q0, q0 + stride, ...; the barrier completes one phase per batch
  const int64_t nbatch = (a.n + K - 1) / K;
  const int64_t stride = (int64_t)gridDim.x * nw;
  int64_t q = (int64_t)blockIdx.x * nw + warp;
  if (q < nbatch) stage_rows<E, L, ES>(a, q * K, (int)(a.n - q * K < K ? a.n - q * K : K), xb, bar, lane);

  for (uint32_t phase = 0; q < nbatch; q += stride, phase ^= 1u) {
    const int64_t row = q * K + kp;
    // the output row (a page slot when appending to a paged cache) and the dither's token index
    const int64_t orow = row < a.n ? (PAGED ? a.pm.slot(row) : row) : -1;
    if (PAGED && row < a.n && orow < 0) atomicOr(a.err, QJL_DEVERR_PAGE);
    const bool valid = orow >= 0;
    if (!__all_sync(0xffffffffu, mbar_wait(bar, phase))) {
      // the batch never landed (the whole warp agrees): flag it, give the copy one more
      // bounded wait, and stop
      if (lane == 0) atomicExch(a.err, 1);
      mbar_wait(bar, phase);
      return;
    }
    const uint64_t tok = PAGED ? (uint64_t)orow : a.first_token + (uint64_t)row;
    float norm = 0.f;

    for (int bl = 0; bl < nbl; ++bl) {
      const int b = a.b0 + bl;
      const float* tb = tab + (size_t)bl * G::TBLK;
      float2 V[E / 2];
      load_x<E, L, ES>(xb + kp * G::ROWP, s, V);
      if (bl == 0) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < E / 2; ++t) sq_acc2(acc, V[t]);
        float ss = acc.x + acc.y;
#pragma unroll
        for (int g = 1; g < L; g <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, g);
        norm = sqrtf(ss);
      }
      // D_r, then the first transform
      {
        const float2* dr = reinterpret_cast<const float2*>(tb + s * G::TSEG);
#pragma unroll
        for (int t = 0; t < E / 2; t += 2) {
          const float4 p = *reinterpret_cast<const float4*>(dr + t);
          mul2(V[t], make_float2(p.x, p.y));
          mul2(V[t + 1], make_float2(p.z, p.w));
        }
      }
      fwht<E, L>(V, lane);
      // permutation gather: element j of key slot kp at word K*(j + j/E) + kp
      if (BUF) {
        float* wb = gb + K * s * (E + 1) + kp;
#pragma unroll
        for (int t = 0; t < E / 2; ++t) {
          wb[K * t] = V[t].x;
          wb[K * (t + E / 2)] = V[t].y;
        }
        __syncwarp();
        const int* ro = reinterpret_cast<const int*>(tb + 2 * L * G::TSEG + s * G::TSEG);
        const unsigned char* rb = reinterpret_cast<const unsigned char*>(gb + kp);
#pragma unroll
        for (int t = 0; t < E / 2; t += 4) {
          const int4 o1 = *reinterpret_cast<const int4*>(ro + t);
          const int4 o2 = *reinterpret_cast<const int4*>(ro + t + E / 2);
          V[t].x = *reinterpret_cast<const float*>(rb + o1.x);
          V[t + 1].x = *reinterpret_cast<const float*>(rb + o1.y);
          V[t + 2].x = *reinterpret_cast<const float*>(rb + o1.z);
          V[t + 3].x = *reinterpret_cast<const float*>(rb + o1.w);
          V[t].y = *reinterpret_cast<const float*>(rb + o2.x);
          V[t + 1].y = *reinterpret_cast<const float*>(rb + o2.y);
          V[t + 2].y = *reinterpret_cast<const float*>(rb + o2.z);
          V[t + 3].y = *reinterpret_cast<const float*>(rb + o2.w);
        }
        __syncwarp();
      }
      const float2* gp = reinterpret_cast<const float2*>(tb + L * G::TSEG + s * G::TSEG);
      if (!a.dg_outer) {
#pragma unroll
        for (int t = 0; t < E / 2; t += 2) {
          const float4 g = *reinterpret_cast<const float4*>(gp + t);
          mulz2(V[t], make_float2(g.x, g.y));
          mulz2(V[t + 1], make_float2(g.z, g.w));
        }
      }
      fwht<E, L>(V, lane);
      if (a.dg_outer) {
#pragma unroll
        for (int t = 0; t < E / 2; t += 2) {
          const float4 g = *reinterpret_cast<const float4*>(gp + t);
          mulz2(V[t], make_float2(g.x, g.y));
          mulz2(V[t + 1], make_float2(g.z, g.w));
        }
      }
      if (MODE == MODE_D) {
        const float amp = a.amp_rel * norm;
        if (amp != 0.f) {
          const uint32_t cb = (uint32_t)((b * d + s * E) >> 3);
          const uint32_t tlo = (uint32_t)tok, thi = (uint32_t)(tok >> 32);
#pragma unroll
          for (int c = 0; c < E / 8; c += 4) {
            qjl::U32x4 w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = qjl::U32x4{cb + c + j, tlo, thi, qjl::kStreamDither};
            philox_x4(w, a.k0, a.k1);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t x[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 xi = box_muller16(x[e], amp);
                const int r = 8 * (c + j) + 2 * e;
                if (r < E / 2) {
                  V[r].x += xi.x;
                  V[r + 1].x += xi.y;
                } else {
                  V[r - E / 2].y += xi.x;
                  V[r + 1 - E / 2].y += xi.y;
                }
              }
            }
          }
        }
      }
      // sign bits: element s*E + r is bit r % 32 of word (b*d + s*E + r) / 32 of the key's row
      if (valid) {
        uint32_t* out = a.bits + orow * (int64_t)a.W + ((b * d + s * E) >> 5);
#pragma unroll
        for (int w = 0; w < E / 32; ++w) {
          uint32_t acc = 0;
#pragma unroll
          for (int k = 31; k >= 0; --k) {
            const int r = 32 * w + k;
            const float y = (r < E / 2) ? V[r].x : V[r - E / 2].y;
            acc = __funnelshift_l(__float_as_uint(y), acc, 1);
          }
          qjl_hint::st_u32(out + w, ~acc, qjl_hint::evict_first());
        }
      }
    }
    if (valid && s == 0 && a.norms) qjl_hint::st_f32(a.norms + orow, norm, qjl_hint::evict_first());
    // fetch the next batch into the same buffer (issuing it at the end of the batch measured
    // faster than right after the last read of the staged rows)
    __syncwarp();
    const int64_t qn = q + stride;
    if (qn < nbatch) stage_rows<E, L, ES>(a, qn * K, (int)(a.n - qn * K < K ? a.n - qn * K : K), xb, bar, lane);
  }
}

// ---- host side ----------------------------------------------------------------------------------

struct Layout {
  int E, L, K;
};

Layout layout_for(int d) {
  Layout g;
  g.E = d < 128 ? d : 128;
  g.L = d / g.E;
  g.K = 32 / g.L;
  return g;
}

template <int E, int L, int ES, int MODE, bool PAGED>
qjl_status launch_t(const qjl_projection* P, KeysArgs a, int64_t n, cudaStream_t st) {
  using G = Geo<E, L, ES>;
  constexpr bool BUF = (MODE == MODE_P);
  auto kern = fqjl_keys_kernel<E, L, ES, MODE, PAGED>;
  const int d = P->d, nb = P->m / d;
  const int per_launch = std::max(1, (int)std::min<size_t>(nb, kTableBudget / ((size_t)G::TBLK * 4)));
  const size_t per_warp = G::XBUF + 8 + (BUF ? G::GBUF : 0);
  int dev = P->device;
  for (int b0 = 0; b0 < nb; b0 += per_launch) {
    const int b1 = std::min(nb, b0 + per_launch);
    const size_t tab = (size_t)(b1 - b0) * G::TBLK * 4;
    int nw = kMaxWarps;
    while (nw > 1 && tab + nw * per_warp > kSmemLimit) --nw;
    const size_t smem = tab + nw * per_warp;
    if (smem > kSmemLimit) return qjl_set_error(QJL_ERR_UNSUPPORTED, "FQJL key kernel: shared memory");
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return qjl_check_launch("fqjl_keys_kernel smem attribute");
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, nw * 32, smem) != cudaSuccess || per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    const int64_t nbatch = (n + G::K - 1) / G::K;
    const int64_t want = (nbatch + nw - 1) / nw;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)qjl_num_sms(dev) * per_sm));
    a.b0 = b0;
    a.b1 = b1;
    if (b0 > 0) a.norms = nullptr;
    qjl_log_launch("fqjl_keys_kernel", grid, nw * 32, smem, per_sm);
    kern<<<grid, nw * 32, smem, st>>>(a);
    const qjl_status s = qjl_check_launch("fqjl_keys_kernel");
    if (s != QJL_OK) return s;
  }
  return QJL_OK;
}

template <int E, int L>
qjl_status launch_el(const qjl_projection* P, const KeysArgs& a, int dtype, int64_t n, cudaStream_t st) {
  const bool dmode = P->kind == QJL_DFQJL;
  if (a.pm.pos) {
    if (dtype == QJL_F32)
      return dmode ? launch_t<E, L, 4, MODE_D, true>(P, a, n, st) : launch_t<E, L, 4, MODE_P, true>(P, a, n, st);
    return dmode ? launch_t<E, L, 2, MODE_D, true>(P, a, n, st) : launch_t<E, L, 2, MODE_P, true>(P, a, n, st);
  }
  if (dtype == QJL_F32)
    return dmode ? launch_t<E, L, 4, MODE_D, false>(P, a, n, st) : launch_t<E, L, 4, MODE_P, false>(P, a, n, st);
  return dmode ? launch_t<E, L, 2, MODE_D, false>(P, a, n, st) : launch_t<E, L, 2, MODE_P, false>(P, a, n, st);
}

}  // namespace

// Per-block tables of the key kernel. For each lane segment s (elements s*E .. s*E + E - 1) a
// block holds three runs of E + 4 words: D_r as register pairs (d_{sE+t}, d_{sE+t+E/2}), D_g as
// register pairs, and for each element i = s*E + r the byte offset of its gather source
// j = pi(i) in the warp's buffer, 4 K (j + j/E) (the identity for D-FQJL). The 4-word pad puts
// the segments of different lanes in different banks.
std::vector<float> fqjl_key_tables(int d, int m, const float* D_r, const int32_t* perm, const float* D_g) {
  const Layout g = layout_for(d);
  const int E = g.E, L = g.L, K = g.K, nb = m / d, tseg = E + 4, tblk = 3 * L * tseg;
  std::vector<float> t((size_t)nb * tblk, 0.f);
  for (int b = 0; b < nb; ++b) {
    float* blk = t.data() + (size_t)b * tblk;
    const float* Dr = D_r + (size_t)b * d;
    const float* Dg = D_g + (size_t)b * d;
    const int32_t* pi = perm + (size_t)b * d;
    for (int s = 0; s < L; ++s) {
      float* dr = blk + s * tseg;
      float* gp = blk + (L + s) * tseg;
      int32_t* ro = reinterpret_cast<int32_t*>(blk + (2 * L + s) * tseg);
      for (int u = 0; u < E / 2; ++u) {
        dr[2 * u] = Dr[s * E + u];
        dr[2 * u + 1] = Dr[s * E + u + E / 2];
        gp[2 * u] = Dg[s * E + u];
        gp[2 * u + 1] = Dg[s * E + u + E / 2];
      }
      for (int r = 0; r < E; ++r) {
        const int j = pi[s * E + r];
        ro[r] = 4 * K * (j + j / E);
      }
    }
  }
  return t;
}

bool fqjl_keys_supported(const qjl_projection* P) { return P->d >= 32 && P->d <= 1024 && P->ktab; }

qjl_status launch_fqjl_keys(const qjl_projection* P, const void* x, int dtype, int64_t n, int64_t ld,
                            uint64_t first_token, uint32_t* bits, float* norms, cudaStream_t st, const PageMap& pm) {
  if (n <= 0) return QJL_OK;
  KeysArgs a{};
  a.x = x;
  a.n = n;
  a.ld = ld;
  a.d = P->d;
  a.m = P->m;
  a.tab = P->ktab;
  a.amp_rel = P->kind == QJL_DFQJL ? sqrtf((float)P->d) * P->dither_sigma : 0.f;
  a.dg_outer = P->opt.dg_outer;
  a.k0 = (uint32_t)P->seed;
  a.k1 = (uint32_t)(P->seed >> 32);
  a.first_token = first_token;
  a.bits = bits;
  a.norms = norms;
  a.W = P->m / 32;
  a.err = qjl_error_flag(P->device);
  a.pm = pm;
  if (!a.err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  switch (P->d) {
    case 32: return launch_el<32, 1>(P, a, dtype, n, st);
    case 64: return launch_el<64, 1>(P, a, dtype, n, st);
    case 128: return launch_el<128, 1>(P, a, dtype, n, st);
    case 256: return launch_el<128, 2>(P, a, dtype, n, st);
    case 512: return launch_el<128, 4>(P, a, dtype, n, st);
    case 1024: return launch_el<128, 8>(P, a, dtype, n, st);
  }
  return qjl_set_error(QJL_ERR_UNSUPPORTED, "FQJL key kernel supports d in {32,...,1024}");
}
