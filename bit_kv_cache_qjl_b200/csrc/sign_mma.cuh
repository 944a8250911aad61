// Sign-bit dot products on the s8 tensor-core path (mma.sync m16n8k32).
//
// Shared by the score kernel and the fused decode kernel. Two schemes, both
// described at the top of scores.cu: weight classes (16-bit fixed-point Sq
// split into int8 hi/lo columns, sign bits fed as u8 A fragments of value
// 4^c, one AND per 4 bits; W MMAs per 16-key tile per column tile of four
// queries) and shift windows (unmasked shifted words as A, B as four int8
// digits of a residue modulo 2^32; W MMAs per tile per two queries).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qjl_sign {

// Named barrier `id` over `threads` threads, or __syncthreads for id 0.
__device__ __forceinline__ void named_barrier_or_sync(int id, int threads) {
  if (id) asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
  else __syncthreads();
}

constexpr int kQmax = 32639;  // 127 * 256 + 127: both int8 halves stay in range
constexpr int kQmaxE = 32638; // the even grid of the single-query tables (127 * 256 + 126)

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ int quant16(float v, float inv) {
  const float q = rintf(v * inv);
  return (int)fminf(fmaxf(q, (float)-kQmax), (float)kQmax);
}

// 2 rint(v inv / 2), clamped to +-kQmaxE: an even 16-bit code
__device__ __forceinline__ int quant16e(float v, float inv) {
  const float q = rintf(v * inv * 0.5f);
  return 2 * (int)fminf(fmaxf(q, (float)-(kQmaxE / 2)), (float)(kQmaxE / 2));
}

// Fills per-query scale data and the B fragments for group `gi`.
// Btab[(pt * W + mu) * 32 + lane] = (b0, b1) for column tile pt and MMA index
// mu = 8 p + j. The entries need W % 8 == 0.
template <int W>
__device__ void build_tables(const float* __restrict__ sqg, int J, int NT, float est_scale,
                             float* s_inv, float* s_mul, int* s_qsum, uint2* Btab, int nwarps,
                             int bar_id = 0) {
  // bar_id 0: all threads of the block take part; otherwise the first
  // 32 * nwarps threads synchronise on named barrier bar_id.
  constexpr int m = 32 * W;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = 32 * nwarps;
  for (int j = warp; j < J; j += nwarps) {
    const float* row = sqg + (int64_t)j * m;
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
      s_inv[j] = inv;
      s_mul[j] = est_scale * (mx > 0.f ? mx / (float)kQmax : 0.f);
      s_qsum[j] = qs;
    }
  }
  if (bar_id) asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthreads) : "memory");
  else __syncthreads();
  const int entries = NT * W * 32;
  for (int idx = threadIdx.x; idx < entries; idx += nthreads) {
    const int ln = idx & 31;
    const int mu = (idx >> 5) % W;
    const int pt = (idx >> 5) / W;
    const int n = ln >> 2, qq = ln & 3;
    const int jq = pt * 4 + (n >> 1);
    const int half = n & 1;  // 0: hi byte, 1: lo byte
    const int p = mu >> 3, jb = mu & 7;
    uint32_t b[2] = {0u, 0u};
    if (jq < J) {
      const float* row = sqg + (int64_t)jq * m;
      const float inv = s_inv[jq];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int word = qq * (W / 4) + 2 * p + r;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int Q = quant16(row[32 * word + 8 * e + jb], inv);
          const int lo = (int)(int8_t)(Q & 0xFF);
          const int hi = (Q - lo) >> 8;
          b[r] |= ((uint32_t)(half ? lo : hi) & 0xFFu) << (8 * e);
        }
      }
    }
    Btab[idx] = make_uint2(b[0], b[1]);
  }
  if (bar_id) asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthreads) : "memory");
  else __syncthreads();
}

template <int W>
__device__ __forceinline__ void load_words(const uint32_t* __restrict__ base, int64_t row, int64_t N,
                                           int q, uint32_t (&w)[W / 4]) {
  if (row < N) {
    const uint32_t* p = base + row * W + q * (W / 4);
    if constexpr (W == 8) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
      for (int k = 0; k < W / 16; ++k) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + k);
        w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < W / 4; ++k) w[k] = 0u;
  }
}


// Single-query variant of build_tables: the n8 B tile's column pairs carry
// the four bit-weight classes instead of four queries. Column 2c + h holds the
// hi (h = 0) or lo (h = 1) byte of Q for the coordinates whose A bytes have
// weight 4^c, and zero elsewhere. All MMAs of a key tile can then accumulate
// into one fragment, with class c landing in column pair c.
//
// Here Q lies on the even grid, Q = 2 rint(Sq kQmaxE / (2 max|Sq|)). So the
// MMAs for the odd bit of each 2-bit pair (s = 1) can take A straight from the
// unshifted word: their A bytes are worth 2 * 4^c, and their B entries hold
// Q / 2, exactly. That saves one shift per A register. The rounding step of Sq
// is twice the 16-bit one's.
template <int W>
__device__ void build_tables_cls(const float* __restrict__ sqg, float est_scale, float* s_inv, float* s_mul,
                                 int* s_qsum, uint2* Btab, int nwarps, int bar_id) {
  constexpr int m = 32 * W;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = 32 * nwarps;
  if (warp == 0) {
    float mx = 0.f;
    for (int i = lane; i < m; i += 32) mx = fmaxf(mx, fabsf(sqg[i]));
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float inv = mx > 0.f ? (float)kQmaxE / mx : 0.f;
    int qs = 0;
    for (int i = lane; i < m; i += 32) qs += quant16e(sqg[i], inv);
#pragma unroll
    for (int o = 16; o; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
    if (lane == 0) {
      s_inv[0] = inv;
      s_mul[0] = est_scale * (mx > 0.f ? mx / (float)kQmaxE : 0.f);
      s_qsum[0] = qs;
    }
  }
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthreads) : "memory");
  const float inv = s_inv[0];
  for (int idx = threadIdx.x; idx < W * 32; idx += nthreads) {
    const int ln = idx & 31, mu = idx >> 5;
    const int n = ln >> 2, qq = ln & 3;
    const int cls = n >> 1, half = n & 1;
    const int p = mu >> 3, jb = mu & 7;  // jb = 2 Ji + s
    uint32_t b[2] = {0u, 0u};
    if (cls == (jb >> 1)) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int word = qq * (W / 4) + 2 * p + r;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // odd bits (jb & 1): A carries twice the weight, so B holds Q / 2
          const int Q = quant16e(sqg[32 * word + 8 * e + jb], inv) >> (jb & 1);
          const int lo = (int)(int8_t)(Q & 0xFF);
          const int hi = (Q - lo) >> 8;
          b[r] |= ((uint32_t)(half ? lo : hi) & 0xFFu) << (8 * e);
        }
      }
    }
    Btab[idx] = make_uint2(b[0], b[1]);
  }
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthreads) : "memory");
}

// One column tile (4 queries) over a 16-key tile. Thread (g = lane/4,
// q = lane%4) receives 64 * sum_i b_i hi_i (hi) and 64 * sum_i b_i lo_i (lo)
// for query q of the column tile and key rows g (r = 0) and g + 8 (r = 1).
template <int W>
__device__ __forceinline__ void tile_sums(const uint32_t (&w0)[W / 4], const uint32_t (&w1)[W / 4],
                                          const uint2* __restrict__ Btab_pt, int lane, int (&hi)[2],
                                          int (&lo)[2]) {
  int acc[4][4];
#pragma unroll
  for (int b = 0; b < 4; ++b)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[b][c] = 0;
#pragma unroll
  for (int p = 0; p < W / 8; ++p) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const uint32_t x0 = w0[2 * p] >> s, x1 = w1[2 * p] >> s;
      const uint32_t x2 = w0[2 * p + 1] >> s, x3 = w1[2 * p + 1] >> s;
#pragma unroll
      for (int Ji = 0; Ji < 4; ++Ji) {
        const uint32_t M = 0x01010101u << (2 * Ji);
        const uint2 bb = Btab_pt[(8 * p + 2 * Ji + s) * 32 + lane];
        mma_u8s8(acc[Ji], x0 & M, x1 & M, x2 & M, x3 & M, bb.x, bb.y);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    hi[r] = ((acc[0][2 * r] * 4 + acc[1][2 * r]) * 4 + acc[2][2 * r]) * 4 + acc[3][2 * r];
    lo[r] = ((acc[0][2 * r + 1] * 4 + acc[1][2 * r + 1]) * 4 + acc[2][2 * r + 1]) * 4 + acc[3][2 * r + 1];
  }
}


// ---------------------------------------------------------------------------
// Shift-window ("digit") sign sums: no masking of the sign words.
//
// The A operand of the u8 MMA is the bit word shifted right by s, s = 0..7,
// unmasked: byte e of (w >> s) is the 8-bit window sum_t 2^t b_{8e+s+t}. Over
// the eight shifts every bit i of the word is the lowest bit of exactly one
// window (the one starting at i), so the windows' weights form a unit
// lower-triangular system. Giving window i the B value
//   B_i = sum_k 256^k (Q_{i-8k} - 2 Q_{i-8k-1})   (mod 2^32, Q_{<0} = 0)
// makes sum_windows A B = sum_i b_i Q_i (mod 2^32): the generating function of
// the window weights is (1 - 256 x^8) / (1 - 2x), and B is Q times its inverse.
// B is a 32-bit residue, carried as four signed base-256 digits in four B
// columns; the int32 column sums are combined as D0 + 2^8 D1 + 2^16 D2 + 2^24
// D3 in wrapping 32-bit arithmetic. As long as sum_i |Q_i| < 2^31 the residue
// is the exact sum, so Q can take 31 - log2(m) bits (2^23 - 1 at m = 256):
// the rounding of Sq to that grid is the only error.
//
// Per MMA the eight columns hold the digits of two queries (columns 4c'..4c'+3
// for query c' of the column tile). A thread (g, q) of the C fragment holds
// digits (2q, 2q+1) of query q >> 1 for key rows g and g + 8.
// ---------------------------------------------------------------------------

__host__ __device__ constexpr int qmax_dig(int m) { return (int)((2147483647u / (unsigned)m)); }

// digit `dg` (0..3) of the balanced base-256 representation of B (mod 2^32), as a byte
__device__ __forceinline__ uint32_t dig_byte(uint32_t B, int dg) {
  for (int c = 0; c < dg; ++c) {
    const int d = (int)(int8_t)(B & 0xFFu);
    B = (B - (uint32_t)d) >> 8;
  }
  return B & 0xFFu;
}

__device__ __forceinline__ int quant_dig(float v, float inv, int Qm) {
  const float q = rintf(v * inv);
  return (int)fminf(fmaxf(q, (float)-Qm), (float)Qm);
}

// Quantises the J query rows of group `sqg` to the digit grid (s_inv, s_mul,
// s_qsum) and fills the B fragments:
// Btab[(nt * W + mu) * 32 + lane] for column tile nt and MMA mu = 8 p + s.
// With PAIR the fragments of MMAs 2a and 2a + 1 sit side by side for each
// lane, so one 16-byte load fetches both: entry (nt, mu, lane) is at
// (nt * W + (mu & ~1)) * 32 + 2 lane + (mu & 1).
// With dup, J must be 1 and the one query's digits fill both column halves.
template <int W, bool PAIR = false>
__device__ void build_tables_dig(const float* __restrict__ sqg, int J, int NT, bool dup, float est_scale,
                                 float* s_inv, float* s_mul, int* s_qsum, uint2* Btab, int nwarps, int bar_id) {
  constexpr int m = 32 * W;
  constexpr int Qm = qmax_dig(m);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = 32 * nwarps;
  for (int j = warp; j < J; j += nwarps) {
    const float* row = sqg + (int64_t)j * m;
    float mx = 0.f;
    for (int i = lane; i < m; i += 32) mx = fmaxf(mx, fabsf(row[i]));
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float inv = mx > 0.f ? (float)Qm / mx : 0.f;
    int qs = 0;
    for (int i = lane; i < m; i += 32) qs += quant_dig(row[i], inv, Qm);
#pragma unroll
    for (int o = 16; o; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
    if (lane == 0) {
      s_inv[j] = inv;
      s_mul[j] = est_scale * (mx > 0.f ? mx / (float)Qm : 0.f);
      s_qsum[j] = qs;
    }
  }
  named_barrier_or_sync(bar_id, nthreads);
  const int entries = NT * W * 32;
  for (int idx = threadIdx.x; idx < entries; idx += nthreads) {
    const int ln = idx & 31;
    const int mu = (idx >> 5) % W;
    const int nt = (idx >> 5) / W;
    const int n = ln >> 2, qq = ln & 3;
    const int jq = dup ? 0 : nt * 2 + (n >> 2);
    const int dg = n & 3;
    const int p = mu >> 3, s = mu & 7;
    uint32_t b[2] = {0u, 0u};
    if (jq < J) {
      const float inv = s_inv[jq];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float* Sw = sqg + (int64_t)jq * m + 32 * (qq * (W / 4) + 2 * p + r);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 8 * e + s;
          uint32_t B = 0u;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int t = i - 8 * k;
            if (t < 0) break;
            const int v = quant_dig(Sw[t], inv, Qm) - (t > 0 ? 2 * quant_dig(Sw[t - 1], inv, Qm) : 0);
            B += (uint32_t)v << (8 * k);
          }
          b[r] |= dig_byte(B, dg) << (8 * e);
        }
      }
    }
    Btab[PAIR ? (nt * W + (mu & ~1)) * 32 + 2 * ln + (mu & 1) : idx] = make_uint2(b[0], b[1]);
  }
  named_barrier_or_sync(bar_id, nthreads);
}

// build_tables_dig from a shared-memory copy of the group's Sq rows (sSq,
// [J][m] fp32), quantising each value once. Scratch: sQ and sDig, [J][m]
// 32-bit words each; sDig may be sSq itself (phase 2 starts after the last
// read of sSq), and sQ may share Btab's space (phase 3 reads only sDig).
// Three phases, each closed by the named barrier:
//   1. per query (one warp each): max |Sq|, the grid scale, Q for every
//      coordinate into sQ, and sum Q;
//   2. per coordinate i: the residue B_i (mod 2^32) of its window, stored as
//      its four balanced base-256 digits, digit dg in byte dg of sDig;
//   3. per B fragment entry: eight digit bytes gathered from sDig.
// The entries are those of build_tables_dig (same layout and values).
template <int W>
__device__ void build_tables_dig_smem(const float* sSq, int J, int NT, bool dup, float est_scale, float* s_mul,
                                      int* s_qsum, int* sQ, uint32_t* sDig, uint2* Btab, int nwarps, int bar_id) {
  static_assert(W % 8 == 0, "whole MMA k-steps");
  constexpr int m = 32 * W;
  constexpr int Qm = qmax_dig(m);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthreads = 32 * nwarps;
  for (int j = warp; j < J; j += nwarps) {
    const float* row = sSq + j * m;
    float mx = 0.f;
#pragma unroll 4
    for (int k = 0; k < W; ++k) mx = fmaxf(mx, fabsf(row[32 * k + lane]));
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float inv = mx > 0.f ? (float)Qm / mx : 0.f;
    int qs = 0;
#pragma unroll 4
    for (int k = 0; k < W; ++k) {
      const int q = quant_dig(row[32 * k + lane], inv, Qm);
      sQ[j * m + 32 * k + lane] = q;
      qs += q;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
    if (lane == 0) {
      s_mul[j] = est_scale * (mx > 0.f ? mx / (float)Qm : 0.f);
      s_qsum[j] = qs;
    }
  }
  named_barrier_or_sync(bar_id, nthreads);
  for (int idx = threadIdx.x; idx < J * m; idx += nthreads) {
    const int i = idx & 31;              // coordinate within its sign word
    const int* Qw = sQ + (idx - i);      // that word's 32 values
    uint32_t B = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = i - 8 * k;
      if (t < 0) break;
      const int v = Qw[t] - (t > 0 ? 2 * Qw[t - 1] : 0);
      B += (uint32_t)v << (8 * k);
    }
    uint32_t packed = 0u;
#pragma unroll
    for (int dg = 0; dg < 4; ++dg) {
      const int d = (int)(int8_t)(B & 0xFFu);
      packed |= ((uint32_t)d & 0xFFu) << (8 * dg);
      B = (B - (uint32_t)d) >> 8;
    }
    sDig[idx] = packed;
  }
  named_barrier_or_sync(bar_id, nthreads);
  const int entries = NT * W * 32;
  for (int idx = threadIdx.x; idx < entries; idx += nthreads) {
    const int ln = idx & 31;
    const int mu = (idx >> 5) % W;
    const int nt = (idx >> 5) / W;
    const int n = ln >> 2, qq = ln & 3;
    const int jq = dup ? 0 : nt * 2 + (n >> 2);
    const int dg = n & 3;
    const int p = mu >> 3, s = mu & 7;
    uint32_t b[2] = {0u, 0u};
    if (jq < J) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint32_t* Dw = sDig + jq * m + 32 * (qq * (W / 4) + 2 * p + r);
#pragma unroll
        for (int e = 0; e < 4; ++e) b[r] |= ((Dw[8 * e + s] >> (8 * dg)) & 0xFFu) << (8 * e);
      }
    }
    Btab[idx] = make_uint2(b[0], b[1]);
  }
  named_barrier_or_sync(bar_id, nthreads);
}

}  // namespace qjl_sign
