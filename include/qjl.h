/*
 * qjl.h: C ABI of the B200 (sm_100a) QJL / FQJL key-sketch library.
 *
 * Method (sources are web pages, cited by title and section):
 *   - QJL abstract by Zandieh, Daliri and Han, on the "Majid Daliri" author
 *     page (scholarfeed). A key k is stored as the sign bits of a JL
 *     projection S k, with no quantisation constants, plus ||k||. A query q
 *     is projected without quantisation. <q,k> is estimated without bias by
 *       est = sqrt(pi/2) / m * ||k|| * sum_i sign(S k)_i * (S q)_i.
 *   - "Fast Quantized Johnson - Lindenstrauss Transforms" (AI Radio episode
 *     page), sections "In short", "Key concepts", "The paper" (abstract) and
 *     "Transcript: The paper's improvements". S is replaced by two randomized
 *     Hadamard transforms with a Gaussian second diagonal. D-FQJL adds
 *     Gaussian dither before the sign. P-FQJL adds a random permutation
 *     between the two Hadamard stages. Both cost O(d log d) per vector.
 *   - KIVI abstract "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV
 *     Cache", on the "Vladimir Braverman" author page (catalyzex). Values are
 *     quantised per token to 2 bits, and a decode step reads the whole cache.
 *
 * Conventions for every call:
 *   - Data pointers are DEVICE pointers owned by the caller, except where a
 *     parameter says "host". The library owns only the projection's parameter
 *     buffers, which qjl_destroy_projection frees.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Compute calls are asynchronous on it. Only make, destroy and
 *     export synchronise.
 *   - All arguments are checked on the host before any launch. A failed check
 *     returns an error status and launches nothing. The outputs are then
 *     untouched, and qjl_last_error_message() says which check failed.
 *     A launch failure returns QJL_ERR_CUDA with the CUDA error text. Output
 *     contents are undefined after any error.
 *   - Packed sign bits: coordinate i of a key is bit (i % 32) of uint32 word
 *     i / 32 (LSB first). Bit = 1 iff the pre-sign value is >= 0.
 *   - Estimator scale: c = sqrt(pi/2)/m, times alpha = sqrt(1 + sigma_rel^2)
 *     for D-FQJL (the dither inflates the pre-sign variance).
 *   - Calls are thread-safe. A projection is immutable after creation and may
 *     be shared by threads and streams.
 */
#ifndef QJL_B200_H
#define QJL_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QJL_OK = 0,
  QJL_ERR_INVALID_ARG = -1, /* bad size, null pointer, misalignment, bad enum */
  QJL_ERR_UNSUPPORTED = -2, /* valid but not implemented for this shape/dtype */
  QJL_ERR_CUDA = -3,        /* a CUDA runtime call or kernel launch failed */
  QJL_ERR_OOM = -4,         /* device or host allocation failed */
  QJL_ERR_WORKSPACE = -5,   /* workspace too small (see *_workspace_bytes) */
  QJL_ERR_DEVICE = -6       /* a kernel reported an internal error (bounded wait expired) */
} qjl_status;

typedef enum {
  QJL_DENSE = 0, /* S: m x d, iid N(0,1) (QJL abstract) */
  QJL_DFQJL = 1, /* H D_g H D_r plus Gaussian dither before the sign (FQJL, "Key concepts") */
  QJL_PFQJL = 2  /* H D_g Pi H D_r (FQJL, "Key concepts", "Transcript") */
} qjl_kind;

typedef enum { QJL_F32 = 0, QJL_BF16 = 1 } qjl_dtype;

typedef struct {
  /* D-FQJL dither std relative to ||k|| (in units where each pre-sign
   * coordinate has std ||k||). Default 0.5, which equals 0.5 ||k|| / sqrt(d)
   * on the normalised Hadamard scale. Ignored for other kinds. */
  float dither_sigma_rel;
  /* FQJL order. 0 (default): y = sqrt(d) H_n D_g Pi H_n D_r k, i.e. randomized
   * Hadamard transforms H*D composed, which keeps the estimator exactly
   * unbiased ("Transcript: The paper's improvements"). 1: the literal order
   * y = sqrt(d) D_g H_n Pi H_n D_r k, which the estimator cannot debias. */
  int dg_outer;
  /* Dense only. 1 (default): S_eff = bf16(S) for keys and queries alike, as
   * the bf16 tensor-core contraction needs. 0: S_eff = fp32 S. */
  int s_bf16;
} qjl_options;

/* Fill *opt with the defaults (0.5, 0, 1). */
void qjl_default_options(qjl_options* opt);

typedef struct qjl_projection qjl_projection;

/*
 * Draw the projection from `seed` and upload it to the current device.
 * Sources: QJL abstract (dense S); FQJL "The paper" abstract and "Key
 * concepts" (D_r, Pi, D_g).
 * Generator: Philox4x32-10 (Salmon et al., SC'11) with key = seed and
 * counter = (index_lo, index_hi, block, stream). The streams are 0 Gaussian
 * (S, D_g), 1 Rademacher (D_r), 2 permutation (Fisher-Yates) and 3 dither.
 * Gaussians use Box-Muller in fp64 and are rounded to fp32. The D-FQJL dither
 * of coordinate e of token t takes the block at counter (e/8, t_lo, t_hi, 3):
 * word w gives coordinates 8(e/8) + 2w and + 1 by Box-Muller on its two
 * 16-bit halves.
 *   d     head dimension, 1..4096. FQJL: a power of two, 32..1024.
 *   m     sketch size, a multiple of 32, 32..16384. FQJL: a multiple of d.
 *   opt   NULL for the defaults.
 *   out   receives the handle. Free it with qjl_destroy_projection.
 * Synchronous. Returns QJL_ERR_OOM if device memory runs out.
 */
qjl_status qjl_make_projection(uint64_t seed, int d, int m, qjl_kind kind,
                               const qjl_options* opt, qjl_projection** out);

/* Free the projection's device buffers. NULL is accepted. Synchronous. */
qjl_status qjl_destroy_projection(qjl_projection* proj);

/* Shape, kind and the estimator scale c * alpha (any pointer may be NULL). */
qjl_status qjl_projection_info(const qjl_projection* proj, int* d, int* m, int* kind,
                               float* est_scale);

typedef enum {
  QJL_EXPORT_S = 0,    /* dense: S_eff as fp32, [m][d] row-major */
  QJL_EXPORT_DR = 1,   /* FQJL: D_r as fp32 (+1/-1), [m/d][d] */
  QJL_EXPORT_PERM = 2, /* FQJL: Pi as int32 gather indices, [m/d][d] (identity for D-FQJL) */
  QJL_EXPORT_DG = 3    /* FQJL: D_g as fp32, [m/d][d] */
} qjl_export_what;

/* Copy one parameter array to HOST memory `host_dst` of `bytes` bytes (must
 * be exactly the array's size). Synchronous. */
qjl_status qjl_projection_export(const qjl_projection* proj, qjl_export_what what,
                                 void* host_dst, size_t bytes);

/*
 * Key sketch (QJL abstract; FQJL "Key concepts" for D/P).
 *   keys        [n][ld] of `dtype` (only the first d of each row are read),
 *               16-byte aligned. ld >= d, and ld*elsize is a multiple of 16 bytes.
 *   n           number of keys, >= 0 (0 is a no-op).
 *   first_token absolute index of row 0 (seeds the D-FQJL dither per token,
 *               so appended keys get the same dither in any batch split).
 *   bits        out [n][m/32] uint32, 16-byte aligned.
 *   norms       out [n] fp32: ||k||_2.
 * Dense with bf16 keys and bf16 S_eff runs the tcgen05/TMA kernel. Every
 * other dense case runs an fp32 SIMT kernel. FQJL with bf16 keys, d in
 * {128, 256}, m a multiple of 256 and the default order (D-FQJL: d = 128)
 * runs its first Hadamard factor as an exact +-1 contraction on tcgen05 and
 * the rest on the FP32 lanes; every other FQJL case runs the register
 * Walsh-Hadamard kernel.
 */
qjl_status qjl_quantize_keys(const qjl_projection* proj, const void* keys, qjl_dtype dtype,
                             int64_t n, int64_t ld, uint64_t first_token, uint32_t* bits,
                             float* norms, void* stream);

/*
 * Query projection without quantisation: the "standard JL transform" of the
 * QJL abstract. sq[i] = S_eff q_i (dense) or the FQJL map of q_i, without
 * dither and without sign.
 *   q   [nq][ld] fp32, ld >= d.   sq  out [nq][m] fp32.
 * The sums are fp32-accurate on every path. A dense map with bf16 S_eff and
 * nq >= 1024 runs on the bf16 tensor cores: each query element splits into
 * three bf16 parts, and the products with the exactly-bf16 S_eff are exact in
 * fp32. That path needs d % 16 == 0, m % 128 == 0, q and sq 8-byte aligned
 * and ld even. Otherwise an fp32 SIMT kernel runs.
 */
qjl_status qjl_project_queries(const qjl_projection* proj, const float* q, int64_t nq,
                               int64_t ld, float* sq, void* stream);

/*
 * Asymmetric estimator (QJL abstract) for every (group, query, key):
 *   scores[g][j][n] = c * alpha * norms[g][n] * sum_i (2 bit_i - 1) * sq[g][j][i]
 *   bits    [groups][N][m/32] uint32, 16-byte aligned.
 *   norms   [groups][N] fp32.
 *   sq      [groups][q_per_group][m] fp32 (from qjl_project_queries).
 *   scores  out [groups][q_per_group][N] fp32.
 *   1 <= q_per_group <= 64. Grouped-query attention puts q_per_group query
 *   heads on one key head's bits.
 * Sq is rounded per (group, query) to fixed point: with 1 or 2 queries per
 * group at m = 256 or 512 to 31 - log2(m) bits (scale max|Sq| / (2^31/m - 1)),
 * otherwise to 16 bits (scale max|Sq|/32639). The sign sums are exact
 * integers, so the added error is at most c*alpha*||k|| * m * max|Sq| / 65278.
 */
qjl_status qjl_scores(const qjl_projection* proj, const uint32_t* bits, const float* norms,
                      int64_t groups, int64_t N, const float* sq, int q_per_group,
                      float* scores, void* stream);

/*
 * KIVI per-token 2-bit value quantisation (KIVI abstract). Each token's d
 * channels form groups of 32. Per group: zero = fp16(min) and
 * scale = fp16(fp32(max - min) / 3).
 * code = clamp(rint_even(fp32(fp32(v - zero) / scale)), 0, 3), or 0 when
 * scale == 0. Channel c is bits 2*(c%16) of word c/16.
 *   v      [n][d] of `dtype`, d a multiple of 32, |v| <= 65504 (fp16 range).
 *   codes  out [n][d/16] uint32.
 *   scale, zero  out [n][d/32] IEEE binary16 bit patterns.
 */
qjl_status qjl_quantize_values_2bit(const void* v, qjl_dtype dtype, int64_t n, int d,
                                    uint32_t* codes, uint16_t* scale, uint16_t* zero,
                                    void* stream);

/* Workspace bytes qjl_decode_attention needs for these sizes. */
size_t qjl_decode_workspace_bytes(int64_t groups, int q_per_group, int64_t N, int d);

/*
 * Fused decode attention over a sketched key cache and 2-bit values (QJL
 * abstract for the scores; KIVI abstract for the per-token values and the
 * whole-cache read per decode step):
 *   out[g][j][:] = sum_n softmax_n(softmax_scale * est[g][j][n]) * v_hat[g][n][:]
 * with est as in qjl_scores and v_hat = code * scale + zero. There is no
 * mask: a decode query sees all N cached tokens. The key axis is split across
 * CTAs, and partial (max, sum, acc) results in `ws` are merged with a
 * log-sum-exp combine.
 *   bits/norms/sq  as in qjl_scores (the projection's d is the head dim).
 *   codes [groups][N][d/16], scale/zero [groups][N][d/32] as written by
 *   qjl_quantize_values_2bit.
 *   out   [groups][q_per_group][d] fp32.
 *   ws    device workspace of >= qjl_decode_workspace_bytes(...) bytes,
 *         16-byte aligned. It is scratch, and calls that overlap on the GPU
 *         must not share it.
 */
qjl_status qjl_decode_attention(const qjl_projection* proj, const uint32_t* bits,
                                const float* norms, const uint32_t* codes,
                                const uint16_t* scale, const uint16_t* zero, int64_t groups,
                                int64_t N, const float* sq, int q_per_group, float softmax_scale,
                                float* out, void* ws, size_t ws_bytes, void* stream);

/* Fixed scratch size of qjl_decode_attention_noalloc: 4 MiB per device. */
#define QJL_DECODE_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * qjl_decode_attention without a caller workspace, for callers that may not
 * allocate device memory while decoding. Examples: a serving engine whose
 * own pool owns the whole GPU and forbids raw cudaMalloc so that its
 * accounting stays exact, or a latency-critical loop that cannot afford
 * cudaMalloc's implicit device-wide synchronisation. The pages have no
 * counterpart to this call. It exists only to suit such callers.
 *
 * Arguments are those of qjl_decode_attention without ws and ws_bytes. The
 * split-N workspace comes from a file-scope device array of
 * QJL_DECODE_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the
 * library holds until exit. The call allocates nothing.
 *   - Returns QJL_ERR_WORKSPACE, launching nothing, when
 *     qjl_decode_workspace_bytes(groups, q_per_group, N, d) exceeds that size.
 *   - The first call on each device resolves the array's device address
 *     (cudaGetSymbolAddress, with that device current), and that of the
 *     kernels' error int, which is static device storage as well. Make that
 *     first call before any stream capture. The cached addresses stay valid
 *     for the life of the device's primary context: after cudaDeviceReset
 *     the library must be reloaded.
 *   - All calls share the one array. Calls that overlap on the GPU (for
 *     example on two streams) race and give undefined results. Serialise
 *     them. Earlier calls' contents need no clearing: every workspace entry
 *     is written before it is read.
 */
qjl_status qjl_decode_attention_noalloc(const qjl_projection* proj, const uint32_t* bits,
                                        const float* norms, const uint32_t* codes,
                                        const uint16_t* scale, const uint16_t* zero,
                                        int64_t groups, int64_t N, const float* sq,
                                        int q_per_group, float softmax_scale, float* out,
                                        void* stream);

/*
 * Paged cache. A decode step appends one token per group (sequence x key head)
 * and then reads the whole cache (KIVI abstract: the decode step loads the
 * whole KV cache per generated token). A serving engine keeps such a cache in
 * fixed-size pages. The pages name no layout; this one is ours:
 *   - A pool holds num_pages pages of page_tokens token slots each.
 *     page_tokens is a multiple of 16.
 *   - Group g's logical token t lives in page block_table[g*max_pages +
 *     t/page_tokens], slot t % page_tokens, i.e. pool row
 *     page * page_tokens + slot.
 *   - Pools are arrays over pool rows:
 *       bits  [num_pages*page_tokens][m/32] uint32
 *       norms [num_pages*page_tokens] fp32
 *       codes [num_pages*page_tokens][d/16] uint32
 *       scale, zero [num_pages*page_tokens][d/32] binary16
 *     Their layout per row is that of the contiguous calls. Every pool is
 *     16-byte aligned.
 *   - block_table is int32 device [groups][max_pages]. positions and seq_lens
 *     are int32 device [groups]. The caller owns pools, tables and lengths,
 *     and assigns pages.
 * The host checks everything it can see. The kernels check, before every
 * access, the positions and the block-table entries they read: a position
 * outside [0, max_pages*page_tokens) or a page id outside [0, num_pages) is
 * skipped, so it is never read or written, and the call's results for it
 * are undefined.
 */

/*
 * Sketch one key per group (as qjl_quantize_keys) into the paged pools, at
 * logical position positions[g] of group g.
 *   keys  [groups][ld] of `dtype`, 16-byte aligned, ld*elsize % 16 == 0.
 * The D-FQJL dither of a key is seeded by its pool row, page*page_tokens +
 * slot (the first_token of the contiguous call). Dense keys take the fp32
 * SIMT projection: one key per group and step is latency work.
 */
qjl_status qjl_append_keys(const qjl_projection* proj, const void* keys, qjl_dtype dtype,
                           int64_t groups, int64_t ld, const int32_t* positions,
                           const int32_t* block_table, int max_pages, int page_tokens,
                           int64_t num_pages, uint32_t* bits_pool, float* norms_pool,
                           void* stream);

/*
 * 2-bit per-token values (as qjl_quantize_values_2bit, bit for bit) of one
 * token per group, written at positions[g] of group g.
 *   v  [groups][d] of `dtype`, 16-byte aligned, d a multiple of 32.
 */
qjl_status qjl_append_values_2bit(const void* v, qjl_dtype dtype, int64_t groups, int d,
                                  const int32_t* positions, const int32_t* block_table,
                                  int max_pages, int page_tokens, int64_t num_pages,
                                  uint32_t* codes_pool, uint16_t* scale_pool,
                                  uint16_t* zero_pool, void* stream);

/*
 * The estimator of qjl_scores over each group's first seq_lens[g] tokens of
 * a paged cache (seq_lens clamped to [0, max_len]).
 *   max_len  host bound on seq_lens, <= max_pages*page_tokens. It is also the
 *            row stride of scores.
 *   sq       [groups][q_per_group][m] fp32, 16-byte aligned.
 *   scores   out [groups][q_per_group][max_len] fp32. Entries at t >=
 *            seq_lens[g] are not written.
 * Supports 1 <= q_per_group <= 2 and m in {256, 512}: it is the shift-window
 * kernel of qjl_scores, with bulk copies gathered per page segment.
 */
qjl_status qjl_scores_paged(const qjl_projection* proj, const uint32_t* bits_pool,
                            const float* norms_pool, const int32_t* block_table, int max_pages,
                            int page_tokens, int64_t num_pages, const int32_t* seq_lens,
                            int64_t groups, int64_t max_len, const float* sq, int q_per_group,
                            float* scores, void* stream);

/* Workspace bytes qjl_decode_attention_paged needs for these sizes. */
size_t qjl_decode_paged_workspace_bytes(int64_t groups, int64_t max_len, int d);

/*
 * Fused decode attention (as qjl_decode_attention, one query per group) over
 * each group's first seq_lens[g] tokens of a paged cache.
 *   max_len  host bound on seq_lens, <= max_pages*page_tokens.
 *   sq       [groups][m] fp32.   out [groups][d] fp32.
 *   ws       device workspace of >= qjl_decode_paged_workspace_bytes(...)
 *            bytes, 16-byte aligned. Calls that overlap on the GPU must not
 *            share it.
 * A group with seq_lens[g] <= 0 gets an all-zero output row. Supports d = 128
 * and m = 256.
 */
qjl_status qjl_decode_attention_paged(const qjl_projection* proj, const uint32_t* bits_pool,
                                      const float* norms_pool, const uint32_t* codes_pool,
                                      const uint16_t* scale_pool, const uint16_t* zero_pool,
                                      const int32_t* block_table, int max_pages, int page_tokens,
                                      int64_t num_pages, const int32_t* seq_lens, int64_t groups,
                                      int64_t max_len, const float* sq, float softmax_scale,
                                      float* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Causal prefill attention over a sketched key cache and 2-bit values (QJL
 * abstract for the scores; KIVI abstract for the values). Every position is a
 * query that attends to the keys at or before it:
 *   out[g][i][:] = sum_{j <= i} softmax_j(softmax_scale * est[g][i][j]) * v_hat[g][j][:]
 * with est as in qjl_scores (sq[g][i] against key j) and v_hat = code * scale
 * + zero. P and v_hat enter the tensor cores as binary16, and the sums run in
 * fp32.
 *   bits/norms/codes/scale/zero  the cache of L tokens per group, as in
 *                                qjl_decode_attention.
 *   sq    [groups][L][m] fp32: the projected query of every position.
 *   out   [groups][L][d] fp32.
 * Supports d = 128 and m = 256. bits, codes, sq and out must be 16-byte aligned.
 */
qjl_status qjl_prefill_attention(const qjl_projection* proj, const uint32_t* bits,
                                 const float* norms, const uint32_t* codes, const uint16_t* scale,
                                 const uint16_t* zero, int64_t groups, int64_t L, const float* sq,
                                 float softmax_scale, float* out, void* stream);

/*
 * KIVI per-channel 2-bit keys: the like-for-like baseline of the QJL sketch on
 * the same shapes. The KIVI abstract ("KIVI: A Tuning-Free Asymmetric 2bit
 * Quantization for KV Cache", "Vladimir Braverman" page) quantises keys per
 * channel and values per token. A channel's group is a block of 32
 * consecutive tokens of one key head; the last block of a ragged N is shorter.
 * Per (block, channel): zero = fp16(min), scale = fp16(fp32(max - min) / 3),
 * code = clamp(rint_even(fp32(fp32(k - zero) / scale)), 0, 3), or 0 when
 * scale == 0. At d = 128 that is 48 bytes per key, against 36 for the QJL
 * sketch at m = 256.
 *   keys   [groups][N][d] of `dtype` (rows contiguous), d in {64, 128, 256}.
 *   codes  out [groups][N][d/16] uint32: channel c at bits 2*(c%16) of word c/16.
 *   scale, zero  out [groups][ceil(N/32)][d] binary16.
 * All four buffers are 16-byte aligned.
 */
qjl_status qjl_kivi_quantize_keys_2bit(const void* keys, qjl_dtype dtype, int64_t groups, int64_t N,
                                       int d, uint32_t* codes, uint16_t* scale, uint16_t* zero,
                                       void* stream);

/*
 * Scores over KIVI keys:
 *   scores[g][j][n] = sum_c q[g][j][c] * (code[g][n][c] * scale + zero)
 * with the scale and zero of token n's block, accumulated in fp32.
 *   q       [groups][q_per_group][d] fp32, 1 <= q_per_group <= 64.
 *   scores  out [groups][q_per_group][N] fp32.
 */
qjl_status qjl_kivi_key_scores(const uint32_t* codes, const uint16_t* scale, const uint16_t* zero,
                               int64_t groups, int64_t N, int d, const float* q, int q_per_group,
                               float* scores, void* stream);

/*
 * Device-side errors. Kernels never trap. A bounded wait that expires (4 s of
 * wall time), or a paged-cache entry that is out of range, sets a bit in a
 * per-device int and the kernel winds down. The int is static device storage
 * of the library (zero when the library loads on a device); no call allocates
 * it. The bits are:
 *   1, 2, 4, 8, 16, 32  a bounded wait expired (1: a producer's wait for a
 *        free stage; 2: a final wait for a CTA's own copies; 4: a consumer's
 *        wait for a full stage; 8, 16, 32: the tcgen05 quantize kernel's
 *        MMA-completion, TMEM and norm-warp waits)
 *   64   a paged-cache position or block-table entry was out of range (skipped)
 *   128  qjl_selftest_bounded_wait's wait expired (as it should)
 * qjl_device_errors synchronises `device`, stores the int in *flags and, if
 * `clear` is nonzero, zeroes it. It returns QJL_ERR_DEVICE when any bit was
 * set, else QJL_OK.
 */
qjl_status qjl_device_errors(int device, int clear, int* flags);

/* Launch (asynchronously, on the legacy default stream) one thread that
 * waits on a barrier nothing completes, bounded by limit_ns (1..1e9). When
 * the limit passes it sets bit 128 and returns. Tests use it to check the
 * expiry path without hanging the GPU. */
qjl_status qjl_selftest_bounded_wait(int device, uint64_t limit_ns);

/* Static text for a status code. */
const char* qjl_status_string(qjl_status s);

/* Text of the last error raised on the calling thread ("" if none). */
const char* qjl_last_error_message(void);

/* Library version string. */
const char* qjl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QJL_B200_H */
