// C ABI of the paged cache: append one token per group, then score or
// attend over each group's pages through a block table.
//
// The pages motivate a compressed KV cache for decoding, where the cache grows
// by one token per generated token and every step reads all of it (KIVI
// abstract, "Vladimir Braverman" page; QJL abstract, "Majid Daliri" page). A
// serving engine keeps such a cache in fixed-size pages and maps each
// sequence's logical tokens onto them with a block table. These calls run the
// same kernels as the contiguous ones: the key and value quantisers write to
// page slots, and the score and fused decode kernels gather page segments
// with their bulk copies.
//
// Every check here runs on the host before any launch. What the host cannot
// see (the block table's entries and the positions, which live on the
// device) the kernels check before every access: an out-of-range position or
// page id is skipped, so it never reads or writes outside the pools, and it
// sets bit 8 of the library's per-device error int.

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "qjl_internal.h"

namespace {

qjl_status check_pages(const int32_t* table, int max_pages, int page_tokens, int64_t num_pages) {
  if (!table) return qjl_set_error(QJL_ERR_INVALID_ARG, "block_table is NULL");
  if (page_tokens < 16 || page_tokens % 16 || page_tokens > (1 << 20))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "page_tokens must be a multiple of 16 in 16..2^20");
  if (max_pages < 1 || (int64_t)max_pages * page_tokens > ((int64_t)1 << 31) - 1)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "max_pages * page_tokens must be in 1..2^31-1");
  if (num_pages < 1 || num_pages > ((int64_t)1 << 40) / page_tokens)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "num_pages out of range");
  if (((uintptr_t)table & 3u)) return qjl_set_error(QJL_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
  return QJL_OK;
}

}  // namespace

extern "C" {

qjl_status qjl_append_keys(const qjl_projection* P, const void* keys, qjl_dtype dtype, int64_t groups, int64_t ld,
                           const int32_t* positions, const int32_t* block_table, int max_pages, int page_tokens,
                           int64_t num_pages, uint32_t* bits_pool, float* norms_pool, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (dtype != QJL_F32 && dtype != QJL_BF16) return qjl_set_error(QJL_ERR_INVALID_ARG, "unknown dtype");
  if (groups < 0 || groups > (1 << 24)) return qjl_set_error(QJL_ERR_INVALID_ARG, "groups out of range");
  if (groups == 0) return QJL_OK;
  qjl_status s = check_pages(block_table, max_pages, page_tokens, num_pages);
  if (s != QJL_OK) return s;
  if (!keys || !positions || !bits_pool || !norms_pool) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  const int es = dtype == QJL_F32 ? 4 : 2;
  if (ld < P->d) return qjl_set_error(QJL_ERR_INVALID_ARG, "ld < d");
  if (!aligned16(keys) || (ld * es) % 16)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "keys must be 16-byte aligned with ld*elsize a multiple of 16");
  if (!aligned16(bits_pool) || !aligned16(norms_pool))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "bits_pool and norms_pool must be 16-byte aligned");
  if (((uintptr_t)positions & 3u)) return qjl_set_error(QJL_ERR_INVALID_ARG, "positions must be 4-byte aligned");
  DeviceGuard g(P->device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  if (!qjl_error_flag(P->device)) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  PageMap pm;
  pm.pos = positions;
  pm.table = block_table;
  pm.max_pages = max_pages;
  pm.page_tokens = page_tokens;
  pm.num_pages = num_pages;
  cudaStream_t st = (cudaStream_t)stream;
  // one key per group: the SIMT projection (dense) or the Walsh-Hadamard kernel (FQJL); the
  // D-FQJL dither of a key is seeded by its pool row
  if (P->kind == QJL_DENSE) return launch_dense_simt(P, keys, dtype, groups, ld, bits_pool, norms_pool, nullptr, st, pm);
  return launch_fqjl_keys(P, keys, dtype, groups, ld, 0, bits_pool, norms_pool, st, pm);
}

qjl_status qjl_append_values_2bit(const void* v, qjl_dtype dtype, int64_t groups, int d, const int32_t* positions,
                                  const int32_t* block_table, int max_pages, int page_tokens, int64_t num_pages,
                                  uint32_t* codes_pool, uint16_t* scale_pool, uint16_t* zero_pool, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (dtype != QJL_F32 && dtype != QJL_BF16) return qjl_set_error(QJL_ERR_INVALID_ARG, "unknown dtype");
  if (groups < 0 || groups > (1 << 24)) return qjl_set_error(QJL_ERR_INVALID_ARG, "groups out of range");
  if (d < 32 || d > 4096 || d % 32) return qjl_set_error(QJL_ERR_INVALID_ARG, "d must be a multiple of 32 in 32..4096");
  if (groups == 0) return QJL_OK;
  qjl_status s = check_pages(block_table, max_pages, page_tokens, num_pages);
  if (s != QJL_OK) return s;
  if (!v || !positions || !codes_pool || !scale_pool || !zero_pool)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(v) || !aligned16(codes_pool) || !aligned16(scale_pool) || !aligned16(zero_pool))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "v and the pools must be 16-byte aligned");
  if (((uintptr_t)positions & 3u)) return qjl_set_error(QJL_ERR_INVALID_ARG, "positions must be 4-byte aligned");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return qjl_set_error(QJL_ERR_CUDA, "cannot query the current device");
  if (!qjl_error_flag(dev)) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  PageMap pm;
  pm.pos = positions;
  pm.table = block_table;
  pm.max_pages = max_pages;
  pm.page_tokens = page_tokens;
  pm.num_pages = num_pages;
  return launch_values_2bit(v, dtype, groups, d, codes_pool, scale_pool, zero_pool, (cudaStream_t)stream, pm);
}

qjl_status qjl_scores_paged(const qjl_projection* P, const uint32_t* bits_pool, const float* norms_pool,
                            const int32_t* block_table, int max_pages, int page_tokens, int64_t num_pages,
                            const int32_t* seq_lens, int64_t groups, int64_t max_len, const float* sq, int J,
                            float* scores, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (groups < 0 || groups > (1 << 24)) return qjl_set_error(QJL_ERR_INVALID_ARG, "groups out of range");
  if (J < 1 || J > 64) return qjl_set_error(QJL_ERR_INVALID_ARG, "q_per_group must be in 1..64");
  if (max_len < 0) return qjl_set_error(QJL_ERR_INVALID_ARG, "max_len must be >= 0");
  if (groups == 0 || max_len == 0) return QJL_OK;
  qjl_status s = check_pages(block_table, max_pages, page_tokens, num_pages);
  if (s != QJL_OK) return s;
  if (max_len > (int64_t)max_pages * page_tokens)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "max_len exceeds max_pages * page_tokens");
  if (!bits_pool || !norms_pool || !seq_lens || !sq || !scores) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(bits_pool) || !aligned16(norms_pool) || !aligned16(sq))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "bits_pool, norms_pool and sq must be 16-byte aligned");
  if (((uintptr_t)seq_lens & 3u) || ((uintptr_t)scores & 3u))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "seq_lens/scores must be 4-byte aligned");
  DeviceGuard g(P->device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  PagedRead pr;
  pr.table = block_table;
  pr.seq_lens = seq_lens;
  pr.max_pages = max_pages;
  pr.page_tokens = page_tokens;
  pr.num_pages = num_pages;
  return launch_scores_paged(P, bits_pool, norms_pool, pr, groups, max_len, sq, J, scores, (cudaStream_t)stream);
}

size_t qjl_decode_paged_workspace_bytes(int64_t groups, int64_t max_len, int d) {
  if (groups <= 0 || max_len <= 0 || d < 32 || d % 32) return 0;
  return decode_paged_workspace_bytes(groups, max_len, d);
}

qjl_status qjl_decode_attention_paged(const qjl_projection* P, const uint32_t* bits_pool, const float* norms_pool,
                                      const uint32_t* codes_pool, const uint16_t* scale_pool,
                                      const uint16_t* zero_pool, const int32_t* block_table, int max_pages,
                                      int page_tokens, int64_t num_pages, const int32_t* seq_lens, int64_t groups,
                                      int64_t max_len, const float* sq, float softmax_scale, float* out, void* ws,
                                      size_t ws_bytes, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (groups < 0 || groups > (1 << 24)) return qjl_set_error(QJL_ERR_INVALID_ARG, "groups out of range");
  if (max_len < 1) return qjl_set_error(QJL_ERR_INVALID_ARG, "max_len must be >= 1");
  if (!isfinite(softmax_scale)) return qjl_set_error(QJL_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (groups == 0) return QJL_OK;
  qjl_status s = check_pages(block_table, max_pages, page_tokens, num_pages);
  if (s != QJL_OK) return s;
  if (max_len > (int64_t)max_pages * page_tokens)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "max_len exceeds max_pages * page_tokens");
  if (!bits_pool || !norms_pool || !codes_pool || !scale_pool || !zero_pool || !seq_lens || !sq || !out || !ws)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(bits_pool) || !aligned16(norms_pool) || !aligned16(codes_pool) || !aligned16(scale_pool) ||
      !aligned16(zero_pool) || !aligned16(sq) || !aligned16(out) || !aligned16(ws))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "the pools, sq, out and ws must be 16-byte aligned");
  if (((uintptr_t)seq_lens & 3u)) return qjl_set_error(QJL_ERR_INVALID_ARG, "seq_lens must be 4-byte aligned");
  if (ws_bytes < decode_paged_workspace_bytes(groups, max_len, P->d))
    return qjl_set_error(QJL_ERR_WORKSPACE, "workspace smaller than qjl_decode_paged_workspace_bytes()");
  DeviceGuard g(P->device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  if (!qjl_error_flag(P->device)) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  PagedRead pr;
  pr.table = block_table;
  pr.seq_lens = seq_lens;
  pr.max_pages = max_pages;
  pr.page_tokens = page_tokens;
  pr.num_pages = num_pages;
  return launch_decode_paged(P, bits_pool, norms_pool, codes_pool, scale_pool, zero_pool, pr, groups, max_len, sq,
                             softmax_scale, out, ws, (cudaStream_t)stream);
}

}  // extern "C"
