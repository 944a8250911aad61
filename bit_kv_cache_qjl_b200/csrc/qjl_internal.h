// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/qjl.h"

struct qjl_projection {
  int d = 0, m = 0, kind = 0, device = 0;
  qjl_options opt{};
  float est_scale = 0.f;      // sqrt(pi/2)/m * alpha
  float dither_sigma = 0.f;   // sigma_rel for D-FQJL, else 0
  uint64_t seed = 0;
  // dense
  uint16_t* S_bf16 = nullptr;   // [m][d] bf16 bit patterns of S_eff (tensor-core path)
  float* St_f32 = nullptr;      // [d][m] S_eff transposed, fp32 (SIMT paths)
  // FQJL, each [m/d][d]
  float* D_r = nullptr;
  int32_t* perm = nullptr;
  float* D_g = nullptr;
  float* ktab = nullptr;        // key-kernel tables, per block (fqjl_key_tables)
  uint16_t* S1_bf16 = nullptr;  // [m][d] bf16 +-1: row b*d + i is row pi_b(i) of H times D_r^b (fqjl_tc.cu)
  // the tensor map of S_bf16 (dense) or S1_bf16 (FQJL) for the tcgen05 quantize
  // kernels (a CUtensorMap), encoded once when the projection is made;
  // s_map_ok is false if that failed
  alignas(64) unsigned char s_map[128] = {};
  bool s_map_ok = false;
  // host copies for export
  float* h_S = nullptr;
  float* h_D_r = nullptr;
  int32_t* h_perm = nullptr;
  float* h_D_g = nullptr;
};

// Row -> slot map of a paged cache (qjl_append_*): row r of an append batch is
// group r's new token at position pos[r]; it lives in page
// table[r * max_pages + pos[r] / page_tokens], slot pos[r] % page_tokens, i.e.
// pool row page * page_tokens + slot. With pos == nullptr rows map to
// themselves (the contiguous calls).
struct PageMap {
  const int32_t* pos = nullptr;
  const int32_t* table = nullptr;
  int max_pages = 0, page_tokens = 0;
  int64_t num_pages = 0;
#if defined(__CUDACC__)
  // pool row of append row r, or -1 when the position or the page id is out of range
  __device__ __forceinline__ int64_t slot(int64_t r) const {
    if (!pos) return r;
    const int p = __ldg(pos + r);
    if (p < 0 || p >= max_pages * page_tokens) return -1;
    const int pg = __ldg(table + r * (int64_t)max_pages + p / page_tokens);
    if (pg < 0 || (int64_t)pg >= num_pages) return -1;
    return (int64_t)pg * page_tokens + p % page_tokens;
  }
#endif
};

// Paged reads (qjl_scores_paged, qjl_decode_attention_paged): group g's token
// t is pool row table[g * max_pages + t / page_tokens] * page_tokens +
// t % page_tokens, for t < seq_lens[g] (clamped to [0, max_len]).
struct PagedRead {
  const int32_t* table = nullptr;
  const int32_t* seq_lens = nullptr;
  int max_pages = 0, page_tokens = 0;
  int64_t num_pages = 0;
};

// Switch to the projection's device for the duration of a call.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Error helpers (qjl_api.cu). set_error stores a thread-local message and returns s.
qjl_status qjl_set_error(qjl_status s, const std::string& msg);
qjl_status qjl_check_launch(const char* what);

// Launchers. They assume validated arguments and return QJL_OK or QJL_ERR_CUDA.
qjl_status launch_dense_simt(const qjl_projection* P, const void* keys, int dtype, int64_t n,
                             int64_t ld, uint32_t* bits, float* norms, float* proj_out,
                             cudaStream_t st, const PageMap& pm = PageMap());
qjl_status launch_project_dense(const qjl_projection* P, const float* q, int64_t nq, int64_t ld,
                                float* out, cudaStream_t st);
// many-query dense projection on the bf16 tensor cores (S_eff exactly bf16; the
// query split into three bf16 parts): fp32 accuracy
bool project_mma_supported(const qjl_projection* P, const float* q, int64_t ld, const float* out);
qjl_status launch_project_mma(const qjl_projection* P, const float* q, int64_t nq, int64_t ld, float* out,
                              cudaStream_t st);
bool dense_tc_supported(const qjl_projection* P, int dtype, const void* keys, int64_t ld);
// encodes P->s_map (called once by qjl_make_projection for a bf16 dense S)
void dense_tc_prepare(qjl_projection* P);
qjl_status launch_dense_tc(const qjl_projection* P, const void* keys, int64_t n, int64_t ld,
                           uint32_t* bits, float* norms, cudaStream_t st);
// 2-D bf16 tensor map (a CUtensorMap written to `map`, 128 bytes, 64-byte
// aligned): rows x cols, row stride ld elements, boxes of 64 columns x
// box_rows rows with 128-byte swizzle. False if the encoder is unavailable or
// rejects the arguments.
bool qjl_make_bf16_map(void* map, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows);
// FQJL keys with the first randomized Hadamard transform on tcgen05
// (fqjl_tc.cu): bf16 keys, d in {128, 256}, m a multiple of 256, the default
// order, not a paged append, and the D-FQJL dither only for d = 128. When the projection is made, fqjl_tc_shape
// decides whether it gets S1 (fqjl_tc_matrix, uploaded to S1_bf16), and
// fqjl_tc_prepare encodes S1's tensor map into s_map.
bool fqjl_tc_shape(int d, int m, bool dg_outer);
std::vector<uint16_t> fqjl_tc_matrix(int d, int m, const float* D_r, const int32_t* perm);
void fqjl_tc_prepare(qjl_projection* P);
bool fqjl_tc_supported(const qjl_projection* P, int dtype, int64_t n);
qjl_status launch_fqjl_tc(const qjl_projection* P, const void* keys, int64_t n, int64_t ld, uint64_t first_token,
                          uint32_t* bits, float* norms, cudaStream_t st);
qjl_status launch_fqjl_queries(const qjl_projection* P, const float* q, int64_t nq, int64_t ld,
                               float* out, cudaStream_t st);
std::vector<float> fqjl_key_tables(int d, int m, const float* D_r, const int32_t* perm, const float* D_g);
qjl_status launch_fqjl_keys(const qjl_projection* P, const void* keys, int dtype, int64_t n, int64_t ld,
                            uint64_t first_token, uint32_t* bits, float* norms, cudaStream_t st,
                            const PageMap& pm = PageMap());
// many-query scores on tcgen05 (scores_many.cu): m in {256, 512, 1024}, J <= 64, N < 2^31 - 128
// (a call of more keys than that in all is split by groups)
bool scores_many_supported(int m, int64_t N);
qjl_status launch_scores_many(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t G,
                              int64_t N, const float* sq, int J, float* scores, cudaStream_t st);
qjl_status launch_scores(const qjl_projection* P, const uint32_t* bits, const float* norms,
                         int64_t groups, int64_t N, const float* sq, int J, float* scores,
                         cudaStream_t st);
qjl_status launch_values_2bit(const void* v, int dtype, int64_t n, int d, uint32_t* codes,
                              uint16_t* scale, uint16_t* zero, cudaStream_t st, const PageMap& pm = PageMap());
qjl_status launch_scores_paged(const qjl_projection* P, const uint32_t* bits_pool, const float* norms_pool,
                               const PagedRead& pr, int64_t groups, int64_t max_len, const float* sq, int J,
                               float* scores, cudaStream_t st);
qjl_status launch_decode_paged(const qjl_projection* P, const uint32_t* bits_pool, const float* norms_pool,
                               const uint32_t* codes_pool, const uint16_t* scale_pool, const uint16_t* zero_pool,
                               const PagedRead& pr, int64_t groups, int64_t max_len, const float* sq,
                               float softmax_scale, float* out, void* ws, cudaStream_t st);
size_t decode_paged_workspace_bytes(int64_t groups, int64_t max_len, int d);
size_t decode_workspace_bytes(int64_t groups, int J, int64_t N, int d);
qjl_status launch_decode(const qjl_projection* P, const uint32_t* bits, const float* norms,
                         const uint32_t* codes, const uint16_t* scale, const uint16_t* zero,
                         int64_t groups, int64_t N, const float* sq, int J, float softmax_scale,
                         float* out, void* ws, size_t ws_bytes, cudaStream_t st);

// Bits of the per-device error int (read by qjl_device_errors). Bits 1..32 mark
// bounded waits that expired (each kernel's producer, drain, consumer and, in
// the tcgen05 kernel, MMA, TMEM and norm-warp waits).
enum : int {
  QJL_DEVERR_WAITS = 63,   // bits 1, 2, 4, 8, 16, 32: a bounded wait expired
  QJL_DEVERR_PAGE = 64,    // a paged-cache position or block-table entry was out of range and skipped
  QJL_DEVERR_SELFTEST = 128  // qjl_selftest_bounded_wait's wait expired, as it should
};

// Per-device int the kernels set when a bounded wait expires (qjl_api.cu):
// static device storage whose address is resolved on first use, so no call
// allocates for it. nullptr if the address cannot be resolved.
int* qjl_error_flag(int device);

// When the environment variable QJL_LOG_LAUNCH is set, print a launch's
// grid and occupancy to stderr (qjl_api.cu).
void qjl_log_launch(const char* kernel, int64_t grid, int block, size_t smem, int per_sm);

// Device properties cached per device (qjl_api.cu).
int qjl_num_sms(int device);
