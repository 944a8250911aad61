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
  // host copies for export
  float* h_S = nullptr;
  float* h_D_r = nullptr;
  int32_t* h_perm = nullptr;
  float* h_D_g = nullptr;
};

// Error helpers (qjl_api.cu). set_error stores a thread-local message and returns s.
qjl_status qjl_set_error(qjl_status s, const std::string& msg);
qjl_status qjl_check_launch(const char* what);

// Launchers. They assume validated arguments and return QJL_OK or QJL_ERR_CUDA.
qjl_status launch_dense_simt(const qjl_projection* P, const void* keys, int dtype, int64_t n,
                             int64_t ld, uint32_t* bits, float* norms, float* proj_out,
                             cudaStream_t st);
qjl_status launch_project_dense(const qjl_projection* P, const float* q, int64_t nq, int64_t ld,
                                float* out, cudaStream_t st);
bool dense_tc_supported(const qjl_projection* P, int dtype, const void* keys, int64_t ld);
qjl_status launch_dense_tc(const qjl_projection* P, const void* keys, int64_t n, int64_t ld,
                           uint32_t* bits, float* norms, cudaStream_t st);
qjl_status launch_fqjl_queries(const qjl_projection* P, const float* q, int64_t nq, int64_t ld,
                               float* out, cudaStream_t st);
std::vector<float> fqjl_key_tables(int d, int m, const float* D_r, const int32_t* perm, const float* D_g);
qjl_status launch_fqjl_keys(const qjl_projection* P, const void* keys, int dtype, int64_t n, int64_t ld,
                            uint64_t first_token, uint32_t* bits, float* norms, cudaStream_t st);
bool scores_mma_supported(int m);
bool scores_tc_supported(int m, int J);
qjl_status launch_scores_tc(const qjl_projection* P, const uint32_t* bits, const float* norms, int64_t groups,
                            int64_t N, const float* sq, int J, float* scores, cudaStream_t st);
qjl_status launch_scores(const qjl_projection* P, const uint32_t* bits, const float* norms,
                         int64_t groups, int64_t N, const float* sq, int J, float* scores,
                         cudaStream_t st);
qjl_status launch_values_2bit(const void* v, int dtype, int64_t n, int d, uint32_t* codes,
                              uint16_t* scale, uint16_t* zero, cudaStream_t st);
size_t decode_workspace_bytes(int64_t groups, int J, int64_t N, int d);
qjl_status launch_decode(const qjl_projection* P, const uint32_t* bits, const float* norms,
                         const uint32_t* codes, const uint16_t* scale, const uint16_t* zero,
                         int64_t groups, int64_t N, const float* sq, int J, float softmax_scale,
                         float* out, void* ws, size_t ws_bytes, cudaStream_t st);

// Per-device int the kernels set when a bounded wait expires (qjl_api.cu).
// It is allocated on first use and never freed.
int* qjl_error_flag(int device);

// When the environment variable QJL_LOG_LAUNCH is set, print a launch's
// grid and occupancy to stderr (qjl_api.cu).
void qjl_log_launch(const char* kernel, int64_t grid, int block, size_t smem, int per_sm);

// Device properties cached per device (qjl_api.cu).
int qjl_num_sms(int device);
