// C ABI: argument checks, projection lifecycle and dispatch to the kernels.
//
// Every check runs on the host before any launch, so a rejected call never
// touches the GPU.

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "philox.h"
#include "qjl_internal.h"

static thread_local std::string g_last_error;

qjl_status qjl_set_error(qjl_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

qjl_status qjl_check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return qjl_set_error(QJL_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return QJL_OK;
}

int qjl_num_sms(int device) {
  static std::mutex mu;
  static std::vector<int> cache;
  std::lock_guard<std::mutex> lock(mu);
  if (device < 0) return 148;
  if ((int)cache.size() <= device) cache.resize(device + 1, 0);
  if (!cache[device]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v <= 0)
      v = 148;
    cache[device] = v;
  }
  return cache[device];
}

void qjl_log_launch(const char* kernel, int64_t grid, int block, size_t smem, int per_sm) {
  static const bool on = getenv("QJL_LOG_LAUNCH") != nullptr;
  if (on)
    fprintf(stderr, "[qjl] %s grid=%lld block=%d smem=%zu ctas_per_sm=%d\n", kernel, (long long)grid, block, smem,
            per_sm);
}

// The per-device error int is static device storage of this module, so no
// call of the library allocates device memory for it: it exists on every
// device from the moment the module is loaded there, zero-initialised. Its
// device address is resolved once per device (with that device current) and
// cached; it stays valid for the life of the device's primary context.
static __device__ int g_kernel_error;

int* qjl_error_flag(int device) {
  static std::mutex mu;
  static int* flags[64] = {};
  if (device < 0 || device >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!flags[device]) {
    DeviceGuard g(device);
    void* p = nullptr;
    if (!g.ok || cudaGetSymbolAddress(&p, g_kernel_error) != cudaSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    flags[device] = (int*)p;
  }
  return flags[device];
}

namespace {

// fp64 standard normal from Philox words 0 and 1 (Box-Muller), rounded to fp32.
float gaussian_f32(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2, uint32_t stream) {
  qjl::U32x4 r = qjl::philox({c0, c1, c2, stream}, (uint32_t)seed, (uint32_t)(seed >> 32));
  const double u0 = ((double)r.x + 0.5) * 0x1p-32;
  const double u1 = ((double)r.y + 0.5) * 0x1p-32;
  return (float)(sqrt(-2.0 * log(u0)) * cos(2.0 * M_PI * u1));
}

// Round an fp32 value to bf16, nearest-even; returns the bf16 bit pattern.
uint16_t bf16_bits_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

float bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// Fault injection on the host: with QJL_FAIL_ALLOC_AFTER=k in the environment,
// the projection's device allocations after the first k (process-wide) report
// failure without calling cudaMalloc, so tests can drive the out-of-memory path
// of qjl_make_projection without exhausting a GPU.
bool injected_alloc_failure() {
  static const long limit = [] {
    const char* v = getenv("QJL_FAIL_ALLOC_AFTER");
    return v ? atol(v) : -1L;
  }();
  static std::mutex mu;
  static long count = 0;
  if (limit < 0) return false;
  std::lock_guard<std::mutex> lock(mu);
  return count++ >= limit;
}

template <class T>
qjl_status dev_upload(T** dst, const T* src, size_t count) {
  if (injected_alloc_failure()) {
    *dst = nullptr;
    return qjl_set_error(QJL_ERR_OOM, "cudaMalloc failed for projection parameters (injected by QJL_FAIL_ALLOC_AFTER)");
  }
  if (cudaMalloc((void**)dst, count * sizeof(T)) != cudaSuccess) {
    cudaGetLastError();
    *dst = nullptr;
    return qjl_set_error(QJL_ERR_OOM, "cudaMalloc failed for projection parameters");
  }
  if (cudaMemcpy(*dst, src, count * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess)
    return qjl_set_error(QJL_ERR_CUDA, "cudaMemcpy of projection parameters failed");
  return QJL_OK;
}

void free_projection(qjl_projection* P) {
  if (!P) return;
  cudaFree(P->S_bf16);
  cudaFree(P->St_f32);
  cudaFree(P->D_r);
  cudaFree(P->perm);
  cudaFree(P->D_g);
  cudaFree(P->ktab);
  cudaFree(P->S1_bf16);
  free(P->h_S);
  free(P->h_D_r);
  free(P->h_perm);
  free(P->h_D_g);
  delete P;
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

}  // namespace

extern "C" {

void qjl_default_options(qjl_options* opt) {
  if (!opt) return;
  opt->dither_sigma_rel = 0.5f;
  opt->dg_outer = 0;
  opt->s_bf16 = 1;
}

const char* qjl_status_string(qjl_status s) {
  switch (s) {
    case QJL_OK: return "ok";
    case QJL_ERR_INVALID_ARG: return "invalid argument";
    case QJL_ERR_UNSUPPORTED: return "unsupported";
    case QJL_ERR_CUDA: return "CUDA error";
    case QJL_ERR_OOM: return "out of memory";
    case QJL_ERR_WORKSPACE: return "workspace too small";
    case QJL_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

const char* qjl_last_error_message(void) { return g_last_error.c_str(); }

const char* qjl_version(void) { return "qjl-b200 0.1 (sm_100a)"; }

qjl_status qjl_make_projection(uint64_t seed, int d, int m, qjl_kind kind, const qjl_options* opt,
                               qjl_projection** out) {
  g_last_error.clear();
  if (!out) return qjl_set_error(QJL_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (kind != QJL_DENSE && kind != QJL_DFQJL && kind != QJL_PFQJL)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "unknown kind");
  if (d < 1 || d > 4096) return qjl_set_error(QJL_ERR_INVALID_ARG, "d must be in 1..4096");
  if (m < 32 || m > 16384 || m % 32)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "m must be a multiple of 32 in 32..16384");
  if (kind != QJL_DENSE) {
    if (!is_pow2(d) || d < 32 || d > 1024)
      return qjl_set_error(QJL_ERR_INVALID_ARG, "FQJL needs d a power of two in 32..1024");
    if (m % d) return qjl_set_error(QJL_ERR_INVALID_ARG, "FQJL needs m a multiple of d");
  }
  qjl_options o;
  qjl_default_options(&o);
  if (opt) o = *opt;
  if (!(o.dither_sigma_rel >= 0.f) || o.dither_sigma_rel > 100.f)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "dither_sigma_rel must be in [0, 100]");

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return qjl_set_error(QJL_ERR_CUDA, "no CUDA device");
  }
  qjl_projection* P = new qjl_projection();
  P->d = d;
  P->m = m;
  P->kind = kind;
  P->device = dev;
  P->opt = o;
  P->seed = seed;
  P->dither_sigma = (kind == QJL_DFQJL) ? o.dither_sigma_rel : 0.f;
  const double alpha = sqrt(1.0 + (double)P->dither_sigma * P->dither_sigma);
  P->est_scale = (float)(sqrt(M_PI / 2.0) / m * alpha);

  qjl_status st = QJL_OK;
  if (kind == QJL_DENSE) {
    const size_t md = (size_t)m * d;
    P->h_S = (float*)malloc(md * sizeof(float));
    std::vector<uint16_t> sb(md);
    std::vector<float> st_f(md);
    if (!P->h_S) { free_projection(P); return qjl_set_error(QJL_ERR_OOM, "host allocation failed"); }
    for (size_t e = 0; e < md; ++e) {
      const float g = gaussian_f32(seed, (uint32_t)e, (uint32_t)(e >> 32), 0, qjl::kStreamGauss);
      const uint16_t b = bf16_bits_rne(g);
      const float eff = o.s_bf16 ? bf16_to_float(b) : g;
      sb[e] = b;
      P->h_S[e] = eff;
      const size_t i = e / d, j = e % d;
      st_f[j * m + i] = eff;
    }
    if (o.s_bf16) st = dev_upload(&P->S_bf16, sb.data(), md);
    if (st == QJL_OK) st = dev_upload(&P->St_f32, st_f.data(), md);
    if (st == QJL_OK && o.s_bf16) dense_tc_prepare(P);
  } else {
    const int nb = m / d;
    const size_t cnt = (size_t)nb * d;
    P->h_D_r = (float*)malloc(cnt * sizeof(float));
    P->h_D_g = (float*)malloc(cnt * sizeof(float));
    P->h_perm = (int32_t*)malloc(cnt * sizeof(int32_t));
    if (!P->h_D_r || !P->h_D_g || !P->h_perm) {
      free_projection(P);
      return qjl_set_error(QJL_ERR_OOM, "host allocation failed");
    }
    for (int b = 0; b < nb; ++b) {
      for (int j = 0; j < d; ++j) {
        qjl::U32x4 r = qjl::philox({(uint32_t)j, 0u, (uint32_t)b, qjl::kStreamRademacher},
                                   (uint32_t)seed, (uint32_t)(seed >> 32));
        P->h_D_r[(size_t)b * d + j] = (r.x & 1u) ? -1.f : 1.f;
        P->h_D_g[(size_t)b * d + j] = gaussian_f32(seed, (uint32_t)j, 0, (uint32_t)b, qjl::kStreamGauss);
      }
      int32_t* pi = P->h_perm + (size_t)b * d;
      for (int j = 0; j < d; ++j) pi[j] = j;
      if (kind == QJL_PFQJL) {
        // Fisher-Yates (Knuth, Algorithm P): j = floor(r * (i + 1) / 2^64) from a 64-bit draw.
        for (int i = d - 1; i >= 1; --i) {
          qjl::U32x4 r = qjl::philox({(uint32_t)i, 0u, (uint32_t)b, qjl::kStreamPerm},
                                     (uint32_t)seed, (uint32_t)(seed >> 32));
          const uint64_t r64 = ((uint64_t)r.x << 32) | r.y;
          const int j = (int)(((unsigned __int128)r64 * (unsigned)(i + 1)) >> 64);
          const int32_t t = pi[i];
          pi[i] = pi[j];
          pi[j] = t;
        }
      }
    }
    st = dev_upload(&P->D_r, P->h_D_r, cnt);
    if (st == QJL_OK) st = dev_upload(&P->D_g, P->h_D_g, cnt);
    if (st == QJL_OK) st = dev_upload(&P->perm, P->h_perm, cnt);
    if (st == QJL_OK) {
      const std::vector<float> kt = fqjl_key_tables(d, m, P->h_D_r, P->h_perm, P->h_D_g);
      st = dev_upload(&P->ktab, kt.data(), kt.size());
    }
    if (st == QJL_OK && fqjl_tc_shape(d, m, o.dg_outer != 0)) {
      const std::vector<uint16_t> s1 = fqjl_tc_matrix(d, m, P->h_D_r, P->h_perm);
      st = dev_upload(&P->S1_bf16, s1.data(), s1.size());
      if (st == QJL_OK) fqjl_tc_prepare(P);
    }
  }
  if (st != QJL_OK) {
    free_projection(P);
    return st;
  }
  *out = P;
  return QJL_OK;
}

qjl_status qjl_destroy_projection(qjl_projection* proj) {
  if (!proj) return QJL_OK;
  DeviceGuard g(proj->device);
  free_projection(proj);
  return QJL_OK;
}

qjl_status qjl_projection_info(const qjl_projection* P, int* d, int* m, int* kind, float* est_scale) {
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (d) *d = P->d;
  if (m) *m = P->m;
  if (kind) *kind = P->kind;
  if (est_scale) *est_scale = P->est_scale;
  return QJL_OK;
}

qjl_status qjl_projection_export(const qjl_projection* P, qjl_export_what what, void* host_dst,
                                 size_t bytes) {
  if (!P || !host_dst) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL argument");
  const void* src = nullptr;
  size_t need = 0;
  const size_t md = (size_t)P->m * P->d, cnt = (size_t)(P->m / P->d) * P->d;
  switch (what) {
    case QJL_EXPORT_S: src = P->h_S; need = md * 4; break;
    case QJL_EXPORT_DR: src = P->h_D_r; need = cnt * 4; break;
    case QJL_EXPORT_PERM: src = P->h_perm; need = cnt * 4; break;
    case QJL_EXPORT_DG: src = P->h_D_g; need = cnt * 4; break;
    default: return qjl_set_error(QJL_ERR_INVALID_ARG, "unknown export selector");
  }
  if (!src) return qjl_set_error(QJL_ERR_INVALID_ARG, "this projection kind has no such array");
  if (bytes != need) return qjl_set_error(QJL_ERR_INVALID_ARG, "bytes must equal the array size");
  memcpy(host_dst, src, need);
  return QJL_OK;
}

qjl_status qjl_quantize_keys(const qjl_projection* P, const void* keys, qjl_dtype dtype, int64_t n,
                             int64_t ld, uint64_t first_token, uint32_t* bits, float* norms,
                             void* stream) {
  g_last_error.clear();
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (dtype != QJL_F32 && dtype != QJL_BF16) return qjl_set_error(QJL_ERR_INVALID_ARG, "unknown dtype");
  if (n < 0 || n > (int64_t)1 << 40) return qjl_set_error(QJL_ERR_INVALID_ARG, "n out of range");
  if (n == 0) return QJL_OK;
  if (!keys || !bits || !norms) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  const int es = dtype == QJL_F32 ? 4 : 2;
  if (ld < P->d) return qjl_set_error(QJL_ERR_INVALID_ARG, "ld < d");
  if (!aligned16(keys) || (ld * es) % 16) return qjl_set_error(QJL_ERR_INVALID_ARG, "keys must be 16-byte aligned with ld*elsize a multiple of 16");
  if (!aligned16(bits)) return qjl_set_error(QJL_ERR_INVALID_ARG, "bits must be 16-byte aligned");
  if (((uintptr_t)norms & 3u)) return qjl_set_error(QJL_ERR_INVALID_ARG, "norms must be 4-byte aligned");
  DeviceGuard g(P->device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  cudaStream_t st = (cudaStream_t)stream;
  if (P->kind == QJL_DENSE) {
    if (dense_tc_supported(P, dtype, keys, ld)) return launch_dense_tc(P, keys, n, ld, bits, norms, st);
    return launch_dense_simt(P, keys, dtype, n, ld, bits, norms, nullptr, st);
  }
  if (fqjl_tc_supported(P, dtype, n)) return launch_fqjl_tc(P, keys, n, ld, first_token, bits, norms, st);
  return launch_fqjl_keys(P, keys, dtype, n, ld, first_token, bits, norms, st);
}

qjl_status qjl_project_queries(const qjl_projection* P, const float* q, int64_t nq, int64_t ld,
                               float* sq, void* stream) {
  g_last_error.clear();
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (nq < 0 || nq > (int64_t)1 << 32) return qjl_set_error(QJL_ERR_INVALID_ARG, "nq out of range");
  if (nq == 0) return QJL_OK;
  if (!q || !sq) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (ld < P->d) return qjl_set_error(QJL_ERR_INVALID_ARG, "ld < d");
  if (!aligned16(q) || (ld * 4) % 16) return qjl_set_error(QJL_ERR_INVALID_ARG, "q must be 16-byte aligned with ld a multiple of 4");
  if (!aligned16(sq)) return qjl_set_error(QJL_ERR_INVALID_ARG, "sq must be 16-byte aligned");
  DeviceGuard g(P->device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  cudaStream_t st = (cudaStream_t)stream;
  if (P->kind == QJL_DENSE) return launch_project_dense(P, q, nq, ld, sq, st);
  return launch_fqjl_queries(P, q, nq, ld, sq, st);
}

qjl_status qjl_scores(const qjl_projection* P, const uint32_t* bits, const float* norms,
                      int64_t groups, int64_t N, const float* sq, int J, float* scores,
                      void* stream) {
  g_last_error.clear();
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (groups < 0 || N < 0 || groups > (1 << 24) || N > ((int64_t)1 << 36))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "groups/N out of range");
  if (J < 1 || J > 64) return qjl_set_error(QJL_ERR_INVALID_ARG, "q_per_group must be in 1..64");
  if (groups == 0 || N == 0) return QJL_OK;
  if (!bits || !norms || !sq || !scores) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(bits) || !aligned16(sq)) return qjl_set_error(QJL_ERR_INVALID_ARG, "bits and sq must be 16-byte aligned");
  if (((uintptr_t)norms & 3u) || ((uintptr_t)scores & 3u)) return qjl_set_error(QJL_ERR_INVALID_ARG, "norms/scores must be 4-byte aligned");
  DeviceGuard g(P->device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  return launch_scores(P, bits, norms, groups, N, sq, J, scores, (cudaStream_t)stream);
}

qjl_status qjl_quantize_values_2bit(const void* v, qjl_dtype dtype, int64_t n, int d, uint32_t* codes,
                                    uint16_t* scale, uint16_t* zero, void* stream) {
  g_last_error.clear();
  if (dtype != QJL_F32 && dtype != QJL_BF16) return qjl_set_error(QJL_ERR_INVALID_ARG, "unknown dtype");
  if (n < 0 || n > (int64_t)1 << 40) return qjl_set_error(QJL_ERR_INVALID_ARG, "n out of range");
  if (d < 32 || d > 4096 || d % 32) return qjl_set_error(QJL_ERR_INVALID_ARG, "d must be a multiple of 32 in 32..4096");
  if (n == 0) return QJL_OK;
  if (!v || !codes || !scale || !zero) return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(v) || !aligned16(codes)) return qjl_set_error(QJL_ERR_INVALID_ARG, "v and codes must be 16-byte aligned");
  if (((uintptr_t)scale & 1u) || ((uintptr_t)zero & 1u)) return qjl_set_error(QJL_ERR_INVALID_ARG, "scale/zero must be 2-byte aligned");
  return launch_values_2bit(v, dtype, n, d, codes, scale, zero, (cudaStream_t)stream);
}

size_t qjl_decode_workspace_bytes(int64_t groups, int J, int64_t N, int d) {
  if (groups <= 0 || N <= 0 || J < 1 || J > 64 || d < 32 || d % 32) return 0;
  return decode_workspace_bytes(groups, J, N, d);
}

qjl_status qjl_decode_attention(const qjl_projection* P, const uint32_t* bits, const float* norms,
                                const uint32_t* codes, const uint16_t* scale, const uint16_t* zero,
                                int64_t groups, int64_t N, const float* sq, int J, float softmax_scale,
                                float* out, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  if (groups < 0 || N < 0 || groups > (1 << 24) || N > ((int64_t)1 << 36))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "groups/N out of range");
  if (J < 1 || J > 64) return qjl_set_error(QJL_ERR_INVALID_ARG, "q_per_group must be in 1..64");
  if (P->d % 32 || P->d > 1024) return qjl_set_error(QJL_ERR_UNSUPPORTED, "decode attention needs d a multiple of 32, <= 1024");
  if (!isfinite(softmax_scale)) return qjl_set_error(QJL_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (groups == 0) return QJL_OK;
  if (N == 0) return qjl_set_error(QJL_ERR_INVALID_ARG, "N must be >= 1 (softmax over an empty context)");
  if (!bits || !norms || !codes || !scale || !zero || !sq || !out || !ws)
    return qjl_set_error(QJL_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(bits) || !aligned16(codes) || !aligned16(sq) || !aligned16(out) || !aligned16(ws))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "bits, codes, sq, out and ws must be 16-byte aligned");
  if (((uintptr_t)norms & 3u) || ((uintptr_t)scale & 1u) || ((uintptr_t)zero & 1u))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "norms/scale/zero misaligned");
  const size_t need = decode_workspace_bytes(groups, J, N, P->d);
  if (ws_bytes < need) return qjl_set_error(QJL_ERR_WORKSPACE, "workspace smaller than qjl_decode_workspace_bytes()");
  DeviceGuard g(P->device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  return launch_decode(P, bits, norms, codes, scale, zero, groups, N, sq, J, softmax_scale, out, ws,
                       ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"
