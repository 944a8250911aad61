// Fused decode attention for callers that must not allocate device memory.
//
// Some embedders may not call cudaMalloc while they decode. One example is a
// serving engine whose own pool owns all of the GPU's memory and forbids raw
// allocations, so that its accounting stays exact. Another is a latency-
// critical decode loop that cannot afford cudaMalloc's implicit device-wide
// synchronisation. This entry point takes the split-N workspace of
// qjl_decode_attention from a fixed file-scope device array instead of a
// caller buffer, and it allocates nothing.
//
// The array is a host-side symbol: its name in host code is not a device
// address. The first call on each device resolves the address with
// cudaGetSymbolAddress, with that device current, and caches it (as it does
// for the kernels' error int, also static device storage). That first call
// should therefore come before any stream capture, and the cached addresses
// last as long as the device's primary context. Every call shares the array,
// and overlapping calls on the GPU race. The kernels write every workspace
// entry they later read, so stale contents need no clearing.

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "qjl_internal.h"

static __device__ __align__(256) unsigned char g_decode_scratch[QJL_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of g_decode_scratch on `device` (which must be current), resolved once per device.
qjl_status scratch_address(int device, void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  if (device < 0 || device >= 64) return qjl_set_error(QJL_ERR_UNSUPPORTED, "device index >= 64");
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return qjl_set_error(QJL_ERR_CUDA, std::string("cudaGetSymbolAddress(decode scratch): ") +
                                             cudaGetErrorString(e));
    }
    addr[device] = p;
  }
  *out = addr[device];
  return QJL_OK;
}

}  // namespace

extern "C" qjl_status qjl_decode_attention_noalloc(const qjl_projection* P, const uint32_t* bits, const float* norms,
                                                   const uint32_t* codes, const uint16_t* scale, const uint16_t* zero,
                                                   int64_t groups, int64_t N, const float* sq, int J,
                                                   float softmax_scale, float* out, void* stream) {
  qjl_set_error(QJL_OK, "");
  if (!P) return qjl_set_error(QJL_ERR_INVALID_ARG, "projection is NULL");
  // the range checks of qjl_decode_attention, before the workspace size is computed from them
  if (groups < 0 || N < 0 || groups > (1 << 24) || N > ((int64_t)1 << 36))
    return qjl_set_error(QJL_ERR_INVALID_ARG, "groups/N out of range");
  if (J < 1 || J > 64) return qjl_set_error(QJL_ERR_INVALID_ARG, "q_per_group must be in 1..64");
  if (P->d % 32 || P->d > 1024)
    return qjl_set_error(QJL_ERR_UNSUPPORTED, "decode attention needs d a multiple of 32, <= 1024");
  if (groups > 0 && N > 0) {
    const size_t need = decode_workspace_bytes(groups, J, N, P->d);
    if (need > QJL_DECODE_NOALLOC_SCRATCH_BYTES)
      return qjl_set_error(QJL_ERR_WORKSPACE,
                           "decode workspace of " + std::to_string(need) + " bytes exceeds the fixed " +
                               std::to_string((size_t)QJL_DECODE_NOALLOC_SCRATCH_BYTES) +
                               "-byte scratch of qjl_decode_attention_noalloc; use qjl_decode_attention");
  }
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) {
    cudaGetLastError();
    return qjl_set_error(QJL_ERR_CUDA, "no CUDA device");
  }
  if (prev != P->device && cudaSetDevice(P->device) != cudaSuccess) {
    cudaGetLastError();
    return qjl_set_error(QJL_ERR_CUDA, "cannot select the projection's device");
  }
  void* ws = nullptr;
  qjl_status st = scratch_address(P->device, &ws);
  if (st == QJL_OK && !qjl_error_flag(P->device))
    st = qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  if (st == QJL_OK)
    st = qjl_decode_attention(P, bits, norms, codes, scale, zero, groups, N, sq, J, softmax_scale, out, ws,
                              QJL_DECODE_NOALLOC_SCRATCH_BYTES, stream);
  if (prev != P->device) cudaSetDevice(prev);
  return st;
}
