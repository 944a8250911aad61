// Device-side error reporting.
//
// The kernels never trap. Every wait on an mbarrier is bounded by wall time,
// and on expiry the kernel records a bit in a per-device error int and winds
// down. The paged-cache kernels record another bit when they skip a position
// or block-table entry that is out of range. qjl_device_errors reads (and may
// clear) that int. qjl_selftest_bounded_wait runs the bounded wait on a
// barrier that nothing completes, with a short limit, so a test can see the
// expiry path end and report without hanging the GPU.

#include <cuda_runtime.h>
#include <stdint.h>

#include "mbarrier.cuh"
#include "qjl_internal.h"

namespace {

// One thread: an mbarrier expecting one arrival that never comes. The bounded
// wait gives up after limit_ns and the kernel records QJL_DEVERR_SELFTEST.
__global__ void selftest_wait_kernel(uint64_t limit_ns, int* __restrict__ err) {
  using namespace qjl_sync;
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_fence_init();
  const uint32_t a = smem_u32(&bar);
  const uint64_t t0 = global_ns();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(0u)
        : "memory");
    if (done) return;  // cannot happen: nothing arrives
    if (global_ns() - t0 > limit_ns) {
      atomicOr(err, QJL_DEVERR_SELFTEST);
      return;
    }
  }
}

}  // namespace

extern "C" {

qjl_status qjl_device_errors(int device, int clear, int* flags) {
  qjl_set_error(QJL_OK, "");
  if (!flags) return qjl_set_error(QJL_ERR_INVALID_ARG, "flags is NULL");
  *flags = 0;
  DeviceGuard g(device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the device");
  int* err = qjl_error_flag(device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  if (cudaDeviceSynchronize() != cudaSuccess) return qjl_check_launch("qjl_device_errors: synchronize");
  if (cudaMemcpy(flags, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return qjl_check_launch("qjl_device_errors: read");
  if (clear && cudaMemset(err, 0, sizeof(int)) != cudaSuccess) return qjl_check_launch("qjl_device_errors: clear");
  return *flags ? qjl_set_error(QJL_ERR_DEVICE, "a kernel reported an error (see the flags)") : QJL_OK;
}

qjl_status qjl_selftest_bounded_wait(int device, uint64_t limit_ns) {
  qjl_set_error(QJL_OK, "");
  if (limit_ns == 0 || limit_ns > 1000000000ull) return qjl_set_error(QJL_ERR_INVALID_ARG, "limit_ns must be in 1..1e9");
  DeviceGuard g(device);
  if (!g.ok) return qjl_set_error(QJL_ERR_CUDA, "cannot select the device");
  int* err = qjl_error_flag(device);
  if (!err) return qjl_set_error(QJL_ERR_CUDA, "cannot resolve the kernel error flag");
  selftest_wait_kernel<<<1, 32>>>(limit_ns, err);
  return qjl_check_launch("selftest_wait_kernel");
}

}  // extern "C"
