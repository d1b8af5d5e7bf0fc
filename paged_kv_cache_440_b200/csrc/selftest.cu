// Self-test of the bounded wait every kernel of this library uses on its
// shared-memory barriers: one thread waits on a barrier that nothing will
// complete, gives up after the limit, records the timeout bit and returns.
// It exercises the failure path without hanging the device.
#include "device.cuh"
#include "internal.h"

namespace pagedkv {
namespace {

__global__ void wait_timeout_kernel(int *status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  dev::mbar_init(&bar, 1);
  dev::fence_barrier_init();
  // nobody arrives: phase 0 never completes
  (void)dev::mbar_wait(&bar, 0, status, limit_ns);
}

}  // namespace
}  // namespace pagedkv

using namespace pagedkv;

extern "C" kv_status kv_selftest_wait_timeout(int32_t *device_status, uint32_t limit_us,
                                              kv_stream_t stream) {
  if (!device_status) return fail(KV_ERR_INVALID, "null device_status");
  if (limit_us == 0 || limit_us > 1000000) return fail(KV_ERR_INVALID, "limit_us must be in [1, 1e6]");
  wait_timeout_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(device_status, (uint64_t)limit_us * 1000ull);
  kv_status s = cuda_check(cudaGetLastError(), "selftest launch");
  return s == KV_OK ? ok() : s;
}
