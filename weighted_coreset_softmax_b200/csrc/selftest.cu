// kv_selftest_wait_timeout: exercises the kernels' failure-detection path -- a
// bounded wait on an mbarrier that gives up, flags KV_DEV_WAIT_TIMEOUT in a
// status word and returns -- without any fault: the barrier is armed for bytes
// that no copy will ever deliver (no copy is issued), so nothing is in flight
// when the wait gives up and the kernel exits normally.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kvsparse.h"

namespace kvs {
void set_last_error(const char* msg);

// One warp. arrive != 0: the expected bytes are cancelled by a plain arrival
// with no transaction count, so the phase completes and the wait succeeds.
// arrive == 0: the phase waits for 16 bytes that never come; the wait gives up
// after limit_ns. out[0] = 1 if the wait succeeded, 0 if it gave up.
__global__ void __launch_bounds__(32) selftest_wait_kernel(uint32_t* status, uint32_t* out, uint64_t limit_ns,
                                                           int arrive) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    if (arrive)
      mbar_arrive(&bar);                 // the phase's one arrival, no bytes expected
    else
      mbar_arrive_expect_tx(&bar, 16u);  // the arrival, plus 16 bytes that never land
  }
  __syncwarp();
  const bool ok = mbar_wait_for(&bar, 0u, threadIdx.x == 0 ? status : nullptr, limit_ns);
  __syncwarp();
  if (threadIdx.x == 0) out[0] = ok ? 1u : 0u;
}
}  // namespace kvs

extern "C" kv_status kv_selftest_wait_timeout(uint32_t* status, uint32_t* waited_ok, uint64_t limit_ns, int arrive,
                                              kv_stream_t stream) {
  if (!status || !waited_ok) {
    kvs::set_last_error("kv_selftest_wait_timeout: status and waited_ok must be device pointers");
    return KV_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(status) & 3u) || (reinterpret_cast<uintptr_t>(waited_ok) & 3u)) {
    kvs::set_last_error("kv_selftest_wait_timeout: status and waited_ok must be 4-byte aligned");
    return KV_ERR_INVALID_ARG;
  }
  if (limit_ns == 0 || limit_ns > 2000000000ull) {
    kvs::set_last_error("kv_selftest_wait_timeout: limit_ns must lie in (0, 2e9]");
    return KV_ERR_INVALID_ARG;
  }
  kvs::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, waited_ok, limit_ns,
                                                                                   arrive ? 1 : 0);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    kvs::set_last_error("kv_selftest_wait_timeout: launch failed");
    return KV_ERR_CUDA;
  }
  return KV_OK;
}
