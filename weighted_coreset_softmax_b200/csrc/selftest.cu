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

namespace kvs {
// Streams `n16` 16-byte words from src with four loads in flight per thread and
// folds them into one word (so the loads cannot be dropped); the word lands in
// *sink only in the impossible case that it equals a fixed constant.
__global__ void __launch_bounds__(256) stream_read_kernel(const uint4* __restrict__ src, size_t n16,
                                                          uint32_t* sink) {
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldcs(src + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldcs(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  if (acc == 0x9e3779b9u) *sink = acc;
}
}  // namespace kvs

extern "C" kv_status kv_stream_read(const void* src, size_t bytes, uint32_t* sink, kv_stream_t stream) {
  if (!src || !sink || (reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(sink) & 3u) ||
      (bytes & 15u)) {
    kvs::set_last_error("kv_stream_read: src must be 16-byte aligned, sink 4-byte aligned, bytes a multiple of 16");
    return KV_ERR_INVALID_ARG;
  }
  if (bytes == 0) return KV_OK;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    kvs::set_last_error("kv_stream_read: no CUDA device");
    return KV_ERR_CUDA;
  }
  kvs::stream_read_kernel<<<sms * 8, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), bytes / 16, sink);
  if (cudaGetLastError() != cudaSuccess) {
    kvs::set_last_error("kv_stream_read: launch failed");
    return KV_ERR_CUDA;
  }
  return KV_OK;
}
