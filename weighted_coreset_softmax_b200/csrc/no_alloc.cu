// kv_sparse_decode_attn_noalloc: the sparse decode-attention kernel with its
// scratch memory taken from a fixed array that lives inside this library, for
// callers that cannot allocate device memory.
//
// Who needs it: code that is handed only input and output pointers and may not
// call cudaMalloc or any allocator itself -- for example a plugin or custom
// operator inside a host framework that owns all device memory, or a serving
// process that reserves its whole memory budget up front and forbids allocation
// on the request path. Such callers cannot provide the workspace that
// kv_sparse_decode_attn asks for, so this entry point brings its own.
//
// The scratch is one file-scope __device__ array of KV_NOALLOC_SCRATCH_BYTES
// (16 MiB). Every GPU that loads the library holds it until the process exits.
// Host code cannot use the array's name as a device address, so the first call
// on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it; make that first call before capturing any
// stream into a CUDA graph. All calls on a device share the array and it keeps
// the previous call's contents: each call, once its arguments have passed every
// check, clears the parts that must start at zero (status word and arrival
// counters) with an async memset on the caller's stream. Two calls whose kernels overlap on the GPU (different streams without
// ordering) race on the shared array and give wrong results; order them.
// Device-side index checks still skip bad entries, but their status bits are
// cleared by the next call and are not reported here.
#include <cuda_runtime.h>

#include <mutex>

#include "kvsparse.h"
#include "partition.h"

namespace kvs {
void set_last_error(const char* msg);
kv_status sparse_attn_check(const kv_shape* shape, const void* q, float scale, const void* K, const void* V,
                            const int32_t* block_idx, const int32_t* n_kept, int kmax, const float* k_sum,
                            const float* v_sum, const int32_t* counts, const float* k_tot, const float* v_tot,
                            int use_tail_proxy, const int32_t* tok_idx, const float* w, int m, float* out, float* lse,
                            void* workspace, size_t ws_bytes);
}

namespace {

constexpr size_t KV_NOALLOC_SCRATCH_BYTES = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[KV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
kv_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    kvs::set_last_error("kv_sparse_decode_attn_noalloc: cudaGetDevice failed");
    return KV_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    kvs::set_last_error("kv_sparse_decode_attn_noalloc: device index out of range");
    return KV_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      kvs::set_last_error("kv_sparse_decode_attn_noalloc: cudaGetSymbolAddress of the scratch array failed");
      return KV_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KV_OK;
}

}  // namespace

extern "C" kv_status kv_sparse_decode_attn_noalloc(
    const kv_shape* shape, const void* q, float scale, const void* K, const void* V, const int32_t* block_idx,
    const int32_t* n_kept, int kmax, const float* k_sum, const float* v_sum, const int32_t* counts,
    const float* k_tot, const float* v_tot, int use_tail_proxy, const int32_t* tok_idx, const float* w, int m,
    float* out, float* lse, kv_stream_t stream) {
  if (!shape) {
    kvs::set_last_error("shape is NULL");
    return KV_ERR_INVALID_ARG;
  }
  const size_t need = kv_workspace_bytes(shape);
  if (need > KV_NOALLOC_SCRATCH_BYTES) {
    kvs::set_last_error(
        "kv_sparse_decode_attn_noalloc: this shape needs more scratch than the fixed 16 MiB array "
        "(reduce B * Hkv, or use kv_sparse_decode_attn with a caller-provided workspace)");
    return KV_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  kv_status st = scratch_address(&scratch);
  if (st != KV_OK) return st;
  // every argument check first: a call that is rejected enqueues nothing (not
  // even the clearing memset below, which would disturb a call still in flight)
  st = kvs::sparse_attn_check(shape, q, scale, K, V, block_idx, n_kept, kmax, k_sum, v_sum, counts, k_tot, v_tot,
                              use_tail_proxy, tok_idx, w, m, out, lse, scratch, KV_NOALLOC_SCRATCH_BYTES);
  if (st != KV_OK) return st;
  if (need > 0 && shape->B > 0 && shape->Hkv > 0) {
    // status word and arrival counters must start at zero
    const size_t zero_bytes = kvs::ws_records_off(shape->B * shape->Hkv);
    cudaError_t e = cudaMemsetAsync(scratch, 0, zero_bytes, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
      kvs::set_last_error("kv_sparse_decode_attn_noalloc: clearing the scratch counters failed");
      return KV_ERR_CUDA;
    }
  }
  return kv_sparse_decode_attn(shape, q, scale, K, V, block_idx, n_kept, kmax, k_sum, v_sum, counts, k_tot, v_tot,
                               use_tail_proxy, tok_idx, w, m, out, lse, scratch, KV_NOALLOC_SCRATCH_BYTES, stream);
}
