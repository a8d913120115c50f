// Per-(type, head dim) launch tables. Included by the instantiation units with
// KVS_T (element type), KVS_D (head dim) and KVS_SUFFIX defined.
#pragma once

#include <cuda_runtime.h>

#include <atomic>

#include "attention.cuh"
#include "launch.h"
#include "select.cuh"

namespace kvs {

template <typename T, int D, int G>
cudaError_t attn_launch_one(const AttnParams& p, int grid, cudaStream_t st) {
  using C = AttnCfg<T, D, G>;
  static std::atomic<int> configured_mask{0};  // one bit per device: smem limit raised
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured_mask & (1 << (dev & 31)))) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    configured_mask.fetch_or(1 << (dev & 31));
  }
  attn_kernel<T, D, G><<<grid, C::NTHREADS, C::SMEM, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t attn_launch_td(int G, const AttnParams& p, int grid, cudaStream_t st) {
  switch (G) {
    case 1: return attn_launch_one<T, D, 1>(p, grid, st);
    case 2: return attn_launch_one<T, D, 2>(p, grid, st);
    case 3: return attn_launch_one<T, D, 3>(p, grid, st);
    case 4: return attn_launch_one<T, D, 4>(p, grid, st);
    case 5: return attn_launch_one<T, D, 5>(p, grid, st);
    case 6: return attn_launch_one<T, D, 6>(p, grid, st);
    case 7: return attn_launch_one<T, D, 7>(p, grid, st);
    case 8: return attn_launch_one<T, D, 8>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

// CTAs per SM the attention kernel is built for (its launch bound).
template <typename T, int D>
int attn_cps_td(int G) {
  switch (G) {
    case 1: return AttnCfg<T, D, 1>::CPS;
    case 2: return AttnCfg<T, D, 2>::CPS;
    case 3: return AttnCfg<T, D, 3>::CPS;
    case 4: return AttnCfg<T, D, 4>::CPS;
    case 5: return AttnCfg<T, D, 5>::CPS;
    case 6: return AttnCfg<T, D, 6>::CPS;
    case 7: return AttnCfg<T, D, 7>::CPS;
    case 8: return AttnCfg<T, D, 8>::CPS;
    default: return 1;
  }
}

template <typename T, int D, int G>
cudaError_t select_launch_one(int mode, const SelParams& p, int grid, cudaStream_t st) {
  if (mode == SEL_SUMMARY)
    select_kernel<T, D, G, SEL_SUMMARY><<<grid, SEL_THREADS, 0, st>>>(p);
  else
    select_kernel<T, D, G, SEL_EXACT><<<grid, SEL_THREADS, 0, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t select_launch_td(int G, int mode, const SelParams& p, int grid, cudaStream_t st) {
  switch (G) {
    case 1: return select_launch_one<T, D, 1>(mode, p, grid, st);
    case 2: return select_launch_one<T, D, 2>(mode, p, grid, st);
    case 3: return select_launch_one<T, D, 3>(mode, p, grid, st);
    case 4: return select_launch_one<T, D, 4>(mode, p, grid, st);
    case 5: return select_launch_one<T, D, 5>(mode, p, grid, st);
    case 6: return select_launch_one<T, D, 6>(mode, p, grid, st);
    case 7: return select_launch_one<T, D, 7>(mode, p, grid, st);
    case 8: return select_launch_one<T, D, 8>(mode, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvs

#define KVS_CAT2(a, b) a##b
#define KVS_CAT(a, b) KVS_CAT2(a, b)

// Exported (internal) entry points of this unit.
namespace kvs {
cudaError_t KVS_CAT(attn_launch_, KVS_SUFFIX)(int G, const AttnParams& p, int grid, cudaStream_t st) {
  return attn_launch_td<KVS_T, KVS_D>(G, p, grid, st);
}
int KVS_CAT(attn_cps_, KVS_SUFFIX)(int G) { return attn_cps_td<KVS_T, KVS_D>(G); }
cudaError_t KVS_CAT(select_launch_, KVS_SUFFIX)(int G, int mode, const SelParams& p, int grid, cudaStream_t st) {
  return select_launch_td<KVS_T, KVS_D>(G, mode, p, grid, st);
}
}  // namespace kvs
