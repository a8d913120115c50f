// Per-(type, head dim) launch tables. Included by the instantiation units with
// KVS_T (element type), KVS_D (head dim) and KVS_SUFFIX defined.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <utility>

#include "attention.cuh"
#include "launch.h"
#include "select.cuh"

namespace kvs {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream finishes; it calls grid_dep_wait()
// before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int threads, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises the kernel's dynamic shared-memory limit once per device and returns how
// many CTAs fit on one SM.
template <typename T, int D, int G, bool MMA>
int attn_prepare(int dev) {
  using C = AttnCfg<T, D, G, MMA>;
  static std::atomic<int> blocks_per_sm[64];
  int v = blocks_per_sm[dev & 63].load();
  if (v > 0) return v;
  if (cudaFuncSetAttribute(attn_kernel<T, D, G, MMA, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, attn_kernel<T, D, G, MMA, false>, C::NTHREADS, C::SMEM) !=
      cudaSuccess)
    return 0;
  blocks_per_sm[dev & 63].store(n);
  return n;
}

template <typename T, int D, int G, bool MMA>
cudaError_t attn_launch_one(const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int grid,
                            cudaStream_t st) {
  using C = AttnCfg<T, D, G, MMA>;
  return launch_pdl(attn_kernel<T, D, G, MMA, false>, grid, C::NTHREADS, C::SMEM, st, p, tk, tv);
}

// Tensor-core consumer for bf16 caches, CUDA-core consumer for fp32 (and for
// bf16 when the caller asks for it).
template <typename T>
constexpr bool has_mma() {
  return sizeof(T) == 2;
}

// Fused decode step (bf16, tensor-core consumer, one CTA per bh): does this
// shape fit the in-CTA selection's shared-memory layout (the block logits in one
// ring slot, keys, counts and scratch in another)?
template <typename T, int D, int G>
bool fused_fits(int NBcap) {
  if constexpr (!has_mma<T>()) {
    return false;
  } else {
    using C = AttnCfg<T, D, G, true>;
    const size_t nbp = static_cast<size_t>((NBcap + 31) & ~31);
    return C::NW >= 2 && G * nbp * 4 <= static_cast<size_t>(C::SLOT) &&
           ((nbp * 12 + 15) & ~static_cast<size_t>(15)) + sizeof(RankMisc<C::NTHREADS>) <= static_cast<size_t>(C::SLOT);
  }
}

template <typename T, int D, int G>
cudaError_t fused_launch_one(const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int grid,
                             cudaStream_t st) {
  if constexpr (!has_mma<T>()) {
    return cudaErrorInvalidValue;
  } else {
    using C = AttnCfg<T, D, G, true>;
    static std::atomic<int> configured{0};  // one bit per device: smem limit raised
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(configured.load() & (1 << (dev & 31)))) {
      const cudaError_t e =
          cudaFuncSetAttribute(attn_kernel<T, D, G, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
      if (e != cudaSuccess) return e;
      configured.fetch_or(1 << (dev & 31));
    }
    return launch_pdl(attn_kernel<T, D, G, true, true>, grid, C::NTHREADS, C::SMEM, st, p, tk, tv);
  }
}

#define KVS_G_SWITCH(FN, ...)                      \
  switch (G) {                                      \
    case 1: return FN<T, D, 1>(__VA_ARGS__);        \
    case 2: return FN<T, D, 2>(__VA_ARGS__);        \
    case 3: return FN<T, D, 3>(__VA_ARGS__);        \
    case 4: return FN<T, D, 4>(__VA_ARGS__);        \
    case 5: return FN<T, D, 5>(__VA_ARGS__);        \
    case 6: return FN<T, D, 6>(__VA_ARGS__);        \
    case 7: return FN<T, D, 7>(__VA_ARGS__);        \
    case 8: return FN<T, D, 8>(__VA_ARGS__);        \
    default: break;                                 \
  }


#define KVS_ATTN_SWITCH(FN, ...)                                       \
  switch (G) {                                                         \
    case 1: return use_mma ? FN<T, D, 1, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 1, false>(__VA_ARGS__);          \
    case 2: return use_mma ? FN<T, D, 2, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 2, false>(__VA_ARGS__);          \
    case 3: return use_mma ? FN<T, D, 3, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 3, false>(__VA_ARGS__);          \
    case 4: return use_mma ? FN<T, D, 4, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 4, false>(__VA_ARGS__);          \
    case 5: return use_mma ? FN<T, D, 5, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 5, false>(__VA_ARGS__);          \
    case 6: return use_mma ? FN<T, D, 6, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 6, false>(__VA_ARGS__);          \
    case 7: return use_mma ? FN<T, D, 7, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 7, false>(__VA_ARGS__);          \
    case 8: return use_mma ? FN<T, D, 8, has_mma<T>()>(__VA_ARGS__)     \
                           : FN<T, D, 8, false>(__VA_ARGS__);          \
    default: break;                                                    \
  }

template <typename T, int D>
cudaError_t attn_launch_td(int G, bool use_mma, const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                           int grid, cudaStream_t st) {
  KVS_ATTN_SWITCH(attn_launch_one, p, tk, tv, grid, st)
  return cudaErrorInvalidValue;
}

template <typename T, int D>
int attn_prepare_td(int G, bool use_mma, int dev) {
  KVS_ATTN_SWITCH(attn_prepare, dev)
  return 0;
}

template <typename T, int D, int G, int MODE>
cudaError_t select_launch_mode(const SelParams& p, int grid, cudaStream_t st) {
  static std::atomic<int> configured{0};  // one bit per device: smem limit raised
  int dev = 0;
  cudaGetDevice(&dev);
  if constexpr ((MODE == SEL_QUEST || MODE == SEL_MEAN16 || MODE == SEL_COBS4) && sizeof(T) != 2)
    return cudaErrorInvalidValue;  // bf16 bounds and bf16 means: bf16 caches only
  const size_t smem = MODE != SEL_EXACT ? sel_summary_smem_bytes(G, p.NBcap) : sel_smem_bytes(G, p.NBcap);
  if (!(configured.load() & (1 << (dev & 31)))) {
    size_t most = MODE != SEL_EXACT ? sel_summary_smem_bytes(G, SEL_MAXNB) : sel_smem_bytes(G, SEL_MAXNB);
    if (most > 227 * 1024) most = 227 * 1024;  // per-CTA limit; larger shapes are refused below
    cudaError_t e = cudaFuncSetAttribute(select_kernel<T, D, G, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(most));
    if (e != cudaSuccess) return e;
    configured.fetch_or(1 << (dev & 31));
  }
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  const cudaError_t le = launch_pdl(select_kernel<T, D, G, MODE>, grid, SEL_THREADS, smem, st, p);
  if (le != cudaSuccess) return le;
  return cudaGetLastError();
}

template <typename T, int D, int G>
cudaError_t select_launch_one(int mode, const SelParams& p, int grid, cudaStream_t st) {
  if (mode == SEL_QUEST) {
    if constexpr (sizeof(T) == 2) return select_launch_mode<T, D, G, SEL_QUEST>(p, grid, st);
    return cudaErrorInvalidValue;
  }
  if (mode == SEL_MEAN16) {
    if constexpr (sizeof(T) == 2) return select_launch_mode<T, D, G, SEL_MEAN16>(p, grid, st);
    return cudaErrorInvalidValue;
  }
  if (mode == SEL_COBS4) {
    if constexpr (sizeof(T) == 2) return select_launch_mode<T, D, G, SEL_COBS4>(p, grid, st);
    return cudaErrorInvalidValue;
  }
  if (mode == SEL_COBS) return select_launch_mode<T, D, G, SEL_COBS>(p, grid, st);
  return mode == SEL_SUMMARY ? select_launch_mode<T, D, G, SEL_SUMMARY>(p, grid, st)
                             : select_launch_mode<T, D, G, SEL_EXACT>(p, grid, st);
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
bool KVS_CAT(fused_fits_, KVS_SUFFIX)(int G, int NBcap) {
  using T = KVS_T;
  constexpr int D = KVS_D;
  KVS_G_SWITCH(fused_fits, NBcap)
  return false;
}
cudaError_t KVS_CAT(fused_launch_, KVS_SUFFIX)(int G, const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                                int grid, cudaStream_t st) {
  using T = KVS_T;
  constexpr int D = KVS_D;
  KVS_G_SWITCH(fused_launch_one, p, tk, tv, grid, st)
  return cudaErrorInvalidValue;
}
cudaError_t KVS_CAT(attn_launch_, KVS_SUFFIX)(int G, bool use_mma, const AttnParams& p, const CUtensorMap& tk,
                                               const CUtensorMap& tv, int grid, cudaStream_t st) {
  return attn_launch_td<KVS_T, KVS_D>(G, use_mma, p, tk, tv, grid, st);
}
int KVS_CAT(attn_prepare_, KVS_SUFFIX)(int G, bool use_mma, int dev) {
  return attn_prepare_td<KVS_T, KVS_D>(G, use_mma, dev);
}
cudaError_t KVS_CAT(select_launch_, KVS_SUFFIX)(int G, int mode, const SelParams& p, int grid, cudaStream_t st) {
  return select_launch_td<KVS_T, KVS_D>(G, mode, p, grid, st);
}
}  // namespace kvs
