// Launchers of the warp-specialised block-mode attention kernel (bf16 caches,
// D in {64, 128}, G in 1..8, chunks of 32 or 64 rows).
#include <cuda_runtime.h>

#include <atomic>

#include "gather_attn.cuh"

namespace kvs {

template <int D, int G, int ROWS>
static cudaError_t gather_launch_one(const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int grid,
                                     cudaStream_t st) {
  using C = GaCfg<D, G, ROWS>;
  static std::atomic<int> configured{0};  // one bit per device: smem limit raised
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured.load() & (1 << (dev & 31)))) {
    const cudaError_t e =
        cudaFuncSetAttribute(gather_attn_kernel<D, G, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();  // do not leave the failure for an unrelated later check
      return e;
    }
    configured.fetch_or(1 << (dev & 31));
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(GA_THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, gather_attn_kernel<D, G, ROWS>, p, tk, tv);
  if (le != cudaSuccess) {
    (void)cudaGetLastError();
    return le;
  }
  return cudaGetLastError();
}

template <int D, int ROWS>
static cudaError_t gather_launch_d(int G, const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int grid,
                                   cudaStream_t st) {
  switch (G) {
    case 1: return gather_launch_one<D, 1, ROWS>(p, tk, tv, grid, st);
    case 2: return gather_launch_one<D, 2, ROWS>(p, tk, tv, grid, st);
    case 3: return gather_launch_one<D, 3, ROWS>(p, tk, tv, grid, st);
    case 4: return gather_launch_one<D, 4, ROWS>(p, tk, tv, grid, st);
    case 5: return gather_launch_one<D, 5, ROWS>(p, tk, tv, grid, st);
    case 6: return gather_launch_one<D, 6, ROWS>(p, tk, tv, grid, st);
    case 7: return gather_launch_one<D, 7, ROWS>(p, tk, tv, grid, st);
    case 8: return gather_launch_one<D, 8, ROWS>(p, tk, tv, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gather(int D, int G, int rows, const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                          int grid, cudaStream_t st) {
  if (rows == 64)
    return D == 64 ? gather_launch_d<64, 64>(G, p, tk, tv, grid, st) : gather_launch_d<128, 64>(G, p, tk, tv, grid, st);
  return D == 64 ? gather_launch_d<64, 32>(G, p, tk, tv, grid, st) : gather_launch_d<128, 32>(G, p, tk, tv, grid, st);
}

}  // namespace kvs
