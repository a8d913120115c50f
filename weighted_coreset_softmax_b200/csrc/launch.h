// Launchers of the kvsparse kernels. Each is instantiated in its own
// translation unit per (element type, head dimension) so the build parallelises.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "partition.h"

namespace kvs {

struct AttnParams;
struct SelParams;

// dtype: 0 = bf16, 1 = fp32. Return cudaSuccess or the launch error.
// use_mma: tensor-core consumer (bf16 only; ignored for fp32).
cudaError_t launch_attn(int dtype, int D, int G, bool use_mma, const AttnParams& p, const CUtensorMap& tk,
                        const CUtensorMap& tv, int grid, cudaStream_t st);
// CTAs of the attention kernel that fit on one SM (0 on error).
int attn_ctas_per_sm(int dtype, int D, int G, bool use_mma, int dev);
// Fused decode step (selection + attention in one kernel, one CTA per bh).
bool fused_fits(int dtype, int D, int G, int NBcap);
cudaError_t launch_fused(int dtype, int D, int G, const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                         int grid, cudaStream_t st);
// Warp-specialised block-mode attention (bf16, tensor cores, block size >= 32):
// one CTA per SM, grid <= number of SMs; rows = min(block size, 64) a chunk, with
// tensor maps whose boxes are one rows x D tile (3-D for D = 128).
cudaError_t launch_gather(int D, int G, int rows, const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                          int grid, cudaStream_t st);
cudaError_t launch_select(int dtype, int D, int G, int mode, const SelParams& p, int grid, cudaStream_t st);
// Few pairs: each pair's blocks over a cluster of S CTAs (summary and bf16-mean modes,
// k_top <= 16); cudaErrorInvalidValue when the shape is not covered.
cudaError_t launch_select_split(int dtype, int D, int G, int mode, const SelParams& p, int NBH, int S,
                                cudaStream_t st);
cudaError_t launch_sums(int dtype, int D, const void* K, const void* V, const int32_t* seq_lens, float* k_sum,
                        float* v_sum, int32_t* counts, float* k_tot, float* v_tot, int NBH, int Hkv, int Ncap,
                        int L, int NBcap, cudaStream_t st);

}  // namespace kvs
