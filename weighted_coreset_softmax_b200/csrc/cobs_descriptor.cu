// The stored second-order block descriptor of "COBS: Cumulant Order Block Sparse
// Attention" (the subspace and quantisation paragraphs), built once after prefill
// (the basis once per model head, from calibration queries):
//   kv_build_query_basis            eigenvectors / eigenvalues of each KV head's query
//                                   second moment (float64 Jacobi, one CTA a head)
//   kv_query_subspace_rank          s: the rank reaching a share of the spectral energy
//                                   per head, averaged over heads and rounded up (host)
//   kv_build_block_cov_factors_ss   rank-r factors of U Sigma_b U^T per block
//   kv_quantize_fp4                 E2M1 FP4 codes with one fp32 scale per vector
// The selector that reads the descriptor is kv_select_blocks_cobs_fp4.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "covariance.cuh"
#include "kvsparse.h"

namespace kvs {
void set_last_error(const char* msg);

// E2M1 code of x / scale: the nearest of the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6,
// a tie to the code with mantissa bit 0, the sign in bit 3 (zero keeps code 0).
// The quotient is an IEEE division, so a float32 reference takes the same decision.
__device__ __forceinline__ uint32_t e2m1_code(float x, float scale) {
  if (!(scale > 0.f)) return 0u;
  const float qv = __fdiv_rn(x, scale);
  const float a = fabsf(qv);
  uint32_t c = a <= 0.25f ? 0u
             : a < 0.75f  ? 1u
             : a <= 1.25f ? 2u
             : a < 1.75f  ? 3u
             : a <= 2.5f  ? 4u
             : a < 3.5f   ? 5u
             : a <= 5.f   ? 6u
                          : 7u;
  if (qv < 0.f && c != 0u) c |= 8u;
  return c;
}

// One warp per vector of len fp32 values (len even): scale = max|x| / 6, then one
// byte per pair of elements (element 2j in the low nibble).
__global__ void fp4_quantize_kernel(const float* __restrict__ x, long long nvec, int len, uint8_t* __restrict__ codes,
                                    float* __restrict__ scales) {
  const long long v = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (v >= nvec) return;  // warp-uniform
  const float* xv = x + v * len;
  float amax = 0.f;
  for (int j = lane; j < len; j += 32) amax = fmaxf(amax, fabsf(xv[j]));
  amax = warp_max(amax);
  const float scale = __fdiv_rn(amax, 6.0f);
  if (lane == 0) scales[v] = scale > 0.f ? scale : 0.f;
  uint8_t* cv = codes + v * (len / 2);
  for (int j = lane; j < len / 2; j += 32)
    cv[j] = static_cast<uint8_t>(e2m1_code(xv[2 * j], scale) | (e2m1_code(xv[2 * j + 1], scale) << 4));
}

template <typename T, int D>
static cudaError_t basis_td(const void* Qc, int Nc, int Hq, int Hkv, float* evecs, float* evals, double* vws,
                            cudaStream_t st) {
  static std::atomic<int> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured.load() & (1 << (dev & 31)))) {
    const cudaError_t e = cudaFuncSetAttribute(query_basis_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(qb_smem_bytes(D)));
    if (e != cudaSuccess) return e;
    configured.fetch_or(1 << (dev & 31));
  }
  query_basis_kernel<T, D><<<Hkv, COV_THREADS, qb_smem_bytes(D), st>>>(static_cast<const T*>(Qc), Nc, Hq, Hkv, evecs,
                                                                      evals, vws);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t cov_ss_td(const void* K, const int32_t* seq_lens, float* xi, int NBH, int Hkv, int Ncap, int L,
                             int NBcap, int r, const float* U, int s_dim, int SP, cudaStream_t st) {
  static std::atomic<int> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured.load() & (1 << (dev & 31)))) {
    const cudaError_t e = cudaFuncSetAttribute(cov_factors_kernel<T, D, true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(cov_smem_bytes(COV_MAX_ROWS, D, D)));
    if (e != cudaSuccess) return e;
    configured.fetch_or(1 << (dev & 31));
  }
  const long long grid = static_cast<long long>(NBH) * NBcap;
  cov_factors_kernel<T, D, true><<<static_cast<unsigned>(grid), COV_THREADS, cov_smem_bytes(L, D, s_dim), st>>>(
      static_cast<const T*>(K), seq_lens, xi, Hkv, Ncap, L, NBcap, r, U, s_dim, SP);
  return cudaGetLastError();
}
}  // namespace kvs

namespace {
kv_status bad(kv_status s, const char* msg) {
  kvs::set_last_error(msg);
  return s;
}
bool aligned(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

extern "C" {

size_t kv_query_basis_workspace_bytes(int Hkv, int D) {
  if (Hkv < 1 || (D != 64 && D != 128)) return 0;
  return static_cast<size_t>(Hkv) * D * (D + 1) * sizeof(double);
}

kv_status kv_build_query_basis(const void* Qc, kv_dtype dtype, int Nc, int Hq, int Hkv, int D, float* evecs,
                               float* evals, void* workspace, size_t ws_bytes, kv_stream_t stream) {
  if (D != 64 && D != 128) return bad(KV_ERR_UNSUPPORTED, "kv_build_query_basis: head dim D must be 64 or 128");
  if (dtype != KV_BF16 && dtype != KV_F32) return bad(KV_ERR_INVALID_ARG, "kv_build_query_basis: unknown dtype");
  if (Nc < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0)
    return bad(KV_ERR_INVALID_ARG, "kv_build_query_basis: need Nc >= 1 and Hq a multiple of Hkv");
  if (static_cast<long long>(Nc) * (Hq / Hkv) > (1LL << 30))
    return bad(KV_ERR_INVALID_ARG, "kv_build_query_basis: too many calibration rows");
  if (!aligned(Qc, 16)) return bad(KV_ERR_INVALID_ARG, "kv_build_query_basis: Qc NULL or not 16-byte aligned");
  if (!aligned(evecs, 4) || !aligned(evals, 4))
    return bad(KV_ERR_INVALID_ARG, "kv_build_query_basis: evecs or evals NULL or misaligned");
  if (!aligned(workspace, 16)) return bad(KV_ERR_INVALID_ARG, "kv_build_query_basis: workspace NULL or misaligned");
  if (ws_bytes < kv_query_basis_workspace_bytes(Hkv, D))
    return bad(KV_ERR_INVALID_ARG, "kv_build_query_basis: workspace too small");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  double* vws = static_cast<double*>(workspace);
  cudaError_t e;
  if (dtype == KV_BF16)
    e = D == 64 ? kvs::basis_td<__nv_bfloat16, 64>(Qc, Nc, Hq, Hkv, evecs, evals, vws, st)
                : kvs::basis_td<__nv_bfloat16, 128>(Qc, Nc, Hq, Hkv, evecs, evals, vws, st);
  else
    e = D == 64 ? kvs::basis_td<float, 64>(Qc, Nc, Hq, Hkv, evecs, evals, vws, st)
                : kvs::basis_td<float, 128>(Qc, Nc, Hq, Hkv, evecs, evals, vws, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return bad(KV_ERR_CUDA, "kv_build_query_basis: launch failed");
  }
  return KV_OK;
}

int kv_query_subspace_rank(const float* evals, int Hkv, int D, double energy) {
  if (!evals || Hkv < 1 || D < 1 || !(energy > 0.0) || energy > 1.0) return -1;
  long long total = 0;
  for (int h = 0; h < Hkv; ++h) {
    const float* lam = evals + static_cast<size_t>(h) * D;
    double tot = 0.0;
    for (int j = 0; j < D; ++j) tot += static_cast<double>(lam[j]);
    double acc = 0.0;
    int pick = D;
    for (int j = 0; j < D; ++j) {
      acc += static_cast<double>(lam[j]);
      if (acc >= energy * tot) {
        pick = j + 1;
        break;
      }
    }
    total += pick;
  }
  return static_cast<int>((total + Hkv - 1) / Hkv);  // ceil of the mean
}

kv_status kv_build_block_cov_factors_ss(const kv_shape* shape, const void* K, const float* U, int s, int rank,
                                        float* xi_ss, kv_stream_t stream) {
  if (!shape) return bad(KV_ERR_INVALID_ARG, "kv_build_block_cov_factors_ss: shape is NULL");
  if (shape->B < 0 || shape->Hkv < 1 || shape->Ncap < 1 || shape->block_size < 1)
    return bad(KV_ERR_INVALID_ARG, "kv_build_block_cov_factors_ss: bad shape");
  if (shape->D != 64 && shape->D != 128)
    return bad(KV_ERR_UNSUPPORTED, "kv_build_block_cov_factors_ss: head dim D must be 64 or 128");
  if (shape->block_size > kvs::COV_MAX_ROWS)
    return bad(KV_ERR_UNSUPPORTED, "kv_build_block_cov_factors_ss: block_size above 64");
  if (shape->dtype != KV_BF16 && shape->dtype != KV_F32)
    return bad(KV_ERR_INVALID_ARG, "kv_build_block_cov_factors_ss: unknown dtype");
  if (rank < 1 || rank > kvs::COV_MAX_RANK) return bad(KV_ERR_INVALID_ARG, "kv_build_block_cov_factors_ss: rank outside 1..8");
  if (s < 1 || s > shape->D) return bad(KV_ERR_INVALID_ARG, "kv_build_block_cov_factors_ss: s outside 1..D");
  if (shape->B > 0 && !aligned(shape->seq_lens, 4))
    return bad(KV_ERR_INVALID_ARG, "kv_build_block_cov_factors_ss: seq_lens NULL or misaligned");
  if (!aligned(K, 16) || !aligned(U, 4) || !aligned(xi_ss, 16))
    return bad(KV_ERR_INVALID_ARG, "kv_build_block_cov_factors_ss: K, U or xi_ss NULL or misaligned");
  const int NBH = shape->B * shape->Hkv;
  if (NBH == 0) return KV_OK;
  const int L = shape->block_size;
  const int NBcap = (shape->Ncap + L - 1) / L;
  const int SP = (s + 31) & ~31;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (shape->dtype == KV_BF16)
    e = shape->D == 64
            ? kvs::cov_ss_td<__nv_bfloat16, 64>(K, shape->seq_lens, xi_ss, NBH, shape->Hkv, shape->Ncap, L, NBcap,
                                                rank, U, s, SP, st)
            : kvs::cov_ss_td<__nv_bfloat16, 128>(K, shape->seq_lens, xi_ss, NBH, shape->Hkv, shape->Ncap, L, NBcap,
                                                 rank, U, s, SP, st);
  else
    e = shape->D == 64 ? kvs::cov_ss_td<float, 64>(K, shape->seq_lens, xi_ss, NBH, shape->Hkv, shape->Ncap, L, NBcap,
                                                   rank, U, s, SP, st)
                       : kvs::cov_ss_td<float, 128>(K, shape->seq_lens, xi_ss, NBH, shape->Hkv, shape->Ncap, L,
                                                    NBcap, rank, U, s, SP, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return bad(KV_ERR_CUDA, "kv_build_block_cov_factors_ss: launch failed");
  }
  return KV_OK;
}

kv_status kv_quantize_fp4(const float* x, long long nvec, int len, uint8_t* codes, float* scales,
                          kv_stream_t stream) {
  if (nvec < 0 || len < 32 || len % 32 != 0 || len > 4096)
    return bad(KV_ERR_INVALID_ARG, "kv_quantize_fp4: len must be a multiple of 32 in 32..4096");
  if (nvec == 0) return KV_OK;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4))
    return bad(KV_ERR_INVALID_ARG, "kv_quantize_fp4: x, codes or scales NULL or misaligned");
  constexpr int WPB = 8;  // warps (vectors) a CTA
  const long long grid = (nvec + WPB - 1) / WPB;
  if (grid > 0x7fffffffLL) return bad(KV_ERR_INVALID_ARG, "kv_quantize_fp4: too many vectors");
  kvs::fp4_quantize_kernel<<<static_cast<unsigned>(grid), WPB * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, nvec, len, codes, scales);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return bad(KV_ERR_CUDA, "kv_quantize_fp4: launch failed");
  return KV_OK;
}

}  // extern "C"
