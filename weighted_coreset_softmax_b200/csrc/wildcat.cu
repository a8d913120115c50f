// kv_build_wildcat_coreset: a weighted coreset of each (sequence, KV head)'s keys,
// for the weighted-coreset mode of kv_sparse_decode_attn.
//
// Method: "WildCat: Near-Linear Attention in Theory and Practice", abstract -- the
// coreset is selected by randomly pivoted Cholesky and its elements are weighted
// to minimise the reconstruction error. Readings (the abstract does not fix them):
// the kernel is attention's exponential kernel on the keys, exp(scale k_i . k_j),
// shifted by the constant scale * max_i |k_i|^2 so that every entry lies in (0, 1]
// (the shift cancels in the pivot draws and in the weights); the error is the
// kernel distance between the sum over all tokens and the weighted coreset, whose
// minimiser w solves A_SS w = A_{S,:} 1; a negative weight is clipped to 0 (the
// attention takes ln w); the uniforms of the pivot draws are inputs.
//
// One CTA per pair runs the m sequential pivot steps. Step t: the residual diagonal
// d is scanned in index order (each thread a contiguous segment, then a CTA scan of
// the segment sums) and the pivot is the first index whose running sum reaches
// u_t times the total; the pivot's residual kernel column g = A[:, s] - F[:, :t]
// F[s, :t]^T becomes factor column t = g / sqrt(g[s]); d drops by its square and
// the column's sum is kept. The factor lives in the workspace as F[t][i] (token
// index fastest, so a warp's reads of one column are contiguous). With the pivots'
// rows F_S (lower triangular in pivot order: a column is zero at every earlier
// pivot), A_SS = F_S F_S^T and A_{S,:} = F_S F^T exactly, so w = F_S^-T (F^T 1): one
// back substitution. Bytes per pair and step: the n keys (for the kernel column) and
// t factor columns; the build runs once after prefill.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>

#include "common.cuh"
#include "kvsparse.h"

namespace kvs {
void set_last_error(const char* msg);

constexpr int WC_THREADS = 512;
constexpr int WC_NW = WC_THREADS / 32;
constexpr int WC_MAX_M = 4096;

template <typename T, int D>
__device__ __forceinline__ float wc_dot(const T* a, const float* b_smem) {
  // row a (global, 16-byte aligned) . b (fp32 in shared memory)
  constexpr int CH = 16 / sizeof(T);
  float acc = 0.f;
#pragma unroll 4
  for (int c = 0; c < D / CH; ++c) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(a) + c);
    float2 f[CH / 2];
    Chunk<T>::unpack(raw, f);
#pragma unroll
    for (int e = 0; e < CH / 2; ++e) {
      acc = fmaf(f[e].x, b_smem[c * CH + 2 * e], acc);
      acc = fmaf(f[e].y, b_smem[c * CH + 2 * e + 1], acc);
    }
  }
  return acc;
}

// Inclusive sum of one value per thread over the CTA; *total gets the CTA's sum.
__device__ __forceinline__ float wc_scan(float v, float* wsum, float* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float x = __shfl_up_sync(FULL_MASK, v, o);
    if (lane >= o) v += x;
  }
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float s = lane < WC_NW ? wsum[lane] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float x = __shfl_up_sync(FULL_MASK, s, o);
      if (lane >= o) s += x;
    }
    if (lane < WC_NW) wsum[lane] = s;
  }
  __syncthreads();
  const float pre = warp > 0 ? wsum[warp - 1] : 0.f;
  *total = wsum[WC_NW - 1];
  __syncthreads();
  return pre + v;
}

__device__ __forceinline__ float wc_sum(float v, float* wsum) {
  float total;
  wc_scan(v, wsum, &total);
  return total;
}

template <typename T, int D>
__global__ void __launch_bounds__(WC_THREADS) wildcat_kernel(const T* __restrict__ K, const int32_t* seq_lens,
                                                             int Hkv, int Ncap, int m, float scale,
                                                             const float* __restrict__ u, int32_t* tok_idx, float* w,
                                                             int32_t* n_sel, float* ws) {
  __shared__ float ks[D];
  __shared__ float wsum[WC_NW];
  __shared__ float fs_row[WC_MAX_M];  // F[j][s] of the current pivot, j < t; later the column sums
  __shared__ int piv, piv_fb;
  __shared__ float gpiv;
  __shared__ float Msh;
  const int bh = blockIdx.x, b = bh / Hkv;
  const int tid = threadIdx.x;
  const int n = max(0, min(seq_lens[b], Ncap));
  const T* Kb = K + static_cast<size_t>(bh) * Ncap * D;
  float* F = ws + static_cast<size_t>(bh) * (static_cast<size_t>(m) + 1) * Ncap;  // F[t][i], t < m
  float* d = F + static_cast<size_t>(m) * Ncap;                                   // residual diagonal
  int32_t* idx_out = tok_idx + static_cast<size_t>(bh) * m;
  float* w_out = w + static_cast<size_t>(bh) * m;
  const float* ub = u + static_cast<size_t>(bh) * m;

  // the shift: M = max_i |k_i|^2; d_i = exp(scale |k_i|^2 - scale M)
  float mx = 0.f;
  for (int i = tid; i < n; i += WC_THREADS) {
    const T* row = Kb + static_cast<size_t>(i) * D;
    float sq = 0.f;
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      const float x = load_as_float(row + c);
      sq = fmaf(x, x, sq);
    }
    d[i] = sq;
    mx = fmaxf(mx, sq);
  }
  mx = warp_max(mx);
  if ((tid & 31) == 0) wsum[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    float M = 0.f;
    for (int q = 0; q < WC_NW; ++q) M = fmaxf(M, wsum[q]);
    Msh = M;
  }
  __syncthreads();
  const float sM = scale * Msh;
  for (int i = tid; i < n; i += WC_THREADS) d[i] = __expf(scale * d[i] - sM);
  __syncthreads();

  const int seg = (n + WC_THREADS - 1) / WC_THREADS;  // contiguous indices per thread
  const int lo = tid * seg, hi = min(n, lo + seg);
  int taken = 0;
  for (int t = 0; t < m; ++t) {
    // ---- pivot: first index whose running sum of d reaches u_t * total
    float part = 0.f;
    for (int i = lo; i < hi; ++i) part += d[i];
    float total;
    const float incl = wc_scan(part, wsum, &total);
    if (!(total > 0.f)) break;  // uniform: the residual is zero (or n = 0)
    const float target = ub[t] * total;
    const float pre = incl - part;
    // the smallest index whose running sum (segment prefix + the segment's own
    // running sum) reaches the target; the minimum over threads keeps the choice
    // deterministic where rounding lets two segments reach it
    if (tid == 0) {
      piv = INT_MAX;
      piv_fb = -1;
    }
    __syncthreads();
    {
      float acc = pre;
      int last_pos = -1;
      for (int i = lo; i < hi; ++i) {
        const float x = d[i];
        if (x > 0.f) last_pos = i;
        acc += x;
        if (x > 0.f && acc >= target) {
          atomicMin(&piv, i);
          break;
        }
      }
      if (last_pos >= 0) atomicMax(&piv_fb, last_pos);
    }
    __syncthreads();
    if (tid == 0 && piv == INT_MAX) piv = piv_fb;  // rounding kept every running sum short: the last positive entry
    __syncthreads();
    const int s = piv;
    if (s < 0) break;  // uniform
    // ---- the pivot's key and its row of the factor so far
    for (int c = tid; c < D; c += WC_THREADS) ks[c] = load_as_float(Kb + static_cast<size_t>(s) * D + c);
    for (int j = tid; j < t; j += WC_THREADS) fs_row[j] = F[static_cast<size_t>(j) * Ncap + s];
    __syncthreads();
    // ---- residual kernel column g into F[t]
    for (int i = tid; i < n; i += WC_THREADS) {
      float g = __expf(scale * wc_dot<T, D>(Kb + static_cast<size_t>(i) * D, ks) - sM);
      for (int j = 0; j < t; ++j) g = fmaf(-F[static_cast<size_t>(j) * Ncap + i], fs_row[j], g);
      F[static_cast<size_t>(t) * Ncap + i] = g;
      if (i == s) gpiv = g;
    }
    __syncthreads();
    const float gp = gpiv;
    if (!(gp > 0.f)) break;  // uniform: no residual left at the pivot
    const float inv = rsqrtf(gp);
    float csum = 0.f;
    for (int i = tid; i < n; i += WC_THREADS) {
      const float f = F[static_cast<size_t>(t) * Ncap + i] * inv;
      F[static_cast<size_t>(t) * Ncap + i] = f;
      d[i] = i == s ? 0.f : fmaxf(d[i] - f * f, 0.f);
      csum += f;
    }
    csum = wc_sum(csum, wsum);
    if (tid == 0) {
      idx_out[t] = s;
      w_out[t] = csum;  // F^T 1, replaced by the weight below
    }
    taken = t + 1;
    __syncthreads();
  }

  // ---- weights: F_S^T w = F^T 1 (F_S[r][c] = F[c][S_r], lower triangular), one
  // back substitution by warp 0; the right-hand side was left in w_out
  __syncthreads();
  for (int r = tid; r < taken; r += WC_THREADS) fs_row[r] = w_out[r];
  __syncthreads();
  if (tid < 32) {
    const int lane = tid;
    for (int c = taken - 1; c >= 0; --c) {
      // w_c = (rhs_c - sum_{r > c} F_S[r][c] w_r) / F_S[c][c]
      float acc = 0.f;
      for (int r = c + 1 + lane; r < taken; r += 32)
        acc = fmaf(F[static_cast<size_t>(c) * Ncap + idx_out[r]], fs_row[r], acc);
      acc = warp_sum(acc);
      if (lane == 0) fs_row[c] = (fs_row[c] - acc) / F[static_cast<size_t>(c) * Ncap + idx_out[c]];
      __syncwarp();
    }
  }
  __syncthreads();
  for (int r = tid; r < m; r += WC_THREADS) {
    if (r < taken) {
      w_out[r] = fmaxf(fs_row[r], 0.f);
    } else {
      idx_out[r] = 0;
      w_out[r] = 0.f;
    }
  }
  if (tid == 0 && n_sel) n_sel[bh] = taken;
}

template <typename T, int D>
static cudaError_t wildcat_launch(const kv_shape* s, const void* K, float scale, int m, const float* u,
                                  int32_t* tok_idx, float* w, int32_t* n_sel, float* ws, cudaStream_t st) {
  wildcat_kernel<T, D><<<s->B * s->Hkv, WC_THREADS, 0, st>>>(static_cast<const T*>(K), s->seq_lens, s->Hkv, s->Ncap,
                                                             m, scale, u, tok_idx, w, n_sel, ws);
  return cudaGetLastError();
}
}  // namespace kvs

extern "C" size_t kv_wildcat_workspace_bytes(const kv_shape* shape, int m) {
  if (!shape || m < 1 || shape->B < 0 || shape->Hkv < 1 || shape->Ncap < 1) return 0;
  return static_cast<size_t>(shape->B) * shape->Hkv * (static_cast<size_t>(m) + 1) * shape->Ncap * sizeof(float);
}

extern "C" kv_status kv_build_wildcat_coreset(const kv_shape* shape, const void* K, float scale, int m, const float* u,
                                              int32_t* tok_idx, float* w, int32_t* n_sel, void* workspace,
                                              size_t ws_bytes, kv_stream_t stream) {
  auto bad = [](const char* msg) {
    kvs::set_last_error(msg);
    return KV_ERR_INVALID_ARG;
  };
  if (!shape) return bad("kv_build_wildcat_coreset: shape is NULL");
  if (shape->B < 0 || shape->Hkv < 1 || shape->Hq < shape->Hkv || shape->Ncap < 1)
    return bad("kv_build_wildcat_coreset: bad shape");
  if (shape->D != 64 && shape->D != 128) {
    kvs::set_last_error("kv_build_wildcat_coreset: head dim D must be 64 or 128");
    return KV_ERR_UNSUPPORTED;
  }
  if (shape->dtype != KV_BF16 && shape->dtype != KV_F32) return bad("kv_build_wildcat_coreset: unknown dtype");
  if (m < 1 || m > kvs::WC_MAX_M || m > shape->Ncap) return bad("kv_build_wildcat_coreset: m outside 1..min(4096, Ncap)");
  if (!std::isfinite(scale) || scale <= 0.f) return bad("kv_build_wildcat_coreset: scale must be finite and > 0");
  auto al = [](const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (shape->B > 0 && !al(shape->seq_lens, 4)) return bad("kv_build_wildcat_coreset: seq_lens NULL or misaligned");
  if (!al(K, 16)) return bad("kv_build_wildcat_coreset: K NULL or not 16-byte aligned");
  if (!al(u, 4) || !al(tok_idx, 4) || !al(w, 4)) return bad("kv_build_wildcat_coreset: u, tok_idx, w NULL or misaligned");
  if (n_sel && !al(n_sel, 4)) return bad("kv_build_wildcat_coreset: n_sel misaligned");
  if (!al(workspace, 16)) return bad("kv_build_wildcat_coreset: workspace NULL or not 16-byte aligned");
  if (ws_bytes < kv_wildcat_workspace_bytes(shape, m)) return bad("kv_build_wildcat_coreset: workspace too small");
  if (static_cast<long long>(shape->B) * shape->Hkv == 0) return KV_OK;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  cudaError_t e;
  if (shape->dtype == KV_BF16)
    e = shape->D == 64 ? kvs::wildcat_launch<__nv_bfloat16, 64>(shape, K, scale, m, u, tok_idx, w, n_sel, ws, st)
                       : kvs::wildcat_launch<__nv_bfloat16, 128>(shape, K, scale, m, u, tok_idx, w, n_sel, ws, st);
  else
    e = shape->D == 64 ? kvs::wildcat_launch<float, 64>(shape, K, scale, m, u, tok_idx, w, n_sel, ws, st)
                       : kvs::wildcat_launch<float, 128>(shape, K, scale, m, u, tok_idx, w, n_sel, ws, st);
  if (e != cudaSuccess) {
    kvs::set_last_error("kv_build_wildcat_coreset: launch failed");
    return KV_ERR_CUDA;
  }
  return KV_OK;
}
