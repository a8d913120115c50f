// Per-block covariance factors for second-order block scoring, built once after
// prefill.
//
// Source: "COBS: Cumulant Order Block Sparse Attention" -- truncating the cumulant
// expansion (8) at second order scores a block by sigma q.mean + (sigma^2 / 2)
// q^T Sigma_b q + ln n_b, and the covariance Sigma_b of the block's keys is kept as
// its top r eigendirections with the square root of each eigenvalue folded into
// the eigenvector (the low-rank spectral decomposition (13)). Sigma_b is the
// population covariance over the block's n_b keys (divided by n_b).
//
// One CTA per block. The nonzero spectrum of Sigma_b = X^T X / n (X: the n
// centred keys, n <= 64 rows of D) is that of the n x n Gram matrix
// G = X X^T / n: if G v = lambda v with |v| = 1, then xi = X^T v / sqrt(n) satisfies
// Sigma_b xi = lambda xi and |xi|^2 = lambda. G is formed in float64 from the keys
// and their float64 mean, and diagonalised by the cyclic Jacobi method with
// rotations applied in parallel: each round rotates n/2 disjoint index pairs (the
// round-robin "circle" schedule, so every pair meets once per sweep), all left
// rotations at once and then all right rotations at once, which is exactly the
// product of the round's rotations; sweeps stop when the off-diagonal mass is
// below 1e-24 of the diagonal's (or after 30 sweeps).
#pragma once

#include "common.cuh"

namespace kvs {

constexpr int COV_THREADS = 256;
constexpr int COV_MAX_ROWS = 64;  // largest block size the build supports
constexpr int COV_MAX_RANK = 8;

// Dynamic shared memory of one CTA: keys [L][D + 1] fp32 | mean [D] f64 |
// A [m][m + 1] f64 | V [m][m + 1] f64 | rotations [m/2] (c, s) f64 | pairs [m/2]
// int2 | scratch. The odd row strides keep column walks free of bank conflicts.
__host__ __device__ inline size_t cov_smem_bytes(int L, int D) {
  const int m = (L + 1) & ~1;
  return ((static_cast<size_t>(L) * (D + 1) * 4 + 15) & ~static_cast<size_t>(15)) + static_cast<size_t>(D) * 8 +
         2 * static_cast<size_t>(m) * (m + 1) * 8 + static_cast<size_t>(m / 2) * 16 + static_cast<size_t>(m / 2) * 8 +
         64 * 8;
}

template <typename T, int D>
__global__ void __launch_bounds__(COV_THREADS) cov_factors_kernel(const T* __restrict__ K,
                                                                  const int32_t* __restrict__ seq_lens,
                                                                  float* __restrict__ xi, int Hkv, int Ncap, int L,
                                                                  int NBcap, int r) {
  extern __shared__ __align__(16) unsigned char cov_smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int blk = static_cast<int>(blockIdx.x % static_cast<unsigned>(NBcap));
  const int bh = static_cast<int>(blockIdx.x / static_cast<unsigned>(NBcap));
  const int nseq = max(0, min(seq_lens[bh / Hkv], Ncap));
  const int start = blk * L;
  const int n = max(0, min(L, nseq - start));
  float* out = xi + (static_cast<size_t>(bh) * NBcap + blk) * static_cast<size_t>(r) * D;
  if (n <= 1) {  // no block, or one key: zero covariance
    for (int e = tid; e < r * D; e += COV_THREADS) out[e] = 0.f;
    return;
  }
  const int m = (n + 1) & ~1;  // even order for the round-robin schedule (a zero row pads odd n)
  const int mL = (L + 1) & ~1;
  const int ld = m + 1;        // row stride of A and V
  constexpr int KS = D + 1;    // row stride of the keys
  float* kx = reinterpret_cast<float*>(cov_smem);
  double* mean = reinterpret_cast<double*>(cov_smem + ((static_cast<size_t>(L) * KS * 4 + 15) & ~static_cast<size_t>(15)));
  double* A = mean + D;
  double* V = A + static_cast<size_t>(mL) * (mL + 1);
  double2* rot = reinterpret_cast<double2*>(V + static_cast<size_t>(mL) * (mL + 1));
  int2* pr = reinterpret_cast<int2*>(rot + mL / 2);
  double* red = reinterpret_cast<double*>(pr + mL / 2);
  int* sel = reinterpret_cast<int*>(red + 32);

  // keys (exact in fp32) and their mean (fp64)
  const T* src = K + (static_cast<size_t>(bh) * Ncap + start) * D;
  for (int e = tid; e < n * D; e += COV_THREADS) kx[(e / D) * KS + (e - (e / D) * D)] = load_as_float(src + e);
  __syncthreads();
  for (int d = tid; d < D; d += COV_THREADS) {
    double s = 0.0;
    for (int k = 0; k < n; ++k) s += static_cast<double>(kx[k * KS + d]);
    mean[d] = s / n;
  }
  __syncthreads();
  // Gram matrix of the centred keys, and V = I
  const double inv_n = 1.0 / n;
  for (int e = tid; e < m * m; e += COV_THREADS) {
    const int i = e / m, j = e - (e / m) * m;
    V[i * ld + j] = i == j ? 1.0 : 0.0;
    if (i > j) continue;
    double v = 0.0;
    if (j < n) {
      const float* ki = kx + i * KS;
      const float* kj = kx + j * KS;
      for (int d = 0; d < D; ++d) v = fma(static_cast<double>(ki[d]) - mean[d], static_cast<double>(kj[d]) - mean[d], v);
      v *= inv_n;
    }
    A[i * ld + j] = v;
    A[j * ld + i] = v;
  }
  __syncthreads();

  const int half = m / 2;
  for (int sweep = 0; sweep < 30; ++sweep) {
    for (int round = 0; round < m - 1; ++round) {
      if (tid < half) {
        // circle schedule: position 0 holds index 0, positions 1..m-1 rotate
        const int a = tid, b = m - 1 - tid;
        int p = a == 0 ? 0 : 1 + (a - 1 + round) % (m - 1);
        int q = 1 + (b - 1 + round) % (m - 1);
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        const double apq = A[p * ld + q], app = A[p * ld + p], aqq = A[q * ld + q];
        double c = 1.0, s = 0.0;
        if (fabs(apq) > 1e-300 && fabs(apq) > 1e-17 * sqrt(fabs(app * aqq))) {
          const double theta = (aqq - app) / (2.0 * apq);
          const double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          s = t * c;
        }
        pr[tid] = make_int2(p, q);
        rot[tid] = make_double2(c, s);
      }
      __syncthreads();
      // rows p, q of A <- J^T A (the pairs' rows are disjoint)
      for (int e = tid; e < half * m; e += COV_THREADS) {
        const int pi = e / m, k = e - (e / m) * m;
        const int2 pq = pr[pi];
        const double2 cs = rot[pi];
        const double apk = A[pq.x * ld + k], aqk = A[pq.y * ld + k];
        A[pq.x * ld + k] = cs.x * apk - cs.y * aqk;
        A[pq.y * ld + k] = cs.y * apk + cs.x * aqk;
      }
      __syncthreads();
      // columns p, q of A and V <- (.) J
      for (int e = tid; e < half * m; e += COV_THREADS) {
        const int pi = e / m, k = e - (e / m) * m;
        const int2 pq = pr[pi];
        const double2 cs = rot[pi];
        const double akp = A[k * ld + pq.x], akq = A[k * ld + pq.y];
        A[k * ld + pq.x] = cs.x * akp - cs.y * akq;
        A[k * ld + pq.y] = cs.y * akp + cs.x * akq;
        const double vkp = V[k * ld + pq.x], vkq = V[k * ld + pq.y];
        V[k * ld + pq.x] = cs.x * vkp - cs.y * vkq;
        V[k * ld + pq.y] = cs.y * vkp + cs.x * vkq;
      }
      __syncthreads();
    }
    // off-diagonal mass against the diagonal's
    double off = 0.0, dia = 0.0;
    for (int e = tid; e < m * m; e += COV_THREADS) {
      const int i = e / m, j = e - (e / m) * m;
      const double v = A[i * ld + j] * A[i * ld + j];
      if (i == j) dia += v;
      else off += v;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      off += __shfl_xor_sync(FULL_MASK, off, o);
      dia += __shfl_xor_sync(FULL_MASK, dia, o);
    }
    if (lane == 0) {
      red[warp] = off;
      red[16 + warp] = dia;
    }
    __syncthreads();
    double toff = 0.0, tdia = 0.0;
#pragma unroll
    for (int w = 0; w < COV_THREADS / 32; ++w) {
      toff += red[w];
      tdia += red[16 + w];
    }
    __syncthreads();  // red is reused by the next sweep
    if (toff <= 1e-24 * tdia) break;  // uniform
  }

  // the r largest eigenvalues (ties to the lower index)
  if (tid == 0) {
    unsigned long long taken[2] = {0ull, 0ull};
    for (int i = 0; i < r; ++i) {
      int best = -1;
      double bv = 0.0;
      for (int j = 0; j < m; ++j) {
        if ((taken[j >> 6] >> (j & 63)) & 1ull) continue;
        const double v = A[j * ld + j];
        if (best < 0 || v > bv) {
          best = j;
          bv = v;
        }
      }
      sel[i] = best;
      if (best >= 0) taken[best >> 6] |= 1ull << (best & 63);
    }
  }
  __syncthreads();
  // xi_i = X^T v_i / sqrt(n)
  const double rs = 1.0 / sqrt(static_cast<double>(n));
  for (int e = tid; e < r * D; e += COV_THREADS) {
    const int i = e / D, d = e - (e / D) * D;
    const int j = sel[i];
    double v = 0.0;
    if (j >= 0)
      for (int k = 0; k < n; ++k) v = fma(static_cast<double>(kx[k * KS + d]) - mean[d], V[k * ld + j], v);
    out[e] = static_cast<float>(v * rs);
  }
}

}  // namespace kvs
