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
__host__ __device__ inline size_t cov_smem_bytes(int L, int D, int s_dim = 0) {
  const int m = (L + 1) & ~1;
  return ((static_cast<size_t>(L) * (D + 1) * 4 + 15) & ~static_cast<size_t>(15)) + static_cast<size_t>(D) * 8 +
         2 * static_cast<size_t>(m) * (m + 1) * 8 + static_cast<size_t>(m / 2) * 16 + static_cast<size_t>(m / 2) * 8 +
         64 * 8 + (s_dim > 0 ? static_cast<size_t>(L) * (s_dim + 1) * 8 : 0);
}

// Cyclic Jacobi diagonalisation of the symmetric m x m matrix A (float64, row
// stride lda, m even) with the rotations accumulated into V (row stride ldv; V = I
// on entry; shared or global memory): each round rotates m/2 disjoint index pairs
// (the round-robin "circle" schedule, so every pair meets once per sweep), all
// left rotations at once and then all right rotations at once; sweeps stop when
// the off-diagonal mass is below 1e-24 of the diagonal's (or after 30 sweeps).
// On return A's diagonal holds the eigenvalues and V's column j the unit
// eigenvector of A[j][j]. Called by all COV_THREADS threads of the CTA.
__device__ inline void cov_jacobi(double* A, int lda, double* V, int ldv, int m, double2* rot, int2* pr,
                                  double* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
        const double apq = A[p * lda + q], app = A[p * lda + p], aqq = A[q * lda + q];
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
        const double apk = A[pq.x * lda + k], aqk = A[pq.y * lda + k];
        A[pq.x * lda + k] = cs.x * apk - cs.y * aqk;
        A[pq.y * lda + k] = cs.y * apk + cs.x * aqk;
      }
      __syncthreads();
      // columns p, q of A and V <- (.) J
      for (int e = tid; e < half * m; e += COV_THREADS) {
        const int pi = e / m, k = e - (e / m) * m;
        const int2 pq = pr[pi];
        const double2 cs = rot[pi];
        const double akp = A[k * lda + pq.x], akq = A[k * lda + pq.y];
        A[k * lda + pq.x] = cs.x * akp - cs.y * akq;
        A[k * lda + pq.y] = cs.y * akp + cs.x * akq;
        const double vkp = V[k * ldv + pq.x], vkq = V[k * ldv + pq.y];
        V[k * ldv + pq.x] = cs.x * vkp - cs.y * vkq;
        V[k * ldv + pq.y] = cs.y * vkp + cs.x * vkq;
      }
      __syncthreads();
    }
    // off-diagonal mass against the diagonal's
    double off = 0.0, dia = 0.0;
    for (int e = tid; e < m * m; e += COV_THREADS) {
      const int i = e / m, j = e - (e / m) * m;
      const double v = A[i * lda + j] * A[i * lda + j];
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
}

// PROJ: the covariance kept within a query subspace ("COBS", the subspace
// paragraph): with U ([s][D] per KV head, rows the basis) and Y = X U^T the
// centred keys' coordinates (n x s), B_b = U Sigma_b U^T = Y^T Y / n has the
// nonzero spectrum of the Gram matrix Y Y^T / n, and xi = Y^T v / sqrt(n) (s
// values, zero-padded to SP) by the same identity as in the full space.
template <typename T, int D, bool PROJ>
__global__ void __launch_bounds__(COV_THREADS) cov_factors_kernel(const T* __restrict__ K,
                                                                  const int32_t* __restrict__ seq_lens,
                                                                  float* __restrict__ xi, int Hkv, int Ncap, int L,
                                                                  int NBcap, int r, const float* __restrict__ U,
                                                                  int s_dim, int SP) {
  extern __shared__ __align__(16) unsigned char cov_smem[];
  const int tid = threadIdx.x;
  const int blk = static_cast<int>(blockIdx.x % static_cast<unsigned>(NBcap));
  const int bh = static_cast<int>(blockIdx.x / static_cast<unsigned>(NBcap));
  const int nseq = max(0, min(seq_lens[bh / Hkv], Ncap));
  const int start = blk * L;
  const int n = max(0, min(L, nseq - start));
  const int OUTW = PROJ ? SP : D;  // values per stored factor
  float* out = xi + (static_cast<size_t>(bh) * NBcap + blk) * static_cast<size_t>(r) * OUTW;
  if (n <= 1) {  // no block, or one key: zero covariance
    for (int e = tid; e < r * OUTW; e += COV_THREADS) out[e] = 0.f;
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
  double* Y = red + 64;  // PROJ: [L][s + 1] coordinates of the centred keys

  // keys (exact in fp32) and their mean (fp64)
  const T* src = K + (static_cast<size_t>(bh) * Ncap + start) * D;
  for (int e = tid; e < n * D; e += COV_THREADS) kx[(e / D) * KS + (e - (e / D) * D)] = load_as_float(src + e);
  __syncthreads();
  for (int d = tid; d < D; d += COV_THREADS) {
    double sum = 0.0;
    for (int k = 0; k < n; ++k) sum += static_cast<double>(kx[k * KS + d]);
    mean[d] = sum / n;
  }
  __syncthreads();
  const int ys = s_dim + 1;
  if constexpr (PROJ) {
    const float* Uh = U + static_cast<size_t>(bh % Hkv) * s_dim * D;
    for (int e = tid; e < n * s_dim; e += COV_THREADS) {
      const int k = e / s_dim, j = e - (e / s_dim) * s_dim;
      const float* kk = kx + k * KS;
      const float* uj = Uh + static_cast<size_t>(j) * D;
      double v = 0.0;
      for (int d = 0; d < D; ++d) v = fma(static_cast<double>(__ldg(uj + d)), static_cast<double>(kk[d]) - mean[d], v);
      Y[k * ys + j] = v;
    }
    __syncthreads();
  }
  // Gram matrix of the centred keys (or of their subspace coordinates), and V = I
  const double inv_n = 1.0 / n;
  for (int e = tid; e < m * m; e += COV_THREADS) {
    const int i = e / m, j = e - (e / m) * m;
    V[i * ld + j] = i == j ? 1.0 : 0.0;
    if (i > j) continue;
    double v = 0.0;
    if (j < n) {
      if constexpr (PROJ) {
        for (int c = 0; c < s_dim; ++c) v = fma(Y[i * ys + c], Y[j * ys + c], v);
      } else {
        const float* ki = kx + i * KS;
        const float* kj = kx + j * KS;
        for (int d = 0; d < D; ++d)
          v = fma(static_cast<double>(ki[d]) - mean[d], static_cast<double>(kj[d]) - mean[d], v);
      }
      v *= inv_n;
    }
    A[i * ld + j] = v;
    A[j * ld + i] = v;
  }
  __syncthreads();

  cov_jacobi(A, ld, V, ld, m, rot, pr, red);

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
  // xi_i = X^T v_i / sqrt(n)  (PROJ: Y^T v_i / sqrt(n), zero past s)
  const double rs = 1.0 / sqrt(static_cast<double>(n));
  for (int e = tid; e < r * OUTW; e += COV_THREADS) {
    const int i = e / OUTW, d = e - (e / OUTW) * OUTW;
    const int j = sel[i];
    double v = 0.0;
    if (j >= 0) {
      if constexpr (PROJ) {
        if (d < s_dim)
          for (int k = 0; k < n; ++k) v = fma(Y[k * ys + d], V[k * ld + j], v);
      } else {
        for (int k = 0; k < n; ++k) v = fma(static_cast<double>(kx[k * KS + d]) - mean[d], V[k * ld + j], v);
      }
    }
    out[e] = static_cast<float>(v * rs);
  }
}

// Query second-moment basis ("COBS", the subspace paragraph: the top eigenvectors
// of E[q q^T]). One CTA per KV head: C = mean over the calibration positions and
// the group's query heads of q q^T, accumulated in float64 in shared memory from
// chunks of QB_ROWS query rows, then diagonalised by cov_jacobi with V in global
// scratch (a 128 x 129 float64 V does not fit beside A). Outputs the eigenvalues
// in descending order (ties to the lower index) and the eigenvectors as rows.
constexpr int QB_ROWS = 32;
__host__ __device__ inline size_t qb_smem_bytes(int D) {
  return static_cast<size_t>(D) * (D + 1) * 8 + static_cast<size_t>(QB_ROWS) * D * 4 +
         static_cast<size_t>(D / 2) * 16 + static_cast<size_t>(D / 2) * 8 + 32 * 8 + static_cast<size_t>(D) * 4;
}

template <typename T, int D>
__global__ void __launch_bounds__(COV_THREADS) query_basis_kernel(const T* __restrict__ Qc, int Nc, int Hq, int Hkv,
                                                                  float* __restrict__ evecs, float* __restrict__ evals,
                                                                  double* __restrict__ vws) {
  extern __shared__ __align__(16) unsigned char qb_smem[];
  constexpr int ld = D + 1;
  const int h = blockIdx.x, tid = threadIdx.x;
  const int G = Hq / Hkv;
  double* A = reinterpret_cast<double*>(qb_smem);
  float* chunk = reinterpret_cast<float*>(A + static_cast<size_t>(D) * ld);
  double2* rot = reinterpret_cast<double2*>(chunk + QB_ROWS * D);
  int2* pr = reinterpret_cast<int2*>(rot + D / 2);
  double* red = reinterpret_cast<double*>(pr + D / 2);
  int* sel = reinterpret_cast<int*>(red + 32);
  double* V = vws + static_cast<size_t>(h) * D * ld;
  for (int e = tid; e < D * ld; e += COV_THREADS) A[e] = 0.0;
  // thread t owns row a = t * D / COV_THREADS .. of C in column range [c0, c0 + D * D / COV_THREADS)
  constexpr int PER = D * D / COV_THREADS;  // entries a thread accumulates (a run within one row)
  const int e0 = tid * PER, a = e0 / D, c0 = e0 - a * D;
  const int rows = Nc * G;
  for (int r0 = 0; r0 < rows; r0 += QB_ROWS) {
    __syncthreads();
    for (int e = tid; e < QB_ROWS * D; e += COV_THREADS) {
      const int rr = r0 + e / D, d = e - (e / D) * D;
      float v = 0.f;
      if (rr < rows) {
        const int pos = rr / G, g = rr - (rr / G) * G;
        v = load_as_float(Qc + (static_cast<size_t>(pos) * Hq + h * G + g) * D + d);
      }
      chunk[e] = v;
    }
    __syncthreads();
    for (int c = 0; c < PER; ++c) {
      double acc = A[a * ld + c0 + c];
      for (int k = 0; k < QB_ROWS; ++k)
        acc = fma(static_cast<double>(chunk[k * D + a]), static_cast<double>(chunk[k * D + c0 + c]), acc);
      A[a * ld + c0 + c] = acc;
    }
  }
  __syncthreads();
  const double inv_rows = rows > 0 ? 1.0 / rows : 0.0;
  for (int e = tid; e < D * D; e += COV_THREADS) {
    const int i = e / D, j = e - (e / D) * D;
    A[i * ld + j] *= inv_rows;
    V[i * ld + j] = i == j ? 1.0 : 0.0;
  }
  __syncthreads();
  cov_jacobi(A, ld, V, ld, D, rot, pr, red);
  if (tid == 0) {  // descending order, ties to the lower index
    unsigned long long taken[2] = {0ull, 0ull};
    for (int i = 0; i < D; ++i) {
      int best = -1;
      double bv = 0.0;
      for (int j = 0; j < D; ++j) {
        if ((taken[j >> 6] >> (j & 63)) & 1ull) continue;
        const double v = A[j * ld + j];
        if (best < 0 || v > bv) {
          best = j;
          bv = v;
        }
      }
      sel[i] = best;
      taken[best >> 6] |= 1ull << (best & 63);
    }
  }
  __syncthreads();
  for (int e = tid; e < D * D; e += COV_THREADS) {
    const int i = e / D, d = e - (e / D) * D;
    evecs[(static_cast<size_t>(h) * D + i) * D + d] = static_cast<float>(V[d * ld + sel[i]]);
  }
  for (int i = tid; i < D; i += COV_THREADS) evals[static_cast<size_t>(h) * D + i] = static_cast<float>(A[sel[i] * ld + sel[i]]);
}

}  // namespace kvs
