// Query-guided clustering with one proxy per cluster and an error-gated read
// budget. Source: "OpenAttention reads 1% of the KV cache", sections "Three helpers
// that make the proxy accurate" (QGC: keys projected onto the top eigenvectors of the
// queries, k-means in 16 dimensions once after prefill; ErrorGate: the exact-read
// budget split across clusters in proportion to the error each proxy would leave,
// estimated from cached mean and variance tokens; QGS: the top tokens inside each
// cluster from low-bit projections) and "Skipping reviews without losing the verdict"
// (the count-aware mean proxy; a proxy's weight error is its mass times the spread of
// the weights it hides).
//
// kv_build_qgc (once after prefill, one CTA per (sequence, KV head)):
//   z = P k for every token (float64 dot products, stored at fp32 in the scratch and
//   at bf16 for the per-query scan); Lloyd k-means on z in float64 (starts at the
//   tokens ((2c + 1) n) // (2C'), C' = min(C, n); distance summed over the 16
//   coordinates in order as separately rounded products and sums; ties to the lower
//   cluster; the labels of the last assignment are the clusters; centroid sums per
//   warp over contiguous token ranges, added in warp order); the members of every
//   cluster in ascending token order (a stable counting sort: ranks inside 32-token
//   chunks from match-any masks); per cluster the count, key sum, value sum and
//   per-channel key sum of squares, accumulated in float64 in member order.
// kv_select_qgc (per query, one CTA per pair):
//   per cluster mu_g = sigma q_g . mean, s2_g = sigma^2 sum_d q_gd^2 var_d, the error
//   E_c = sum_g n_c e^(mu - M_g) expm1(s2 / 2) / Zhat_g, Zhat_g = sum_c n_c e^(mu + s2/2 - M_g);
//   the read budget R = floor(budget n) - ceil(1.5 C_live) and r_c = min(n_c,
//   floor(R E_c / sum E)); token scores t_i = sum_g exp(sigma (P q_g) . z16_i - LSE_g)
//   in two passes; in every cluster the r_c tokens of largest (t, then lower index)
//   found by bisection on the 64-bit key (t's bits, inverted index); the read list
//   with weight 1 (padding weight 0) for kv_sparse_decode_attn's weighted mode; and
//   per cluster the proxy of its unread tokens (cluster sums minus the read rows,
//   over their count).
// kv_merge_qgc_proxies: folds the proxies (logit sigma q . mean + ln count) into the
//   weighted attention's out / lse by the exact log-sum-exp merge.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "kvsparse.h"

namespace kvs {
void set_last_error(const char* msg);

constexpr int QG_THREADS = 512;
constexpr int QG_NW = QG_THREADS / 32;
constexpr int QG_DIM = 16;     // projection dimension
constexpr int QG_MAX_C = 64;   // clusters per (sequence, KV head)
constexpr int QG_TCAP = 49152;  // token scores kept in shared memory (longer sequences use the scratch)

__host__ __device__ inline size_t qgc_build_smem_bytes(int D, int C) {
  return static_cast<size_t>(QG_DIM) * D * 4 +                 // P rows
         static_cast<size_t>(C) * QG_DIM * 8 +                 // centroids
         static_cast<size_t>(QG_NW) * C * QG_DIM * 8 +         // per-warp centroid sums
         static_cast<size_t>(QG_NW) * C * 4 +                  // per-warp counts / scatter bases
         static_cast<size_t>(C + 1) * 4 + 16;                  // cluster starts
}

template <typename T, int D>
__global__ void __launch_bounds__(QG_THREADS) qgc_build_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                               const int32_t* __restrict__ seq_lens, int Hkv,
                                                               int Ncap, const float* __restrict__ P, int C,
                                                               int iters, __nv_bfloat16* __restrict__ z16,
                                                               int32_t* __restrict__ labels,
                                                               int32_t* __restrict__ perm, int32_t* __restrict__ offs,
                                                               int32_t* __restrict__ counts, float* __restrict__ k_sum,
                                                               float* __restrict__ v_sum, float* __restrict__ k_sq,
                                                               float* __restrict__ zws) {
  extern __shared__ __align__(16) unsigned char qg_smem[];
  float* Ps = reinterpret_cast<float*>(qg_smem);
  double* cent = reinterpret_cast<double*>(Ps + QG_DIM * D);
  double* acc = cent + static_cast<size_t>(C) * QG_DIM;
  int* wcnt = reinterpret_cast<int*>(acc + static_cast<size_t>(QG_NW) * C * QG_DIM);
  int* cstart = wcnt + QG_NW * C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, b = bh / Hkv, h = bh - (bh / Hkv) * Hkv;
  const int n = max(0, min(seq_lens[b], Ncap));
  const int Ce = min(C, n);
  const size_t tok0 = static_cast<size_t>(bh) * Ncap;
  const T* Kb = K + tok0 * D;
  const T* Vb = V + tok0 * D;
  float* Z = zws + tok0 * QG_DIM;
  int32_t* lab = labels + tok0;
  int32_t* pm = perm + tok0;

  for (int e = tid; e < QG_DIM * D; e += QG_THREADS) Ps[e] = P[static_cast<size_t>(h) * QG_DIM * D + e];
  __syncthreads();

  // ---- 1. projection z = P k (float64), stored at fp32 (scratch) and bf16 (output)
  constexpr int CH = 16 / sizeof(T);
  for (int i = tid; i < Ncap; i += QG_THREADS) {
    __nv_bfloat16* zo = z16 + (tok0 + i) * QG_DIM;
    if (i < n) {
      double a[QG_DIM];
#pragma unroll
      for (int j = 0; j < QG_DIM; ++j) a[j] = 0.0;
      const T* row = Kb + static_cast<size_t>(i) * D;
      for (int c = 0; c < D / CH; ++c) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(row) + c);
        float2 f[CH / 2];
        Chunk<T>::unpack(raw, f);
#pragma unroll
        for (int e = 0; e < CH / 2; ++e) {
          const int d0 = c * CH + 2 * e;
#pragma unroll
          for (int j = 0; j < QG_DIM; ++j) {
            a[j] = fma(static_cast<double>(f[e].x), static_cast<double>(Ps[j * D + d0]), a[j]);
            a[j] = fma(static_cast<double>(f[e].y), static_cast<double>(Ps[j * D + d0 + 1]), a[j]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < QG_DIM; ++j) {
        const float zf = static_cast<float>(a[j]);
        Z[static_cast<size_t>(i) * QG_DIM + j] = zf;
        zo[j] = __float2bfloat16_rn(zf);
      }
    } else {
#pragma unroll
      for (int j = 0; j < QG_DIM; ++j) zo[j] = __float2bfloat16_rn(0.f);
      lab[i] = -1;
      pm[i] = -1;
    }
  }
  __syncthreads();

  // ---- 2. k-means
  for (int e = tid; e < Ce * QG_DIM; e += QG_THREADS) {
    const int c = e / QG_DIM, j = e - (e / QG_DIM) * QG_DIM;
    const long long s = ((2LL * c + 1) * n) / (2LL * Ce);
    cent[e] = static_cast<double>(Z[s * QG_DIM + j]);
  }
  const int lo = static_cast<int>(static_cast<long long>(n) * warp / QG_NW);
  const int hi = static_cast<int>(static_cast<long long>(n) * (warp + 1) / QG_NW);
  for (int it = 0; it < iters; ++it) {
    __syncthreads();
    for (int i = tid; i < n; i += QG_THREADS) {
      double zd[QG_DIM];
#pragma unroll
      for (int j = 0; j < QG_DIM; ++j) zd[j] = static_cast<double>(Z[static_cast<size_t>(i) * QG_DIM + j]);
      int best = 0;
      double bd = INFINITY;
      for (int c = 0; c < Ce; ++c) {
        double a = 0.0;
#pragma unroll
        for (int j = 0; j < QG_DIM; ++j) {
          const double df = __dsub_rn(zd[j], cent[c * QG_DIM + j]);
          a = __dadd_rn(a, __dmul_rn(df, df));
        }
        if (a < bd) {
          bd = a;
          best = c;
        }
      }
      lab[i] = best;
    }
    if (it == iters - 1) break;  // the last assignment's labels are the clusters
    __syncthreads();
    // per-warp centroid sums over the warp's contiguous token range, in token order
    double* aw = acc + static_cast<size_t>(warp) * C * QG_DIM;
    for (int e = lane; e < Ce * QG_DIM; e += 32) aw[e] = 0.0;
    for (int e = lane; e < Ce; e += 32) wcnt[warp * C + e] = 0;
    __syncwarp();
    for (int i = lo; i < hi; ++i) {
      const int c = lab[i];
      if (lane < QG_DIM) aw[c * QG_DIM + lane] += static_cast<double>(Z[static_cast<size_t>(i) * QG_DIM + lane]);
      if (lane == QG_DIM) wcnt[warp * C + c] += 1;
    }
    __syncthreads();
    for (int e = tid; e < Ce * QG_DIM; e += QG_THREADS) {
      const int c = e / QG_DIM;
      double sum = 0.0;
      int cnt = 0;
      for (int w = 0; w < QG_NW; ++w) {
        sum += acc[(static_cast<size_t>(w) * C + c) * QG_DIM + (e - c * QG_DIM)];
        cnt += wcnt[w * C + c];
      }
      if (cnt > 0) cent[e] = sum / cnt;
    }
  }
  __syncthreads();

  // ---- 3. members in ascending token order (stable counting sort by label)
  for (int e = lane; e < C; e += 32) wcnt[warp * C + e] = 0;
  __syncwarp();
  for (int i0 = lo; i0 < hi; i0 += 32) {
    const int i = i0 + lane;
    const bool in = i < hi;
    const unsigned act = __ballot_sync(FULL_MASK, in);
    const int c = in ? lab[i] : -1;
    const unsigned same = __match_any_sync(FULL_MASK, c);
    if (in && (__ffs(same & act) - 1) == lane) wcnt[warp * C + c] += __popc(same & act);
    __syncwarp();
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int c = 0; c < C; ++c) {
      cstart[c] = run;
      for (int w = 0; w < QG_NW; ++w) {
        const int k = wcnt[w * C + c];
        wcnt[w * C + c] = run;  // the warp's first position in cluster c
        run += k;
      }
    }
    cstart[C] = run;
  }
  __syncthreads();
  for (int i0 = lo; i0 < hi; i0 += 32) {
    const int i = i0 + lane;
    const bool in = i < hi;
    const unsigned act = __ballot_sync(FULL_MASK, in);
    const int c = in ? lab[i] : -1;
    const unsigned same = __match_any_sync(FULL_MASK, c) & act;
    if (in) {
      const int rank = __popc(same & ((1u << lane) - 1u));
      pm[wcnt[warp * C + c] + rank] = i;
    }
    __syncwarp();
    if (in && (__ffs(same) - 1) == lane) wcnt[warp * C + c] += __popc(same);
    __syncwarp();
  }
  __syncthreads();
  for (int c = tid; c <= C; c += QG_THREADS) offs[static_cast<size_t>(bh) * (C + 1) + c] = cstart[c];
  for (int c = tid; c < C; c += QG_THREADS) counts[static_cast<size_t>(bh) * C + c] = cstart[c + 1] - cstart[c];

  // ---- 4. cluster statistics, a warp per cluster, lanes over the channels
  constexpr int CPL = D / 32;
  for (int c = warp; c < C; c += QG_NW) {
    double ks[CPL], vs[CPL], kq[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) ks[k] = vs[k] = kq[k] = 0.0;
    for (int m = cstart[c]; m < cstart[c + 1]; ++m) {
      const int i = pm[m];
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const double kx = static_cast<double>(load_as_float(Kb + static_cast<size_t>(i) * D + lane * CPL + k));
        const double vx = static_cast<double>(load_as_float(Vb + static_cast<size_t>(i) * D + lane * CPL + k));
        ks[k] += kx;
        vs[k] += vx;
        kq[k] += kx * kx;
      }
    }
    const size_t o = (static_cast<size_t>(bh) * C + c) * D + lane * CPL;
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      k_sum[o + k] = static_cast<float>(ks[k]);
      v_sum[o + k] = static_cast<float>(vs[k]);
      k_sq[o + k] = static_cast<float>(kq[k]);
    }
  }
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(FULL_MASK, x, o);
    x = y > x ? y : x;
  }
  return x;
}

// A lane's CPL consecutive channels of a row, as fp32 (one vector load).
template <typename T, int CPL>
__device__ __forceinline__ void qg_slice(const T* row, int lane, float (&x)[CPL]) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (CPL == 4) {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(row) + lane);
      x[0] = __uint_as_float(r.x << 16);
      x[1] = __uint_as_float(r.x & 0xffff0000u);
      x[2] = __uint_as_float(r.y << 16);
      x[3] = __uint_as_float(r.y & 0xffff0000u);
    } else {
      const uint32_t r = __ldg(reinterpret_cast<const uint32_t*>(row) + lane);
      x[0] = __uint_as_float(r << 16);
      x[1] = __uint_as_float(r & 0xffff0000u);
    }
  } else {
    if constexpr (CPL == 4) {
      const float4 r = __ldg(reinterpret_cast<const float4*>(row) + lane);
      x[0] = r.x;
      x[1] = r.y;
      x[2] = r.z;
      x[3] = r.w;
    } else {
      const float2 r = __ldg(reinterpret_cast<const float2*>(row) + lane);
      x[0] = r.x;
      x[1] = r.y;
    }
  }
}

struct QgcSel {
  const void* q;
  const void* K;
  const void* V;
  const int32_t* seq_lens;
  const float* P;  // [Hkv][16][D]
  const __nv_bfloat16* z16;
  const int32_t* perm;
  const int32_t* offs;
  const int32_t* counts;
  const float* k_sum;
  const float* v_sum;
  const float* k_sq;
  int32_t* tok_idx;  // [B][Hkv][max_read]
  float* w;          // [B][Hkv][max_read]
  int32_t* n_read;   // [B][Hkv]
  float* pk;         // [B][Hkv][C][D]
  float* pv;
  int32_t* pn;       // [B][Hkv][C]
  float* tws;        // [B][Hkv][Ncap] token scores (scratch)
  int Hq, Hkv, Ncap, C, max_read;
  float sigma, budget;
};

struct QgcSelShared {
  float mu[8][QG_MAX_C], s2[8][QG_MAX_C];
  float E[QG_MAX_C];
  int r[QG_MAX_C], roff[QG_MAX_C + 1];
  float qt[8][QG_DIM];
  float lse[8];
  float pmx[QG_NW][8], psm[QG_NW][8];
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(QG_THREADS) qgc_select_kernel(const QgcSel p) {
  __shared__ QgcSelShared sh;
  extern __shared__ __align__(16) float qg_ts[];  // token scores, when n <= QG_TCAP
  constexpr int CPL = D / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, b = bh / p.Hkv, h = bh - (bh / p.Hkv) * p.Hkv;
  const int n = max(0, min(p.seq_lens[b], p.Ncap));
  const int C = p.C;
  const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(h) * G) * D;
  const int32_t* cnt = p.counts + static_cast<size_t>(bh) * C;
  const int32_t* off = p.offs + static_cast<size_t>(bh) * (C + 1);
  const int32_t* pm = p.perm + static_cast<size_t>(bh) * p.Ncap;
  const T* Kb = static_cast<const T*>(p.K) + static_cast<size_t>(bh) * p.Ncap * D;
  const T* Vb = static_cast<const T*>(p.V) + static_cast<size_t>(bh) * p.Ncap * D;
  float* t = p.Ncap <= QG_TCAP ? qg_ts : p.tws + static_cast<size_t>(bh) * p.Ncap;

  // the group's queries, a lane CPL channels of each
  float qf[G][CPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int k = 0; k < CPL; ++k) qf[g][k] = load_as_float(qrow + g * D + lane * CPL + k);

  // ---- projected queries q~_g = P q_g (warp j: row j of P)
  for (int j = warp; j < QG_DIM; j += QG_NW) {
    float u[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) u[k] = __ldg(p.P + (static_cast<size_t>(h) * QG_DIM + j) * D + lane * CPL + k);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float v = 0.f;
#pragma unroll
      for (int k = 0; k < CPL; ++k) v = fmaf(u[k], qf[g][k], v);
      v = warp_sum(v);
      if (lane == 0) sh.qt[g][j] = v;
    }
  }

  // ---- per cluster mean logit and logit variance (a warp per cluster)
  for (int c = warp; c < C; c += QG_NW) {
    const int nc = cnt[c];
    const size_t o = (static_cast<size_t>(bh) * C + c) * D + lane * CPL;
    float mean[CPL], var[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const float m = nc > 0 ? __fdiv_rn(p.k_sum[o + k], static_cast<float>(nc)) : 0.f;
      const float sq = nc > 0 ? __fdiv_rn(p.k_sq[o + k], static_cast<float>(nc)) : 0.f;
      mean[k] = m;
      var[k] = fmaxf(sq - m * m, 0.f);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float a = 0.f, v = 0.f;
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        a = fmaf(qf[g][k], mean[k], a);
        v = fmaf(qf[g][k] * qf[g][k], var[k], v);
      }
      a = warp_sum(a);
      v = warp_sum(v);
      if (lane == 0) {
        sh.mu[g][c] = nc > 0 ? p.sigma * a : -INFINITY;
        sh.s2[g][c] = nc > 0 ? p.sigma * p.sigma * v : 0.f;
      }
    }
  }
  __syncthreads();

  // ---- errors, the read budget and its split (warp 0, lanes over clusters)
  if (warp == 0) {
    float e0 = 0.f, e1 = 0.f;  // clusters lane and lane + 32
    int live = 0;
    for (int c = lane; c < C; c += 32) live += cnt[c] > 0;
    live = __reduce_add_sync(FULL_MASK, live);
    for (int g = 0; g < G; ++g) {
      float M = -INFINITY;
      for (int c = lane; c < C; c += 32)
        if (cnt[c] > 0) M = fmaxf(M, sh.mu[g][c] + 0.5f * sh.s2[g][c]);
      M = warp_max(M);
      if (M == -INFINITY) continue;
      float z = 0.f;
      for (int c = lane; c < C; c += 32)
        if (cnt[c] > 0) z += static_cast<float>(cnt[c]) * __expf(sh.mu[g][c] + 0.5f * sh.s2[g][c] - M);
      z = warp_sum(z);
      for (int c = lane, k = 0; c < C; c += 32, ++k) {
        if (cnt[c] <= 0) continue;
        const float e = static_cast<float>(cnt[c]) * __expf(sh.mu[g][c] - M) * expm1f(0.5f * sh.s2[g][c]) / z;
        if (k == 0) e0 += e; else e1 += e;
      }
    }
    const float tot = warp_sum(e0 + e1);
    const long long Rb = static_cast<long long>(floor(static_cast<double>(p.budget) * n));
    const int R = static_cast<int>(max(0LL, Rb - static_cast<long long>(ceil(1.5 * live))));
    int rsum = 0;
    for (int c = lane, k = 0; c < C; c += 32, ++k) {
      const float e = k == 0 ? e0 : e1;
      sh.E[c] = e;
      int rc = 0;
      if (tot > 0.f && R > 0 && cnt[c] > 0)
        rc = static_cast<int>(min(static_cast<double>(cnt[c]), floor(static_cast<double>(R) * e / tot)));
      sh.r[c] = rc;
    }
    __syncwarp();
    if (lane == 0) {
      for (int c = 0; c < C; ++c) {
        sh.roff[c] = rsum;
        rsum += sh.r[c];
      }
      sh.roff[C] = rsum;
      p.n_read[bh] = rsum;
    }
  }
  __syncthreads();

  // ---- token scores: LSE per head over the tokens, then t_i (two passes; the next
  // token's coordinates are loaded before the current one's arithmetic)
  {
    const uint4* zbase = reinterpret_cast<const uint4*>(p.z16 + static_cast<size_t>(bh) * p.Ncap * QG_DIM);
    auto logits = [&](uint4 a, uint4 bq, float (&sg)[G]) {
      float z[QG_DIM];
      float2 f[4];
      Chunk<__nv_bfloat16>::unpack(a, f);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        z[2 * e] = f[e].x;
        z[2 * e + 1] = f[e].y;
      }
      Chunk<__nv_bfloat16>::unpack(bq, f);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        z[8 + 2 * e] = f[e].x;
        z[8 + 2 * e + 1] = f[e].y;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a2 = 0.f;
#pragma unroll
        for (int j = 0; j < QG_DIM; ++j) a2 = fmaf(sh.qt[g][j], z[j], a2);
        sg[g] = a2 * p.sigma;
      }
    };
    float m[G], l[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
    }
    uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0;
    if (tid < n) {
      c0 = __ldg(zbase + 2 * tid);
      c1 = __ldg(zbase + 2 * tid + 1);
    }
    for (int i = tid; i < n; i += QG_THREADS) {
      const int inx = i + QG_THREADS;
      uint4 n0 = c0, n1 = c1;
      if (inx < n) {
        n0 = __ldg(zbase + 2 * inx);
        n1 = __ldg(zbase + 2 * inx + 1);
      }
      float sg[G];
      logits(c0, c1, sg);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (sg[g] > m[g]) {
          l[g] = l[g] * __expf(m[g] - sg[g]) + 1.f;
          m[g] = sg[g];
        } else {
          l[g] += __expf(sg[g] - m[g]);
        }
      }
      c0 = n0;
      c1 = n1;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float M = warp_max(m[g]);
      float L = (m[g] == -INFINITY) ? 0.f : l[g] * __expf(m[g] - M);
      L = warp_sum(L);
      if (lane == 0) {
        sh.pmx[warp][g] = M;
        sh.psm[warp][g] = L;
      }
    }
    __syncthreads();
    if (tid < G) {
      float M = -INFINITY;
      for (int w = 0; w < QG_NW; ++w) M = fmaxf(M, sh.pmx[w][tid]);
      float L = 0.f;
      if (M != -INFINITY)
        for (int w = 0; w < QG_NW; ++w)
          if (sh.pmx[w][tid] != -INFINITY) L += sh.psm[w][tid] * __expf(sh.pmx[w][tid] - M);
      sh.lse[tid] = M == -INFINITY ? -INFINITY : M + __logf(L);
    }
    __syncthreads();
    if (tid < n) {
      c0 = __ldg(zbase + 2 * tid);
      c1 = __ldg(zbase + 2 * tid + 1);
    }
    for (int i = tid; i < n; i += QG_THREADS) {
      const int inx = i + QG_THREADS;
      uint4 n0 = c0, n1 = c1;
      if (inx < n) {
        n0 = __ldg(zbase + 2 * inx);
        n1 = __ldg(zbase + 2 * inx + 1);
      }
      float sg[G];
      logits(c0, c1, sg);
      float tv = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) tv += __expf(sg[g] - sh.lse[g]);
      t[i] = tv;
      c0 = n0;
      c1 = n1;
    }
  }
  __syncthreads();

  // ---- per cluster: the r_c largest keys (t's bits, inverted index), the read list,
  // the read rows' sums and the proxy of the unread tokens (a warp per cluster); the
  // scores are read through the member list (shared memory for sequences up to
  // QG_TCAP tokens)
  auto key_of = [&](int i) {
    return (static_cast<unsigned long long>(__float_as_uint(t[i])) << 32) |
           static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(i));
  };
  for (int c = warp; c < C; c += QG_NW) {
    const int nc = cnt[c], rc = sh.r[c];
    const int m0 = off[c], m1 = off[c + 1];
    unsigned long long thr = 0ull;  // keys >= thr are read
    if (rc > 0 && rc < nc) {
      if (rc <= 32) {
        // rc rounds of "largest key below the previous one" (keys are distinct)
        unsigned long long prev = ~0ull;
        for (int k = 0; k < rc; ++k) {
          unsigned long long best = 0ull;
          for (int m = m0 + lane; m < m1; m += 32) {
            const unsigned long long x = key_of(pm[m]);
            if (x < prev && x > best) best = x;
          }
          prev = warp_max_u64(best);
        }
        thr = prev;
      } else {
        unsigned long long prefix = 0ull;
        for (int bit = 63; bit >= 0; --bit) {
          const unsigned long long cand = prefix | (1ull << bit);
          int k = 0;
          for (int m = m0 + lane; m < m1; m += 32) k += key_of(pm[m]) >= cand;
          k = __reduce_add_sync(FULL_MASK, k);
          if (k >= rc) prefix = cand;
        }
        thr = prefix;
      }
    }
    float rk[CPL], rv[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) rk[k] = rv[k] = 0.f;
    int pos = sh.roff[c];
    if (rc > 0) {
      for (int m = m0; m < m1; m += 32) {
        const int mi = m + lane;
        int i = -1;
        bool take = false;
        if (mi < m1) {
          i = pm[mi];
          take = rc >= nc || key_of(i) >= thr;
        }
        const unsigned bal = __ballot_sync(FULL_MASK, take);
        if (take) {
          const int q = pos + __popc(bal & ((1u << lane) - 1u));
          if (q < p.max_read) {
            p.tok_idx[static_cast<size_t>(bh) * p.max_read + q] = i;
            p.w[static_cast<size_t>(bh) * p.max_read + q] = 1.f;
          }
        }
        pos += __popc(bal);
      }
      // the read rows' key and value sums, eight rows' loads in flight
      __syncwarp();  // the list entries written above are visible to every lane
      const int32_t* lst = p.tok_idx + static_cast<size_t>(bh) * p.max_read + sh.roff[c];
      const int nl = min(rc, p.max_read - sh.roff[c]);
      for (int j0 = 0; j0 < nl; j0 += 8) {
        float kx[8][CPL], vx[8][CPL];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (j0 + u < nl) {
            const int ti = lst[j0 + u];
            qg_slice<T, CPL>(Kb + static_cast<size_t>(ti) * D, lane, kx[u]);
            qg_slice<T, CPL>(Vb + static_cast<size_t>(ti) * D, lane, vx[u]);
          } else {
#pragma unroll
            for (int k = 0; k < CPL; ++k) kx[u][k] = vx[u][k] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            rk[k] += kx[u][k];
            rv[k] += vx[u][k];
          }
      }
    }
    const int un = nc - rc;  // unread tokens of the cluster
    const size_t o = (static_cast<size_t>(bh) * C + c) * D + lane * CPL;
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      p.pk[o + k] = un > 0 ? __fdiv_rn(p.k_sum[o + k] - rk[k], static_cast<float>(un)) : 0.f;
      p.pv[o + k] = un > 0 ? __fdiv_rn(p.v_sum[o + k] - rv[k], static_cast<float>(un)) : 0.f;
    }
    if (lane == 0) p.pn[static_cast<size_t>(bh) * C + c] = max(un, 0);
  }
  // padding of the read list
  for (int q = sh.roff[C] + tid; q < p.max_read; q += QG_THREADS) {
    p.tok_idx[static_cast<size_t>(bh) * p.max_read + q] = 0;
    p.w[static_cast<size_t>(bh) * p.max_read + q] = 0.f;
  }
}

// Folds the proxies into the attention over the read tokens: a warp per query head,
// lanes over the channels. With the read tokens' (out, lse) and proxy logits
// l_c = sigma q . pk_c + ln pn_c (pn_c > 0): M = max(lse, l_c),
// out = (e^(lse - M) out + sum_c e^(l_c - M) pv_c) / (e^(lse - M) + sum_c e^(l_c - M)).
template <typename T, int D>
__global__ void __launch_bounds__(256) qgc_merge_kernel(const T* __restrict__ q, int B, int Hq, int Hkv, int C,
                                                        float sigma, const float* __restrict__ pk,
                                                        const float* __restrict__ pv, const int32_t* __restrict__ pn,
                                                        float* __restrict__ out, float* __restrict__ lse) {
  __shared__ float lgs[8][QG_MAX_C];
  constexpr int CPL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (row >= static_cast<long long>(B) * Hq) return;  // warp-uniform; no block-wide barrier below
  const int b = static_cast<int>(row / Hq), g = static_cast<int>(row - static_cast<long long>(b) * Hq);
  const int G = Hq / Hkv, h = g / G;
  const size_t bh = static_cast<size_t>(b) * Hkv + h;
  float qf[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) qf[k] = load_as_float(q + static_cast<size_t>(row) * D + lane * CPL + k);
  float M = lse[row];
  for (int c = 0; c < C; ++c) {
    const int nc = pn[bh * C + c];
    float a = 0.f;
    if (nc > 0) {
#pragma unroll
      for (int k = 0; k < CPL; ++k) a = fmaf(qf[k], pk[(bh * C + c) * D + lane * CPL + k], a);
    }
    a = warp_sum(a);
    const float lc = nc > 0 ? sigma * a + __logf(static_cast<float>(nc)) : -INFINITY;
    if (lane == 0) lgs[warp][c] = lc;
    M = fmaxf(M, lc);
  }
  __syncwarp();
  if (M == -INFINITY) return;  // nothing read and no proxy (an empty sequence)
  const float l0 = lse[row];
  const float a0 = l0 == -INFINITY ? 0.f : __expf(l0 - M);
  float den = a0;
  float o[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) o[k] = a0 * out[static_cast<size_t>(row) * D + lane * CPL + k];
  for (int c = 0; c < C; ++c) {
    const float lc = lgs[warp][c];
    if (lc == -INFINITY) continue;
    const float e = __expf(lc - M);
    den += e;
#pragma unroll
    for (int k = 0; k < CPL; ++k) o[k] = fmaf(e, pv[(bh * C + c) * D + lane * CPL + k], o[k]);
  }
#pragma unroll
  for (int k = 0; k < CPL; ++k) out[static_cast<size_t>(row) * D + lane * CPL + k] = o[k] / den;
  __syncwarp();
  if (lane == 0) lse[row] = M + __logf(den);
}
}  // namespace kvs

namespace {
kv_status qbad(kv_status s, const char* msg) {
  kvs::set_last_error(msg);
  return s;
}
bool qal(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

kv_status qgc_check_shape(const kv_shape* s, const char* who) {
  (void)who;
  if (!s) return qbad(KV_ERR_INVALID_ARG, "qgc: shape is NULL");
  if (s->B < 0 || s->Hkv < 1 || s->Hq < s->Hkv || s->Hq % s->Hkv != 0 || s->Ncap < 1)
    return qbad(KV_ERR_INVALID_ARG, "qgc: bad shape");
  if (s->D != 64 && s->D != 128) return qbad(KV_ERR_UNSUPPORTED, "qgc: head dim D must be 64 or 128");
  if (s->Hq / s->Hkv > 8) return qbad(KV_ERR_UNSUPPORTED, "qgc: group size above 8");
  if (s->dtype != KV_BF16 && s->dtype != KV_F32) return qbad(KV_ERR_INVALID_ARG, "qgc: unknown dtype");
  if (s->B > 0 && !qal(s->seq_lens, 4)) return qbad(KV_ERR_INVALID_ARG, "qgc: seq_lens NULL or misaligned");
  return KV_OK;
}

template <typename T, int D>
cudaError_t qgc_build_td(const kv_shape* s, const void* K, const void* V, const float* P, int C, int iters,
                         __nv_bfloat16* z16, int32_t* labels, int32_t* perm, int32_t* offs, int32_t* counts,
                         float* k_sum, float* v_sum, float* k_sq, float* zws, cudaStream_t st) {
  static std::atomic<int> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured.load() & (1 << (dev & 31)))) {
    const cudaError_t e = cudaFuncSetAttribute(kvs::qgc_build_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(kvs::qgc_build_smem_bytes(D, kvs::QG_MAX_C)));
    if (e != cudaSuccess) return e;
    configured.fetch_or(1 << (dev & 31));
  }
  kvs::qgc_build_kernel<T, D><<<s->B * s->Hkv, kvs::QG_THREADS, kvs::qgc_build_smem_bytes(D, C), st>>>(
      static_cast<const T*>(K), static_cast<const T*>(V), s->seq_lens, s->Hkv, s->Ncap, P, C, iters, z16, labels,
      perm, offs, counts, k_sum, v_sum, k_sq, zws);
  return cudaGetLastError();
}

constexpr int QG_KEY_SMEM = kvs::QG_TCAP * 4;

template <typename T, int D>
cudaError_t qgc_select_td(int G, const kvs::QgcSel& p, int grid, cudaStream_t st) {
  switch (G) {
#define QG_CASE(GG)                                                                                     \
  case GG: {                                                                                             \
    static std::atomic<int> cfg_##GG{0};                                                                 \
    int dev = 0;                                                                                         \
    cudaGetDevice(&dev);                                                                                 \
    if (!(cfg_##GG.load() & (1 << (dev & 31)))) {                                                        \
      const cudaError_t e = cudaFuncSetAttribute(kvs::qgc_select_kernel<T, D, GG>,                       \
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, QG_KEY_SMEM); \
      if (e != cudaSuccess) return e;                                                                    \
      cfg_##GG.fetch_or(1 << (dev & 31));                                                                \
    }                                                                                                    \
    kvs::qgc_select_kernel<T, D, GG><<<grid, kvs::QG_THREADS,                                           \
                                       p.Ncap <= kvs::QG_TCAP ? p.Ncap * 4 : 0, st>>>(p);                \
    break;                                                                                               \
  }
    QG_CASE(1) QG_CASE(2) QG_CASE(3) QG_CASE(4) QG_CASE(5) QG_CASE(6) QG_CASE(7) QG_CASE(8)
#undef QG_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}
}  // namespace

extern "C" {

size_t kv_qgc_workspace_bytes(const kv_shape* shape) {
  if (!shape || shape->B < 0 || shape->Hkv < 1 || shape->Ncap < 1) return 0;
  return static_cast<size_t>(shape->B) * shape->Hkv * shape->Ncap * kvs::QG_DIM * sizeof(float);
}

kv_status kv_build_qgc(const kv_shape* shape, const void* K, const void* V, const float* P, int C, int iters,
                       void* z16, int32_t* labels, int32_t* perm, int32_t* offs, int32_t* counts, float* k_sum,
                       float* v_sum, float* k_sq, void* workspace, size_t ws_bytes, kv_stream_t stream) {
  kv_status st0 = qgc_check_shape(shape, "kv_build_qgc");
  if (st0 != KV_OK) return st0;
  if (C < 1 || C > kvs::QG_MAX_C) return qbad(KV_ERR_INVALID_ARG, "kv_build_qgc: clusters outside 1..64");
  if (iters < 1 || iters > 100) return qbad(KV_ERR_INVALID_ARG, "kv_build_qgc: iterations outside 1..100");
  if (!qal(K, 16) || !qal(V, 16) || !qal(P, 4)) return qbad(KV_ERR_INVALID_ARG, "kv_build_qgc: K, V or P NULL or misaligned");
  if (!qal(z16, 16) || !qal(labels, 4) || !qal(perm, 4) || !qal(offs, 4) || !qal(counts, 4) || !qal(k_sum, 4) ||
      !qal(v_sum, 4) || !qal(k_sq, 4))
    return qbad(KV_ERR_INVALID_ARG, "kv_build_qgc: an output is NULL or misaligned");
  if (!qal(workspace, 16) || ws_bytes < kv_qgc_workspace_bytes(shape))
    return qbad(KV_ERR_INVALID_ARG, "kv_build_qgc: workspace NULL, misaligned or too small");
  if (shape->B * shape->Hkv == 0) return KV_OK;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* z = static_cast<__nv_bfloat16*>(z16);
  auto* zws = static_cast<float*>(workspace);
  cudaError_t e;
  if (shape->dtype == KV_BF16)
    e = shape->D == 64 ? qgc_build_td<__nv_bfloat16, 64>(shape, K, V, P, C, iters, z, labels, perm, offs, counts,
                                                        k_sum, v_sum, k_sq, zws, st)
                       : qgc_build_td<__nv_bfloat16, 128>(shape, K, V, P, C, iters, z, labels, perm, offs, counts,
                                                         k_sum, v_sum, k_sq, zws, st);
  else
    e = shape->D == 64 ? qgc_build_td<float, 64>(shape, K, V, P, C, iters, z, labels, perm, offs, counts, k_sum,
                                                 v_sum, k_sq, zws, st)
                       : qgc_build_td<float, 128>(shape, K, V, P, C, iters, z, labels, perm, offs, counts, k_sum,
                                                  v_sum, k_sq, zws, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return qbad(KV_ERR_CUDA, "kv_build_qgc: launch failed");
  }
  return KV_OK;
}

size_t kv_qgc_select_workspace_bytes(const kv_shape* shape) {
  if (!shape || shape->B < 0 || shape->Hkv < 1 || shape->Ncap < 1) return 0;
  return static_cast<size_t>(shape->B) * shape->Hkv * shape->Ncap * sizeof(float);
}

kv_status kv_select_qgc(const kv_shape* shape, const void* q, float scale, const float* P, int C, const void* z16,
                        const int32_t* perm, const int32_t* offs, const int32_t* counts, const float* k_sum,
                        const float* v_sum, const float* k_sq, const void* K, const void* V, float budget,
                        int max_read, int32_t* tok_idx, float* w, int32_t* n_read, float* proxy_k, float* proxy_v,
                        int32_t* proxy_n, void* workspace, size_t ws_bytes, kv_stream_t stream) {
  kv_status st0 = qgc_check_shape(shape, "kv_select_qgc");
  if (st0 != KV_OK) return st0;
  if (C < 1 || C > kvs::QG_MAX_C) return qbad(KV_ERR_INVALID_ARG, "kv_select_qgc: clusters outside 1..64");
  if (!std::isfinite(scale) || !std::isfinite(budget) || budget < 0.f || budget > 1.f)
    return qbad(KV_ERR_INVALID_ARG, "kv_select_qgc: scale not finite or budget outside 0..1");
  const long long need_read = static_cast<long long>(std::floor(static_cast<double>(budget) * shape->Ncap));
  if (max_read < 1 || max_read < need_read)
    return qbad(KV_ERR_INVALID_ARG, "kv_select_qgc: max_read below floor(budget * Ncap)");
  if (!qal(q, 16) || !qal(P, 4) || !qal(z16, 16) || !qal(perm, 4) || !qal(offs, 4) || !qal(counts, 4) ||
      !qal(k_sum, 4) || !qal(v_sum, 4) || !qal(k_sq, 4) || !qal(K, 16) || !qal(V, 16))
    return qbad(KV_ERR_INVALID_ARG, "kv_select_qgc: an input is NULL or misaligned");
  if (!qal(tok_idx, 4) || !qal(w, 4) || !qal(n_read, 4) || !qal(proxy_k, 4) || !qal(proxy_v, 4) || !qal(proxy_n, 4))
    return qbad(KV_ERR_INVALID_ARG, "kv_select_qgc: an output is NULL or misaligned");
  if (!qal(workspace, 16) || ws_bytes < kv_qgc_select_workspace_bytes(shape))
    return qbad(KV_ERR_INVALID_ARG, "kv_select_qgc: workspace NULL, misaligned or too small");
  const int NBH = shape->B * shape->Hkv;
  if (NBH == 0) return KV_OK;
  kvs::QgcSel p{};
  p.q = q;
  p.K = K;
  p.V = V;
  p.seq_lens = shape->seq_lens;
  p.P = P;
  p.z16 = static_cast<const __nv_bfloat16*>(z16);
  p.perm = perm;
  p.offs = offs;
  p.counts = counts;
  p.k_sum = k_sum;
  p.v_sum = v_sum;
  p.k_sq = k_sq;
  p.tok_idx = tok_idx;
  p.w = w;
  p.n_read = n_read;
  p.pk = proxy_k;
  p.pv = proxy_v;
  p.pn = proxy_n;
  p.tws = static_cast<float*>(workspace);
  p.Hq = shape->Hq;
  p.Hkv = shape->Hkv;
  p.Ncap = shape->Ncap;
  p.C = C;
  p.max_read = max_read;
  p.sigma = scale;
  p.budget = budget;
  const int G = shape->Hq / shape->Hkv;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (shape->dtype == KV_BF16)
    e = shape->D == 64 ? qgc_select_td<__nv_bfloat16, 64>(G, p, NBH, st) : qgc_select_td<__nv_bfloat16, 128>(G, p, NBH, st);
  else
    e = shape->D == 64 ? qgc_select_td<float, 64>(G, p, NBH, st) : qgc_select_td<float, 128>(G, p, NBH, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return qbad(KV_ERR_CUDA, "kv_select_qgc: launch failed");
  }
  return KV_OK;
}

kv_status kv_merge_qgc_proxies(const kv_shape* shape, const void* q, float scale, int C, const float* proxy_k,
                               const float* proxy_v, const int32_t* proxy_n, float* out, float* lse,
                               kv_stream_t stream) {
  kv_status st0 = qgc_check_shape(shape, "kv_merge_qgc_proxies");
  if (st0 != KV_OK) return st0;
  if (C < 1 || C > kvs::QG_MAX_C) return qbad(KV_ERR_INVALID_ARG, "kv_merge_qgc_proxies: clusters outside 1..64");
  if (!std::isfinite(scale)) return qbad(KV_ERR_INVALID_ARG, "kv_merge_qgc_proxies: scale not finite");
  if (!qal(q, 16) || !qal(proxy_k, 4) || !qal(proxy_v, 4) || !qal(proxy_n, 4) || !qal(out, 4) || !qal(lse, 4))
    return qbad(KV_ERR_INVALID_ARG, "kv_merge_qgc_proxies: a pointer is NULL or misaligned (lse is required)");
  const long long rows = static_cast<long long>(shape->B) * shape->Hq;
  if (rows == 0) return KV_OK;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (shape->dtype == KV_BF16) {
    if (shape->D == 64)
      kvs::qgc_merge_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), shape->B,
          shape->Hq, shape->Hkv, C, scale, proxy_k, proxy_v, proxy_n, out, lse);
    else
      kvs::qgc_merge_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), shape->B,
          shape->Hq, shape->Hkv, C, scale, proxy_k, proxy_v, proxy_n, out, lse);
  } else {
    if (shape->D == 64)
      kvs::qgc_merge_kernel<float, 64><<<grid, 256, 0, st>>>(static_cast<const float*>(q), shape->B, shape->Hq,
          shape->Hkv, C, scale, proxy_k, proxy_v, proxy_n, out, lse);
    else
      kvs::qgc_merge_kernel<float, 128><<<grid, 256, 0, st>>>(static_cast<const float*>(q), shape->B, shape->Hq,
          shape->Hkv, C, scale, proxy_k, proxy_v, proxy_n, out, lse);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return qbad(KV_ERR_CUDA, "kv_merge_qgc_proxies: launch failed");
  return KV_OK;
}

}  // extern "C"
