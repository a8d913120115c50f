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
//   z = P k for every token (float64 dot products, stored at fp32 in the scratch);
//   Lloyd k-means on z in float64 (starts at the
//   tokens ((2c + 1) n) // (2C'), C' = min(C, n); distance summed over the 16
//   coordinates in order as separately rounded products and sums; ties to the lower
//   cluster; the labels of the last assignment are the clusters; centroid sums per
//   warp over contiguous token ranges, added in warp order); the members of every
//   cluster in ascending token order (a stable counting sort: ranks inside 32-token
//   chunks from match-any masks); per cluster the count, key sum, value sum and
//   per-channel key sum of squares, accumulated in float64 in member order; z at
//   bf16 in member order for the per-query scan (each cluster one contiguous run).
// kv_select_qgc (per query, one CTA per pair):
//   per cluster mu_g = sigma q_g . mean, s2_g = sigma^2 sum_d q_gd^2 var_d, the error
//   E_c = sum_g n_c e^(mu - M_g) expm1(s2 / 2) / Zhat_g, Zhat_g = sum_c n_c e^(mu + s2/2 - M_g);
//   the read budget R = floor(budget n) - ceil(1.5 C_live) and r_c = min(n_c,
//   floor(R E_c / sum E)); token scores t_i = sum_g exp(sigma (P q_g) . z16_i - LSE_g)
//   in two passes over the members on the tensor cores; in every cluster the r_c
//   tokens of largest (t, then lower index), from its contiguous run of scores, by
//   repeated maxima or bisection on the 64-bit key (t's bits, inverted position); the read list
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
#include <type_traits>

#include "common.cuh"
#include "kvsparse.h"

namespace kvs {
void set_last_error(const char* msg);

constexpr int QG_THREADS = 512;
constexpr int QG_NW = QG_THREADS / 32;
constexpr int QG_DIM = 16;     // projection dimension
constexpr int QG_MAX_C = 64;   // clusters per (sequence, KV head)
constexpr int QG_STAGES = 3;          // ring stages a warp
constexpr int QG_CHUNK = 4096;        // ring stage bytes: 128 tokens' bf16 projections
constexpr int QG_CHUNK_TOK = QG_CHUNK / (QG_DIM * 2);
// The per-query selection runs 256 threads a CTA, two CTAs an SM: while one CTA of an
// SM streams its projections, the other can run its cluster phase.
constexpr int QS_THREADS = 256;
constexpr int QS_NW = QS_THREADS / 32;
constexpr int QG_RING = QS_NW * QG_STAGES * QG_CHUNK;  // dynamic shared memory of the selection (96 KB)

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

  // ---- 1. projection z = P k (float64), stored at fp32 (scratch)
  constexpr int CH = 16 / sizeof(T);
  for (int i = tid; i < Ncap; i += QG_THREADS) {
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
      for (int j = 0; j < QG_DIM; ++j) Z[static_cast<size_t>(i) * QG_DIM + j] = static_cast<float>(a[j]);
    } else {
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

  // ---- 3b. the bf16 projections in member order (entry m: token pm[m]; zero past n),
  // so that the per-query scan reads every cluster's tokens as one contiguous run
  for (int e = tid; e < Ncap * 2; e += QG_THREADS) {
    const int m = e >> 1, hf = e & 1;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (m < n) {
      const float* zr = Z + static_cast<size_t>(pm[m]) * QG_DIM + 8 * hf;
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(zr[2 * k], zr[2 * k + 1]);
        w[k] = *reinterpret_cast<const uint32_t*>(&v);
      }
      o = make_uint4(w[0], w[1], w[2], w[3]);
    }
    reinterpret_cast<uint4*>(z16 + (tok0 + m) * QG_DIM)[hf] = o;
  }

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

// A lane's CPL consecutive channels of a row as loaded (one vector) -> fp32.
template <typename T, int CPL, typename R>
__device__ __forceinline__ void qg_unpack(const R& r, float (&x)[CPL]) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (CPL == 4) {
      x[0] = __uint_as_float(r.x << 16);
      x[1] = __uint_as_float(r.x & 0xffff0000u);
      x[2] = __uint_as_float(r.y << 16);
      x[3] = __uint_as_float(r.y & 0xffff0000u);
    } else {
      x[0] = __uint_as_float(r << 16);
      x[1] = __uint_as_float(r & 0xffff0000u);
    }
  } else {
    if constexpr (CPL == 4) {
      x[0] = r.x;
      x[1] = r.y;
      x[2] = r.z;
      x[3] = r.w;
    } else {
      x[0] = r.x;
      x[1] = r.y;
    }
  }
}

// D += A B, m16n8k16, bf16 inputs, fp32 accumulation (a: the four A words in
// fragment order, b0 / b1: the two B words)
__device__ __forceinline__ void qg_mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The rc-th largest of the keys of members m0 .. m1 - 1 (distinct 64-bit keys,
// 1 <= rc < m1 - m0), by one warp: radix selection on 8-bit digits from the highest
// bit where the keys differ (a histogram of the digit among the keys that match the
// digits chosen so far; the digit whose range holds the rc-th key is kept), until at
// most 32 keys match; those are ranked directly. a, o: the AND and the OR of all the
// keys (the same in every lane). hist: 256 counters, cand: 32 keys, both the warp's own.
template <typename KeyOf>
__device__ unsigned long long qg_kth_largest(KeyOf key_of, int m0, int m1, int rc, unsigned long long a,
                                             unsigned long long o, unsigned* hist, unsigned long long* cand,
                                             int lane) {
  const int hb = 63 - __clzll(static_cast<long long>(a ^ o));  // >= 0: at least two distinct keys
  unsigned long long pmask = hb == 63 ? 0ull : ~((2ull << hb) - 1ull);  // bits above hb: shared
  unsigned long long prefix = a & pmask;
  unsigned need = static_cast<unsigned>(rc);  // rank of the threshold among the keys matching prefix
  for (int top = hb;; top -= 8) {
    const int lo = top - 7;  // the digit is bits max(lo, 0) .. top
    const unsigned long long dmask = lo >= 0 ? (255ull << lo) : (255ull >> (-lo));
    for (int bn = lane; bn < 256; bn += 32) hist[bn] = 0u;
    __syncwarp();
    for (int m = m0 + lane; m < m1; m += 32) {
      const unsigned long long x = key_of(m);
      if ((x & pmask) == prefix)
        atomicAdd(hist + static_cast<int>(lo >= 0 ? (x >> lo) & 255ull : (x << (-lo)) & 255ull), 1u);
    }
    __syncwarp();
    // lane L holds bins 255 - 8L - j (j < 8), so lower lanes hold higher digits
    unsigned cb[8], sum = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      cb[j] = hist[255 - 8 * lane - j];
      sum += cb[j];
    }
    unsigned incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const unsigned v = __shfl_up_sync(FULL_MASK, incl, d);
      if (lane >= d) incl += v;
    }
    const unsigned excl = incl - sum;  // keys in higher digits than this lane's
    const bool mine = excl < need && need <= incl;
    const int src = __ffs(__ballot_sync(FULL_MASK, mine)) - 1;
    unsigned dig = 0u, above = 0u, cdig = 0u;
    if (mine) {
      unsigned acc = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (cdig == 0u && acc + cb[j] >= need) {
          dig = static_cast<unsigned>(255 - 8 * lane - j);
          above = acc;
          cdig = cb[j];
        }
        acc += cb[j];
      }
    }
    dig = __shfl_sync(FULL_MASK, dig, src);
    above = __shfl_sync(FULL_MASK, above, src);
    cdig = __shfl_sync(FULL_MASK, cdig, src);
    need -= above;
    prefix |= lo >= 0 ? (static_cast<unsigned long long>(dig) << lo) : (static_cast<unsigned long long>(dig) >> (-lo));
    pmask |= dmask;
    if (cdig <= 32u) break;  // always by the last digit: the keys are distinct
  }
  // the (at most 32) keys matching prefix, compacted, then ranked
  int base = 0;
  for (int m = m0; m < m1; m += 32) {
    const int mi = m + lane;
    const unsigned long long x = mi < m1 ? key_of(mi) : 0ull;
    const bool match = mi < m1 && (x & pmask) == prefix;
    const unsigned bal = __ballot_sync(FULL_MASK, match);
    const int slot = base + __popc(bal & ((1u << lane) - 1u));
    if (match && slot < 32) cand[slot] = x;  // (never more than 32: the keys are distinct)
    base += __popc(bal);
  }
  __syncwarp();
  base = min(base, 32);
  const unsigned long long kj = lane < base ? cand[lane] : 0ull;
  unsigned rank = 0u;
  for (int i = 0; i < base; ++i) rank += cand[i] > kj;
  const int win = max(__ffs(__ballot_sync(FULL_MASK, lane < base && rank == need - 1u)) - 1, 0);
  __syncwarp();  // cand and hist are free again
  return __shfl_sync(FULL_MASK, kj, win);
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
  float pmx[QS_NW][8], psm[QS_NW][8];
  alignas(8) unsigned long long rbar[QS_NW][QG_STAGES];
  unsigned long long cand[QS_NW][32];  // the radix selection's last candidates, per warp
  unsigned hist[QS_NW][256];           // its digit histogram, per warp
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(QS_THREADS, 2) qgc_select_kernel(const QgcSel p) {
  __shared__ QgcSelShared sh;
  extern __shared__ __align__(128) unsigned char qg_ring[];  // the warps' rings, then their score runs
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
  float* t = p.tws + static_cast<size_t>(bh) * p.Ncap;  // token scores in member order
  unsigned char* ring = qg_ring + static_cast<size_t>(warp) * QG_STAGES * QG_CHUNK;
  uint64_t* rbar = reinterpret_cast<uint64_t*>(sh.rbar[warp]);
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < QG_STAGES; ++k) mbar_init(rbar + k, 1);
    fence_mbar_init();
  }
  __syncwarp();
  // The projections stream through the warp's ring: chunk j of warp w is tokens
  // 128 (w + QS_NW j) .. + 127 in member order, one bulk copy into stage j % QG_STAGES;
  // both passes take the same chunk sequence (copy u < nmine of pass 1, u - nmine of
  // pass 2). A lane reads its A words from the stage: token row r at r * 32 bytes,
  // coordinates 4tq .. 4tq + 3 at + 8 tq (8 rows x 32 bytes a warp load, no conflicts).
  const unsigned char* zsrc = reinterpret_cast<const unsigned char*>(p.z16) + static_cast<size_t>(bh) * p.Ncap * QG_DIM * 2;
  const int nck = (n + QG_CHUNK_TOK - 1) / QG_CHUNK_TOK;
  const int nmine = nck > warp ? (nck - warp + QS_NW - 1) / QS_NW : 0;
  // evict-first in both passes: keeping a share of pass 1 in L2 for pass 2 (evict-last)
  // measured no faster
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int u) {
    if (u >= 2 * nmine) return;  // warp-uniform
    const int ck = warp + QS_NW * (u < nmine ? u : u - nmine);
    const int rows = min(QG_CHUNK_TOK, n - ck * QG_CHUNK_TOK);  // >= 1
    if (lane == 0) {
      uint64_t* bar = rbar + u % QG_STAGES;
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * QG_DIM * 2);
      bulk_g2s(ring + (u % QG_STAGES) * QG_CHUNK, zsrc + static_cast<size_t>(ck) * QG_CHUNK,
               static_cast<uint32_t>(rows) * QG_DIM * 2, bar, pol);
    }
  };
  // the first copies go out before the cluster statistics, so their latency overlaps them
#pragma unroll
  for (int u = 0; u < QG_STAGES; ++u) issue(u);

  // the group's queries, a lane CPL channels of each
  float qf[G][CPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int k = 0; k < CPL; ++k) qf[g][k] = load_as_float(qrow + g * D + lane * CPL + k);

  // ---- projected queries q~_g = P q_g (warp w: rows w, w + QS_NW of P, both loaded
  // before the first use)
  static_assert(QG_DIM == 2 * QS_NW, "two projection rows a warp");
  {
    float u[2][CPL];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int k = 0; k < CPL; ++k)
        u[r][k] = __ldg(p.P + (static_cast<size_t>(h) * QG_DIM + warp + r * QS_NW) * D + lane * CPL + k);
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = 0.f;
#pragma unroll
        for (int k = 0; k < CPL; ++k) v = fmaf(u[r][k], qf[g][k], v);
        v = warp_sum(v);
        if (lane == 0) sh.qt[g][warp + r * QS_NW] = v;
      }
  }

  // ---- per cluster mean logit and logit variance (a warp per cluster; a warp's
  // clusters four at a time, their cached tokens all requested before the first use)
  for (int c0 = warp; c0 < C; c0 += 4 * QS_NW) {
    float ksr[4][CPL], kqr[4][CPL];
    int ncr[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u * QS_NW;
      const size_t o = (static_cast<size_t>(bh) * C + (c < C ? c : 0)) * D + lane * CPL;
      ncr[u] = c < C ? __ldg(cnt + c) : 0;
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        ksr[u][k] = c < C ? __ldg(p.k_sum + o + k) : 0.f;
        kqr[u][k] = c < C ? __ldg(p.k_sq + o + k) : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u * QS_NW;
      if (c >= C) break;  // warp-uniform
      const int nc = ncr[u];
      float mean[CPL], var[CPL];
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const float m = nc > 0 ? __fdiv_rn(ksr[u][k], static_cast<float>(nc)) : 0.f;
        const float sq = nc > 0 ? __fdiv_rn(kqr[u][k], static_cast<float>(nc)) : 0.f;
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

  // ---- token scores in member order: LSE per head over the tokens, then t_m (two
  // passes over the bf16 projections on the tensor cores). mma.sync m16n8k16: the 16
  // tokens of a step as M, the 16 coordinates as K, the G <= 8 heads as N. The bf16
  // projections are exact operands; sigma q~ is split into a bf16 high part and a
  // bf16 remainder (two products into one fp32 accumulator, about 16 significant
  // bits of sigma q~). K is taken in the order the A words load: MMA k = 2tq + e is
  // coordinate 4tq + e and k = 2tq + 8 + e is 4tq + 2 + e (tq = lane % 4), so a lane
  // reads coordinates 4tq .. 4tq + 3 of its two rows as one 8-byte word pair each.
  // With G <= 4 one product does both parts: B's columns 0..3 are the heads' high
  // parts and 4..7 their remainders, so lanes tq and tq + 2 hold the two parts of the
  // same heads; one exchange adds them, lane tq < 2 keeping row gq and lane tq >= 2 row
  // gq + 8, and each lane then has one row's logits for heads 2 (tq % 2) and + 1.
  {
    constexpr bool PK = G <= 4;
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t bhi[2], blo[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int hd = PK ? (gq & 3) : gq;  // the head of B column gq
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) v[e] = hd < G ? p.sigma * sh.qt[hd < G ? hd : 0][4 * tq + 2 * k + e] : 0.f;
      const __nv_bfloat162 hv = __floats2bfloat162_rn(v[0], v[1]);
      const float2 hf = __bfloat1622float2(hv);
      const __nv_bfloat162 lv = __floats2bfloat162_rn(v[0] - hf.x, v[1] - hf.y);
      bhi[k] = *reinterpret_cast<const uint32_t*>(PK && gq >= 4 ? &lv : &hv);
      blo[k] = *reinterpret_cast<const uint32_t*>(&lv);
    }
    // waits for copy u and returns its stage (a bounded wait: a copy that never lands
    // leaves stale words, never a hang)
    auto stage_of = [&](int u) {
      const int k = u % QG_STAGES;
      if (!mbar_wait(rbar + k, static_cast<uint32_t>((u / QG_STAGES) & 1), nullptr))
        mbar_wait(rbar + k, static_cast<uint32_t>((u / QG_STAGES) & 1), nullptr);
      return ring + k * QG_CHUNK;
    };
    // after the warp's last read of copy u's stage: the copy that refills it
    auto release = [&](int u) {
      __syncwarp();
      fence_proxy_async_smem();
      issue(u + QG_STAGES);
    };
    // the logits of a 16-token step at row offset r16 of a stage: c[0..1] the heads
    // 2tq, 2tq + 1 of token row r16 + gq, c[2..3] those of row r16 + gq + 8
    auto step_logits = [&](const unsigned char* stg, int r16, float (&c)[4]) {
      const uint2 ra = *reinterpret_cast<const uint2*>(stg + (r16 + gq) * 32 + 8 * tq);
      const uint2 rb = *reinterpret_cast<const uint2*>(stg + (r16 + gq + 8) * 32 + 8 * tq);
      const uint32_t a[4] = {ra.x, rb.x, ra.y, rb.y};
      c[0] = c[1] = c[2] = c[3] = 0.f;
      qg_mma_bf16(c, a, bhi[0], bhi[1]);
      if constexpr (!PK) qg_mma_bf16(c, a, blo[0], blo[1]);
    };
    // G <= 4: this lane's row (r16 + gq, + 8 when tq >= 2) and its two logits
    const int prow = tq >= 2 ? gq + 8 : gq;
    auto step_pair = [&](const unsigned char* stg, int r16, float (&v)[2]) {
      float c[4];
      step_logits(stg, r16, c);
      const float x0 = tq < 2 ? c[2] : c[0], x1 = tq < 2 ? c[3] : c[1];
      const float y0 = __shfl_xor_sync(FULL_MASK, x0, 2), y1 = __shfl_xor_sync(FULL_MASK, x1, 2);
      v[0] = tq < 2 ? c[0] + y0 : y0 + c[2];
      v[1] = tq < 2 ? c[1] + y1 : y1 + c[3];
    };
    const int hb = PK ? 2 * (tq & 1) : 2 * tq;  // this lane's heads: hb, hb + 1
    const bool h0 = hb < G, h1 = hb + 1 < G;
    float mx[2] = {-INFINITY, -INFINITY}, sm[2] = {0.f, 0.f};
    for (int j = 0; j < nmine; ++j) {
      const unsigned char* stg = stage_of(j);
      const int tok0 = (warp + QS_NW * j) * QG_CHUNK_TOK;
      const int nst = min(QG_CHUNK_TOK, n - tok0 + 15) >> 4;  // steps with a live row
#pragma unroll 2
      for (int k = 0; k < nst; ++k) {
        if constexpr (PK) {
          // one value a head: the smaller of (running max, value) minus the larger,
          // one exponential, and the running sum rescaled when the value is larger
          const int r = tok0 + 16 * k + prow;
          float v[2];
          step_pair(stg, 16 * k, v);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x = r < n ? v[e] : -INFINITY;
            const float mn = fmaxf(mx[e], x);
            if (mn != -INFINITY) {
              const float ex = __expf(fminf(mx[e], x) - mn);
              sm[e] = x > mx[e] ? fmaf(sm[e], ex, 1.f) : sm[e] + ex;
              mx[e] = mn;
            }
          }
        } else {
          const int r0 = tok0 + 16 * k + gq;
          float c[4];
          step_logits(stg, 16 * k, c);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {  // rows r0, r0 + 8: one exponential each
              const float x = r0 + 8 * hf < n ? c[2 * hf + e] : -INFINITY;
              const float mn = fmaxf(mx[e], x);
              if (mn != -INFINITY) {
                const float ex = __expf(fminf(mx[e], x) - mn);
                sm[e] = x > mx[e] ? fmaf(sm[e], ex, 1.f) : sm[e] + ex;
                mx[e] = mn;
              }
            }
          }
        }
      }
      release(j);
    }
    // combine over the lanes of a head column (and, with G <= 4, of both row halves),
    // then over the warps
#pragma unroll
    for (int e = 0; e < 2; ++e) {
#pragma unroll
      for (int o = PK ? 2 : 4; o <= 16; o <<= 1) {
        if (o == 2 && !PK) continue;
        const float m2 = __shfl_xor_sync(FULL_MASK, mx[e], o), s2 = __shfl_xor_sync(FULL_MASK, sm[e], o);
        const float M = fmaxf(mx[e], m2);
        if (M != -INFINITY) {
          sm[e] = (mx[e] == -INFINITY ? 0.f : sm[e] * __expf(mx[e] - M)) + (m2 == -INFINITY ? 0.f : s2 * __expf(m2 - M));
          mx[e] = M;
        }
      }
    }
    if (gq == 0 && (!PK || tq < 2)) {
      if (h0) {
        sh.pmx[warp][hb] = mx[0];
        sh.psm[warp][hb] = sm[0];
      }
      if (h1) {
        sh.pmx[warp][hb + 1] = mx[1];
        sh.psm[warp][hb + 1] = sm[1];
      }
    }
    __syncthreads();
    if (tid < G) {
      float M = -INFINITY;
      for (int w = 0; w < QS_NW; ++w) M = fmaxf(M, sh.pmx[w][tid]);
      float L = 0.f;
      if (M != -INFINITY)
        for (int w = 0; w < QS_NW; ++w)
          if (sh.pmx[w][tid] != -INFINITY) L += sh.psm[w][tid] * __expf(sh.pmx[w][tid] - M);
      sh.lse[tid] = M == -INFINITY ? -INFINITY : M + __logf(L);
    }
    __syncthreads();
    const float le0 = h0 ? sh.lse[hb] : 0.f, le1 = h1 ? sh.lse[hb + 1] : 0.f;
    for (int j = 0; j < nmine; ++j) {
      const unsigned char* stg = stage_of(nmine + j);
      const int tok0 = (warp + QS_NW * j) * QG_CHUNK_TOK;
      const int nst = min(QG_CHUNK_TOK, n - tok0 + 15) >> 4;
#pragma unroll 2
      for (int k = 0; k < nst; ++k) {
        if constexpr (PK) {
          // the lanes tq, tq ^ 1 hold the same row's heads 0, 1 and 2, 3
          const int r = tok0 + 16 * k + prow;
          float v[2];
          step_pair(stg, 16 * k, v);
          float ta = (h0 ? __expf(v[0] - le0) : 0.f) + (h1 ? __expf(v[1] - le1) : 0.f);
          ta += __shfl_xor_sync(FULL_MASK, ta, 1);
          if ((tq & 1) == 0 && r < n) t[r] = ta;
          continue;
        }
        const int r0 = tok0 + 16 * k + gq;
        float c[4];
        step_logits(stg, 16 * k, c);
        float ta = (h0 ? __expf(c[0] - le0) : 0.f) + (h1 ? __expf(c[1] - le1) : 0.f);
        float tb = (h0 ? __expf(c[2] - le0) : 0.f) + (h1 ? __expf(c[3] - le1) : 0.f);
        ta += __shfl_xor_sync(FULL_MASK, ta, 1);
        tb += __shfl_xor_sync(FULL_MASK, tb, 1);
        ta += __shfl_xor_sync(FULL_MASK, ta, 2);
        tb += __shfl_xor_sync(FULL_MASK, tb, 2);
        if (tq == 0) {
          if (r0 < n) t[r0] = ta;
          if (r0 + 8 < n) t[r0 + 8] = tb;
        }
      }
      release(nmine + j);
    }
  }
  __syncthreads();  // every score is written; the rings are idle (no copy in flight)

  // ---- per cluster: the r_c largest keys (t's bits, inverted member position), the
  // read list, the read rows' sums and the proxy of the unread tokens (a warp per
  // cluster). Members are in ascending token order inside a cluster, so the inverted
  // member position orders ties as the inverted token index does. A cluster's scores
  // are one contiguous run of the scratch, first copied into the warp's idle ring (up
  // to QG_RUN scores; longer runs are read from the scratch).
  constexpr int QG_RUN = QG_STAGES * QG_CHUNK / 4;
  float* run = reinterpret_cast<float*>(ring);
  for (int c = warp; c < C; c += QS_NW) {
    const int nc = cnt[c], rc = sh.r[c];
    const int m0 = off[c], m1 = off[c + 1];
    const float* tc = t + m0;
    unsigned tand = ~0u, tor = 0u;  // AND and OR of the cluster's score bits
    __syncwarp();  // the previous cluster's reads of the run are done
    // the proxy's cluster sums, needed at the end, requested now
    const size_t o = (static_cast<size_t>(bh) * C + c) * D + lane * CPL;
    float ksum[CPL], vsum[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      ksum[k] = __ldg(p.k_sum + o + k);
      vsum[k] = __ldg(p.v_sum + o + k);
    }
    if (rc > 0 && rc < nc && nc <= QG_RUN) {
      // 16 loads a lane in flight per round; the AND and OR of the score bits on the way
      for (int m = lane; m < nc; m += 32 * 16) {
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = m + 32 * k < nc ? __ldcg(tc + m + 32 * k) : 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (m + 32 * k < nc) {
            run[m + 32 * k] = v[k];
            tand &= __float_as_uint(v[k]);
            tor |= __float_as_uint(v[k]);
          }
      }
      __syncwarp();
      tc = run;
    } else if (rc > 0 && rc < nc) {
      for (int m = lane; m < nc; m += 32) {
        tand &= __float_as_uint(tc[m]);
        tor |= __float_as_uint(tc[m]);
      }
    }
    auto key_of = [&](int m) {
      return (static_cast<unsigned long long>(__float_as_uint(tc[m - m0])) << 32) |
             static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(m));
    };
    unsigned long long thr = 0ull;  // keys >= thr are read
    if (rc > 0 && rc < nc) {
      // AND and OR of the keys: the score bits' from the lanes; the inverted positions
      // are the contiguous range [2^32 - m1, 2^32 - 1 - m0], whose AND and OR are its
      // common high bits followed by zeros and by ones
      const unsigned ha = __reduce_and_sync(FULL_MASK, tand), ho = __reduce_or_sync(FULL_MASK, tor);
      const unsigned lo_v = 0xffffffffu - static_cast<uint32_t>(m1 - 1), hi_v = 0xffffffffu - static_cast<uint32_t>(m0);
      const unsigned dv = lo_v ^ hi_v;
      const unsigned lmask = dv == 0u ? 0u : (0xffffffffu >> __clz(dv));
      const unsigned long long ka = (static_cast<unsigned long long>(ha) << 32) | (lo_v & ~lmask);
      const unsigned long long ko = (static_cast<unsigned long long>(ho) << 32) | (lo_v | lmask);
      thr = qg_kth_largest(key_of, m0, m1, rc, ka, ko, sh.hist[warp], sh.cand[warp], lane);
    }
    float rk[CPL], rv[CPL];
#pragma unroll
    for (int k = 0; k < CPL; ++k) rk[k] = rv[k] = 0.f;
    // the read list of the cluster: the takers' member positions are collected in
    // the warp's shared list (up to 256 a round; hist is free after the selection),
    // then turned into token indices with all their loads in flight, then written
    int* li = reinterpret_cast<int*>(sh.hist[warp]);
    const int nl = rc > 0 ? min(rc, p.max_read - sh.roff[c]) : 0;
    if (rc > 0) {
      int32_t* lo_idx = p.tok_idx + static_cast<size_t>(bh) * p.max_read + sh.roff[c];
      float* lo_w = p.w + static_cast<size_t>(bh) * p.max_read + sh.roff[c];
      int mb = m0, done = 0;  // members scanned up to mb; list entries written: done
      while (done < nl) {
        int cnt_r = 0;  // entries of this round, at most 256
        for (; mb < m1 && cnt_r < 256 - 32; mb += 32) {
          const int mi = mb + lane;
          const bool take = mi < m1 && (rc >= nc || key_of(mi) >= thr);
          const unsigned bal = __ballot_sync(FULL_MASK, take);
          if (take) li[cnt_r + __popc(bal & ((1u << lane) - 1u))] = mi;
          cnt_r += __popc(bal);
        }
        __syncwarp();
        const int nr = min(cnt_r, nl - done);
        for (int j0 = 0; j0 < nr; j0 += 32 * 8) {
          int tk[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = j0 + 32 * u + lane;
            tk[u] = j < nr ? __ldg(pm + li[j]) : 0;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = j0 + 32 * u + lane;
            if (j < nr) {
              li[j] = tk[u];
              lo_idx[done + j] = tk[u];
              lo_w[done + j] = 1.f;
            }
          }
        }
        __syncwarp();
        // the read rows' key and value sums of this round, RW rows' loads in flight
        using Raw = typename std::conditional<sizeof(T) == 2, typename std::conditional<CPL == 4, uint2, uint32_t>::type,
                                              typename std::conditional<CPL == 4, float4, float2>::type>::type;
        constexpr int RW = sizeof(Raw) >= 16 ? 6 : 12;  // 48 registers of rows at most
        for (int j0 = 0; j0 < nr; j0 += RW) {
          Raw kr[RW], vr[RW];
#pragma unroll
          for (int u = 0; u < RW; ++u) {
            if (j0 + u < nr) {
              const int ti = li[j0 + u];
              kr[u] = __ldg(reinterpret_cast<const Raw*>(Kb + static_cast<size_t>(ti) * D) + lane);
              vr[u] = __ldg(reinterpret_cast<const Raw*>(Vb + static_cast<size_t>(ti) * D) + lane);
            }
          }
#pragma unroll
          for (int u = 0; u < RW; ++u) {
            if (j0 + u < nr) {
              float kx[CPL], vx[CPL];
              qg_unpack<T, CPL>(kr[u], kx);
              qg_unpack<T, CPL>(vr[u], vx);
#pragma unroll
              for (int k = 0; k < CPL; ++k) {
                rk[k] += kx[k];
                rv[k] += vx[k];
              }
            }
          }
        }
        __syncwarp();  // li is refilled by the next round
        done += nr;
        if (mb >= m1) break;
      }
    }
    const int un = nc - rc;  // unread tokens of the cluster
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      p.pk[o + k] = un > 0 ? __fdiv_rn(ksum[k] - rk[k], static_cast<float>(un)) : 0.f;
      p.pv[o + k] = un > 0 ? __fdiv_rn(vsum[k] - rv[k], static_cast<float>(un)) : 0.f;
    }
    if (lane == 0) p.pn[static_cast<size_t>(bh) * C + c] = max(un, 0);
  }
  // padding of the read list
  for (int q = sh.roff[C] + tid; q < p.max_read; q += QS_THREADS) {
    p.tok_idx[static_cast<size_t>(bh) * p.max_read + q] = 0;
    p.w[static_cast<size_t>(bh) * p.max_read + q] = 0.f;
  }
}

// Folds the proxies into the attention over the read tokens: a warp per query head,
// lanes over the channels, sixteen proxies at a time. With the read tokens' (out, lse) and proxy logits
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
  // proxy logits sixteen at a time: all sixteen rows' loads first, then one transpose
  // reduction leaves proxy c0 + j's dot product in the lanes with (lane >> 1) == j
  constexpr int PB = 16;
  float M = lse[row];
  for (int c0 = 0; c0 < C; c0 += PB) {
    float part[PB];
    int ncs[PB];
#pragma unroll
    for (int j = 0; j < PB; ++j) {
      const int c = c0 + j;
      ncs[j] = c < C ? pn[bh * C + c] : 0;
      float kv[CPL];
#pragma unroll
      for (int k = 0; k < CPL; ++k) kv[k] = c < C ? pk[(bh * C + c) * D + lane * CPL + k] : 0.f;
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < CPL; ++k) a = fmaf(qf[k], kv[k], a);
      part[j] = a;
    }
    transpose_reduce<PB, 16>(part, lane);
    const int j = (lane >> 1) & (PB - 1);
    int nc = ncs[0];
#pragma unroll
    for (int jj = 1; jj < PB; ++jj)
      if (jj == j) nc = ncs[jj];
    const float lc = (c0 + j < C && nc > 0) ? sigma * part[0] + __logf(static_cast<float>(nc)) : -INFINITY;
    if ((lane & 1) == 0 && c0 + j < C) lgs[warp][c0 + j] = lc;
    M = fmaxf(M, warp_max(lc));
  }
  __syncwarp();
  if (M == -INFINITY) return;  // nothing read and no proxy (an empty sequence)
  const float l0 = lse[row];
  const float a0 = l0 == -INFINITY ? 0.f : __expf(l0 - M);
  float den = a0;
  float o[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) o[k] = a0 * out[static_cast<size_t>(row) * D + lane * CPL + k];
  // the proxies' values sixteen at a time, all sixteen rows' loads first
  for (int c0 = 0; c0 < C; c0 += PB) {
    float vv[PB][CPL], e[PB];
#pragma unroll
    for (int j = 0; j < PB; ++j) {
      const int c = c0 + j;
      const float lc = c < C ? lgs[warp][c] : -INFINITY;
      e[j] = lc == -INFINITY ? 0.f : __expf(lc - M);
#pragma unroll
      for (int k = 0; k < CPL; ++k) vv[j][k] = lc != -INFINITY ? pv[(bh * C + c) * D + lane * CPL + k] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < PB; ++j) {
      den += e[j];
#pragma unroll
      for (int k = 0; k < CPL; ++k) o[k] = fmaf(e[j], vv[j][k], o[k]);
    }
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
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kvs::QG_RING); \
      if (e != cudaSuccess) return e;                                                                    \
      cfg_##GG.fetch_or(1 << (dev & 31));                                                                \
    }                                                                                                    \
    kvs::qgc_select_kernel<T, D, GG><<<grid, kvs::QS_THREADS, kvs::QG_RING, st>>>(p);                    \
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
