// Per-KV-head block choice for one decode step.
//
// Sources: "COBS: Cumulant Order Block Sparse Attention" -- Equation (5): a KV
// head's shared block set is ranked by the group score, the sum over its G query
// heads of per-head block softmax probabilities m_b / Z^(g,h); the first-order
// (mean-pool) estimate of ln m_b, s = q . (block mean key) + ln n_b (text after
// Equation (8) and the affine score (18)); OSA computes the exact masses from all
// block keys instead (the OSA paragraph).
//
// Design (sm_100a). One thread-block cluster of SEL_CS CTAs per (sequence, KV
// head). Each CTA scores a contiguous slice of the blocks into shared memory
// (summary mode: a GEMV over the fp32 key sums, 16-byte loads, transpose
// reduction; exact mode: all block keys, an online log-sum-exp per block), then
// the cluster exchanges per-head (max, sum) pairs through distributed shared
// memory to form the normalisers, each CTA ranks its candidates locally, and the
// global rank of a candidate is its local rank plus a binary search in every other
// CTA's sorted candidate list. Selected blocks are written in ascending order.
// Nothing goes through global scratch memory and no CTA spins on another:
// cluster barriers are hardware barriers of co-scheduled CTAs.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace kvs {

namespace cg = cooperative_groups;

constexpr int SEL_CS = 8;          // CTAs per cluster (one cluster per bh)
constexpr int SEL_THREADS = 256;   // 8 warps
constexpr int SEL_NW = SEL_THREADS / 32;
constexpr int SEL_MAXNB = 4096;    // NBcap limit
constexpr int SEL_MAXLOCAL = SEL_MAXNB / SEL_CS;

enum SelMode { SEL_SUMMARY = 0, SEL_EXACT = 1 };

struct SelParams {
  const void* q;
  const float* k_sum;
  const int32_t* counts;
  const void* K;
  const int32_t* seq_lens;
  int32_t* block_idx;
  int32_t* n_kept;
  float* scores;
  int B, Hq, Hkv, Ncap, L, NBcap;
  int k_top, force_first, force_last, kmax;
  float qscale;  // softmax scale * log2(e)
};

template <int G>
struct SelShared {
  float lg[G][SEL_MAXLOCAL];               // block log2-mass estimates
  unsigned long long key[SEL_MAXLOCAL];    // ranking keys (0 = not competing)
  unsigned long long cand[SEL_MAXLOCAL];   // local candidates, descending
  float2 part[G];                          // per-head (max, sum) over the slice
  float lse[G];
  int flag[SEL_MAXLOCAL];
  int wsum[SEL_NW];
  int ncand;
  int nsel;
};

// Sum of one int per thread over the CTA; every thread gets the result.
__device__ __forceinline__ int block_sum(int v, int* wsum) {
  v = __reduce_add_sync(FULL_MASK, v);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int w = 0; w < SEL_NW; ++w) s += wsum[w];
  __syncthreads();
  return s;
}

__device__ __forceinline__ int count_greater(const unsigned long long* arr, int n, unsigned long long x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (arr[mid] > x)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

// Summary mode: s2[g][i] = (q_g * qscale) . k_sum_b / n_b + log2 n_b for the
// slice [lo, lo + nl) of blocks.
template <typename T, int D, int G>
__device__ void score_summary(const SelParams& p, SelShared<G>& sh, int bh, int lo, int nl) {
  constexpr int LPR = D / 4;  // fp32 rows, float4 per lane
  constexpr int RPW = 32 / LPR;
  constexpr int GP = pow2ceil(G);
  constexpr int RS0 = LPR / GP;
  constexpr int RS = RS0 < 1 ? 1 : (RS0 > 8 ? 8 : RS0);  // rows per lane per batch
  constexpr int NV = RS * GP;
  using HV = HeldValues<NV, LPR, GP>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane / LPR, c = lane % LPR;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * D + c * 4;
  float4 qf[G];
#pragma unroll
  for (int g = 0; g < G; ++g)
    qf[g] = make_float4(load_as_float(qrow + g * D) * p.qscale, load_as_float(qrow + g * D + 1) * p.qscale,
                        load_as_float(qrow + g * D + 2) * p.qscale, load_as_float(qrow + g * D + 3) * p.qscale);
  const float* ks = p.k_sum + (static_cast<size_t>(bh) * p.NBcap + lo) * D + c * 4;
  const int32_t* cn = p.counts + static_cast<size_t>(b) * p.NBcap + lo;
  constexpr int BATCH = RPW * RS;
  for (int rb = warp * BATCH; rb < nl; rb += SEL_NW * BATCH) {
    float part[NV];
    int cnt[RS];
#pragma unroll
    for (int i = 0; i < RS; ++i) {
      const int row = rb + i * RPW + rg;
      float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f);
      cnt[i] = 0;
      if (row < nl) {
        k4 = __ldg(reinterpret_cast<const float4*>(ks + static_cast<size_t>(row) * D));
        cnt[i] = __ldg(cn + row);
      }
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        if (g < G) {
          float d = qf[g].x * k4.x;
          d = fmaf(qf[g].y, k4.y, d);
          d = fmaf(qf[g].z, k4.z, d);
          d = fmaf(qf[g].w, k4.w, d);
          part[i * GP + g] = d;
        } else {
          part[i * GP + g] = 0.f;
        }
      }
    }
    transpose_reduce<NV, LPR / 2>(part, lane);
#pragma unroll
    for (int j = 0; j < HV::NH; ++j) {
      const int vi = HV::index(c, j);
      const int ri = vi / GP, g = vi % GP;
      const int row = rb + ri * RPW + rg;
      int nb = cnt[0];
#pragma unroll
      for (int i = 1; i < RS; ++i)
        if (ri == i) nb = cnt[i];
      if (g < G && row < nl)
        sh.lg[g][row] = nb > 0 ? part[j] / static_cast<float>(nb) + log2f(static_cast<float>(nb)) : -INFINITY;
    }
  }
}

// Exact mode: s2[g][i] = log2 sum_{r in block} exp2((q_g * qscale) . k_r).
template <typename T, int D, int G>
__device__ void score_exact(const SelParams& p, SelShared<G>& sh, int bh, int lo, int nl, int n) {
  constexpr int ES = sizeof(T);
  constexpr int RB = D * ES;
  constexpr int LPR = RB / 16;
  constexpr int RPW = 32 / LPR;
  constexpr int CH2 = 8 / ES;
  constexpr int R = 4;
  constexpr int GP = pow2ceil(G);
  constexpr int NV = R * GP;
  using HV = HeldValues<NV, LPR, GP>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane / LPR, c = lane % LPR;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  const unsigned char* qrow =
      static_cast<const unsigned char*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * RB + c * 16;
  float2 qf[G][CH2];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + g * RB));
    float2 f[CH2];
    Chunk<T>::unpack(raw, f);
#pragma unroll
    for (int e = 0; e < CH2; ++e) qf[g][e] = make_float2(f[e].x * p.qscale, f[e].y * p.qscale);
  }
  const unsigned char* Kb = static_cast<const unsigned char*>(p.K) + static_cast<size_t>(bh) * p.Ncap * RB + c * 16;
  constexpr int BATCH = RPW * R;
  for (int i = warp; i < nl; i += SEL_NW) {
    const int blk = lo + i;
    const int t0 = blk * p.L;
    const int cnt = min(p.L, n - t0);
    float M[HV::NH], S[HV::NH];
#pragma unroll
    for (int j = 0; j < HV::NH; ++j) {
      M[j] = -INFINITY;
      S[j] = 0.f;
    }
    for (int rb = 0; rb < cnt; rb += BATCH) {
      float part[NV];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int row = rb + r * RPW + rg;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (row < cnt) raw = __ldcs(reinterpret_cast<const uint4*>(Kb + static_cast<size_t>(t0 + row) * RB));
        float2 kf[CH2];
        Chunk<T>::unpack(raw, kf);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (g < G) {
            float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < CH2; ++e) a2 = ffma2(qf[g][e], kf[e], a2);
            part[r * GP + g] = a2.x + a2.y;
          } else {
            part[r * GP + g] = 0.f;
          }
        }
      }
      transpose_reduce<NV, LPR / 2>(part, lane);
#pragma unroll
      for (int j = 0; j < HV::NH; ++j) {
        const int vi = HV::index(c, j);
        const int ri = vi / GP;
        const int row = rb + ri * RPW + rg;
        const float s = row < cnt ? part[j] : -INFINITY;
        // reduce over every lane bit that changes the row: the row bits inside a
        // row group and the row-group bits above them
        float cm = s;
#pragma unroll
        for (int mask = HV::ROW_MASK_LO; mask < 32; mask <<= 1) cm = fmaxf(cm, __shfl_xor_sync(FULL_MASK, cm, mask));
        const float Mn = fmaxf(M[j], cm);  // finite: row rb of the batch is valid
        float e = exp2f(s - Mn);
#pragma unroll
        for (int mask = HV::ROW_MASK_LO; mask < 32; mask <<= 1) e += __shfl_xor_sync(FULL_MASK, e, mask);
        S[j] = S[j] * exp2f(M[j] - Mn) + e;
        M[j] = Mn;
      }
    }
#pragma unroll
    for (int j = 0; j < HV::NH; ++j) {
      const int g = HV::index(c, j) % GP;
      if (g < G) sh.lg[g][i] = cnt > 0 ? M[j] + log2f(S[j]) : -INFINITY;
    }
  }
}

template <typename T, int D, int G, int MODE>
__global__ void __cluster_dims__(SEL_CS, 1, 1) __launch_bounds__(SEL_THREADS)
    select_kernel(const SelParams p) {
  __shared__ SelShared<G> sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / SEL_CS;
  const int b = bh / p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = max(0, min(p.seq_lens[b], p.Ncap));
  const int nbv = (n + p.L - 1) / p.L;
  const int per = (nbv + SEL_CS - 1) / SEL_CS;
  const int lo = min(nbv, rank * per);
  const int nl = min(nbv, lo + per) - lo;

  if (MODE == SEL_SUMMARY)
    score_summary<T, D, G>(p, sh, bh, lo, nl);
  else
    score_exact<T, D, G>(p, sh, bh, lo, nl, n);
  __syncthreads();

  // per-head (max, sum of 2^(s - max)) over this slice
  if (warp < G) {
    float M = -INFINITY;
    for (int i = lane; i < nl; i += 32) M = fmaxf(M, sh.lg[warp][i]);
    M = warp_max(M);
    float S = 0.f;
    if (M != -INFINITY)
      for (int i = lane; i < nl; i += 32) S += exp2f(sh.lg[warp][i] - M);
    S = warp_sum(S);
    if (lane == 0) sh.part[warp] = make_float2(M, S);
  }
  cluster.sync();
  if (tid < G) {
    float M = -INFINITY;
    for (int r = 0; r < SEL_CS; ++r) M = fmaxf(M, cluster.map_shared_rank(&sh.part[tid], r)->x);
    float S = 0.f;
    if (M != -INFINITY)
      for (int r = 0; r < SEL_CS; ++r) {
        const float2 pr = *cluster.map_shared_rank(&sh.part[tid], r);
        S += pr.y * exp2f(pr.x - M);
      }
    sh.lse[tid] = (M == -INFINITY || S <= 0.f) ? -INFINITY : M + log2f(S);
  }
  __syncthreads();

  // group score (Equation 5) and ranking keys
  for (int i = tid; i < nl; i += SEL_THREADS) {
    float Sg = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (sh.lse[g] != -INFINITY) Sg += exp2f(sh.lg[g][i] - sh.lse[g]);
    const int blk = lo + i;
    if (p.scores) p.scores[static_cast<size_t>(bh) * p.NBcap + blk] = Sg;
    const bool forced = (p.force_first && blk == 0) || (p.force_last && blk == nbv - 1);
    sh.key[i] = forced ? 0ull
                       : ((static_cast<unsigned long long>(__float_as_uint(Sg)) << 32) |
                          static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(blk)));
    sh.flag[i] = forced ? 1 : 0;
  }
  if (p.scores) {
    // blocks past the sequence: score 0, split over the cluster
    const int tail = p.NBcap - nbv;
    const int tper = (tail + SEL_CS - 1) / SEL_CS;
    const int a0 = nbv + rank * tper, a1 = min(p.NBcap, a0 + tper);
    for (int blk = a0 + tid; blk < a1; blk += SEL_THREADS) p.scores[static_cast<size_t>(bh) * p.NBcap + blk] = 0.f;
  }
  __syncthreads();

  // local ranks; the best min(k, candidates) go to cand[] in descending order
  int mine = 0;
  for (int i = tid; i < nl; i += SEL_THREADS) {
    const unsigned long long x = sh.key[i];
    if (x == 0ull) continue;
    ++mine;
    int r = 0;
    for (int j = 0; j < nl; ++j) r += sh.key[j] > x;
    if (r < p.k_top) sh.cand[r] = x;
  }
  mine = block_sum(mine, sh.wsum);
  if (tid == 0) sh.ncand = min(mine, p.k_top);
  cluster.sync();

  // global rank = local rank + candidates of other CTAs that beat it
  for (int r = tid; r < sh.ncand; r += SEL_THREADS) {
    const unsigned long long x = sh.cand[r];
    int grank = r;
    for (int q = 0; q < SEL_CS; ++q) {
      if (q == rank) continue;
      const SelShared<G>* other = cluster.map_shared_rank(&sh, q);
      grank += count_greater(other->cand, other->ncand, x);
    }
    if (grank < p.k_top) {
      const int blk = static_cast<int>(0xffffffffu - static_cast<uint32_t>(x & 0xffffffffull));
      sh.flag[blk - lo] = 1;
    }
  }
  __syncthreads();
  int nflag = 0;
  for (int i = tid; i < nl; i += SEL_THREADS) nflag += sh.flag[i];
  nflag = block_sum(nflag, sh.wsum);
  if (tid == 0) sh.nsel = nflag;
  cluster.sync();
  int offset = 0, total = 0;
  for (int q = 0; q < SEL_CS; ++q) {
    const int v = cluster.map_shared_rank(&sh, q)->nsel;
    if (q < rank) offset += v;
    total += v;
  }
  for (int i = tid; i < nl; i += SEL_THREADS) {
    if (!sh.flag[i]) continue;
    int pos = offset;
    for (int j = 0; j < i; ++j) pos += sh.flag[j];
    if (pos < p.kmax) p.block_idx[static_cast<size_t>(bh) * p.kmax + pos] = lo + i;
  }
  if (rank == 0 && tid == 0) p.n_kept[bh] = min(total, p.kmax);
  cluster.sync();
}

}  // namespace kvs
