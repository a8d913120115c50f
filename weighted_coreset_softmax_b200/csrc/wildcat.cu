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
// Work split: a cluster of C CTAs per pair (C = SMs / pairs, at most 8), CTA c
// owning a contiguous range of 32-token groups. Pivot step t:
//   1. draw: every CTA sums its groups' residual diagonal d (kept per group in
//      shared memory by the previous pass); the C totals are exchanged through
//      distributed shared memory and every CTA adds them in the same order, so all
//      agree on the total and on the CTA whose range holds u_t * total. That CTA
//      walks its group sums, then one warp scans the group's 32 entries, and
//      writes the pivot s into every CTA's shared memory.
//   2. every CTA computes the residual at the pivot, g_s, itself with the same code
//      as the column pass (bit-identical everywhere, so nothing else is exchanged).
//   3. one fused pass over the CTA's tokens: the residual kernel column
//      g_i = exp(scale k_i.k_s - shift) - sum_{j<t} F[j][i] F[j][s], the factor
//      column F[t][i] = g_i / sqrt(g_s), d_i -= F[t][i]^2 (0 at the pivot), the new
//      group sums of d for the next draw, and the column's sum.
// The key dot products are warp-cooperative: 8 lanes share a row, each holding 1/8 of
// the pivot's key in 16-byte chunks, a warp load covers 4 rows, and a transpose
// reduction over the 8 lanes leaves row r's dot product in lane r, which owns token r
// for the coalesced factor, d and output traffic. The factor lives in the workspace
// as F[t][i] in tiles of 32 tokens (each batch's factor rows contiguous). With the
// pivots' rows F_S (lower triangular in
// pivot order), A_SS = F_S F_S^T and A_{S,:} = F_S F^T exactly, so
// w = F_S^-T (F^T 1): CTA 0 adds the C partial column sums in rank order and runs
// one back substitution. Bytes per pair and step: the n keys, t factor rows read
// and one written; the build runs once after prefill.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "kvsparse.h"

namespace cg = cooperative_groups;

namespace kvs {
void set_last_error(const char* msg);

constexpr int WC_THREADS = 512;
constexpr int WC_NW = WC_THREADS / 32;
constexpr int WC_MAX_M = 4096;
constexpr int WC_MAX_C = 8;
constexpr int WC_MAX_NCAP = 1 << 20;

// The factor matrix is stored in tiles of 32 tokens: F[j][i] at
// (i / 32) * 32 m + 32 j + i % 32, so that the t factor rows a warp reads for one
// batch of 32 tokens are one contiguous t * 128-byte run and the factor column it
// writes is one 128-byte piece.
__device__ __forceinline__ size_t wc_fidx(int j, int i, int m) {
  return static_cast<size_t>(i >> 5) * (32 * static_cast<size_t>(m)) + 32 * j + (i & 31);
}

// Lane layout of the key-row dot products: 8 lanes a row, lane c (= lane % 8) of a
// group holding the 16-byte chunks c, c + 8, ... of the row (so a warp load reads 4
// rows as 4 contiguous 128-byte pieces); group gq (= lane / 8) takes the rows
// i0 + 8 gq + k, k < 8, so that an 8-value transpose reduction over the group leaves
// row i0 + lane's dot product in lane `lane`.
template <typename T, int D>
struct WcLay {
  static constexpr int CHE = 16 / static_cast<int>(sizeof(T));  // elements a chunk
  static constexpr int CPL = D / CHE / 8;                        // chunks a lane (1, 2 or 4)
  static constexpr int EPL = CPL * CHE;                          // elements a lane (8 or 16)
  static constexpr int RBK = CPL * 4 * 8 > 64 ? 4 : 8;          // rows loaded at once (64 registers)
  static constexpr bool R64 = CPL == 2 && CHE == 8;              // factor rounds of 64 rows fit (16-bit, D = 128)
};

// This lane's elements of one row (the pivot's key), as fp32 pairs.
template <typename T, int D>
__device__ __forceinline__ void wc_slice2(const T* row, int lane, float2 (&x)[WcLay<T, D>::EPL / 2]) {
  using Ly = WcLay<T, D>;
  const int c = lane & 7;
#pragma unroll
  for (int kk = 0; kk < Ly::CPL; ++kk) {
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(row) + c + 8 * kk);
    float2 f[Ly::CHE / 2];
    Chunk<T>::unpack(r, f);
#pragma unroll
    for (int e = 0; e < Ly::CHE / 2; ++e) x[kk * (Ly::CHE / 2) + e] = f[e];
  }
}

// Dot products of the 32 key rows i0 .. i0+31 with the lane-split vector ks (SELF:
// each row with itself); lane j returns row i0+j's. Rows at or past n read row n-1
// (in bounds) and their results are ignored by the caller.
template <typename T, int D, bool SELF>
__device__ __forceinline__ float wc_dots(const T* Kb, int i0, int n, const float2 (&ks)[WcLay<T, D>::EPL / 2],
                                         int lane) {
  using Ly = WcLay<T, D>;
  const int gq = lane >> 3, c = lane & 7;
  float v[8];
#pragma unroll
  for (int k0 = 0; k0 < 8; k0 += Ly::RBK) {
    uint4 raw[Ly::RBK][Ly::CPL];
#pragma unroll
    for (int k = 0; k < Ly::RBK; ++k) {
      const int row = min(i0 + 8 * gq + k0 + k, n - 1);
#pragma unroll
      for (int kk = 0; kk < Ly::CPL; ++kk)
        raw[k][kk] = __ldcs(reinterpret_cast<const uint4*>(Kb + static_cast<size_t>(row) * D) + c + 8 * kk);
    }
#pragma unroll
    for (int k = 0; k < Ly::RBK; ++k) {
      float2 a = make_float2(0.f, 0.f);
#pragma unroll
      for (int kk = 0; kk < Ly::CPL; ++kk) {
        float2 f[Ly::CHE / 2];
        Chunk<T>::unpack(raw[k][kk], f);
#pragma unroll
        for (int e = 0; e < Ly::CHE / 2; ++e) a = ffma2(f[e], SELF ? f[e] : ks[kk * (Ly::CHE / 2) + e], a);
      }
      v[k0 + k] = a.x + a.y;
    }
  }
  transpose_reduce<8, 4>(v, lane);
  return v[0];
}

// Residual kernel column at token i0 + lane: exp(scale k_i.k_s - sM) minus the
// factor rows so far times fs (fs[j] = F[j][s]). The factor is read through L2
// (it is written by every CTA of the cluster).
template <typename T, int D>
__device__ __forceinline__ float wc_column(const T* Kb, int i0, int n, const float2 (&ks)[WcLay<T, D>::EPL / 2],
                                           const float* F, int m, const float* fs, int t, float scale, float sM,
                                           int lane) {
  // the first FP factor rows are requested before the key rows, so that both
  // round trips overlap (none where the key rows already take 64 registers at 4
  // rows a batch). The rest go in unpredicated rounds of 64 rows (16-bit keys,
  // D = 128) or 32 (the key rows' registers are free by then), all loads of a round
  // issued before the first use, and a predicated tail of fewer than 32 rows (rows
  // past t load nothing and add nothing). The sum runs in row order whatever the
  // rounds.
  constexpr int FP = WcLay<T, D>::RBK == 4 ? 0 : 16;
  const int i = i0 + lane;
  const float* Fi = F + wc_fidx(0, min(i, n - 1), m);
  float f0[FP > 0 ? FP : 1];
#pragma unroll
  for (int k = 0; k < FP; ++k) f0[k] = k < t ? __ldcg(Fi + 32 * k) : 0.f;
  const float dot = wc_dots<T, D, false>(Kb, i0, n, ks, lane);
  float g = __expf(scale * dot - sM);
#pragma unroll
  for (int k = 0; k < FP; ++k)
    if (k < t) g = fmaf(-f0[k], fs[k], g);
  int j = FP;  // a multiple of 4: fs + j is 16-byte aligned
  for (; WcLay<T, D>::R64 && j + 64 <= t; j += 64) {
    const float* Fj = Fi + 32 * j;
    float f[64];
#pragma unroll
    for (int k = 0; k < 64; ++k) f[k] = __ldcg(Fj + 32 * k);
#pragma unroll
    for (int k = 0; k < 64; k += 4) {
      const float4 c = *reinterpret_cast<const float4*>(fs + j + k);
      g = fmaf(-f[k], c.x, g);
      g = fmaf(-f[k + 1], c.y, g);
      g = fmaf(-f[k + 2], c.z, g);
      g = fmaf(-f[k + 3], c.w, g);
    }
  }
  for (; j + 32 <= t; j += 32) {
    const float* Fj = Fi + 32 * j;
    float f[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) f[k] = __ldcg(Fj + 32 * k);
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
      const float4 c = *reinterpret_cast<const float4*>(fs + j + k);
      g = fmaf(-f[k], c.x, g);
      g = fmaf(-f[k + 1], c.y, g);
      g = fmaf(-f[k + 2], c.z, g);
      g = fmaf(-f[k + 3], c.w, g);
    }
  }
  if (j < t) {
    const float* Fj = Fi + 32 * j;
    float f[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) f[k] = j + k < t ? __ldcg(Fj + 32 * k) : 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k)
      if (j + k < t) g = fmaf(-f[k], fs[j + k], g);
  }
  return g;
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

struct alignas(16) WcShared {
  float fs[WC_MAX_M];     // F[j][s] of the current pivot, j < t; at the end the weights
  int piv_list[WC_MAX_M];  // the pivots in the order drawn
  float wsum[WC_NW];
  float ctot[WC_MAX_C];  // the cluster's per-CTA totals of d (written by every CTA)
  float cmax[WC_MAX_C];  // the cluster's per-CTA max |k|^2
  int piv;               // the pivot (written by the CTA that draws it)
  int pg, pg_fb;
  float base, gpiv;
};

template <typename T, int D>
__global__ void __launch_bounds__(WC_THREADS, 1)
    wildcat_kernel(const T* __restrict__ K, const int32_t* seq_lens, int Hkv, int Ncap, int m, float scale,
                   const float* __restrict__ u, int32_t* tok_idx, float* w, int32_t* n_sel, float* ws) {
  constexpr int E2 = WcLay<T, D>::EPL / 2;
  __shared__ WcShared sh;
  extern __shared__ float gsum[];  // this CTA's group sums of d
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / C, b = bh / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = max(0, min(seq_lens[b], Ncap));
  const T* Kb = K + static_cast<size_t>(bh) * Ncap * D;
  const size_t n32 = static_cast<size_t>((Ncap + 31) & ~31);
  const size_t stride = (static_cast<size_t>(m) + 1) * n32 + static_cast<size_t>(WC_MAX_C) * m;
  float* F = ws + static_cast<size_t>(bh) * stride;  // F[t][i], t < m, tiled by wc_fidx
  float* d = F + static_cast<size_t>(m) * n32;       // residual diagonal
  float* cs = d + n32;                               // column sums [C][m]
  const float* ub = u + static_cast<size_t>(bh) * m;
  const int ngrp = (n + 31) / 32;
  const int g_beg = static_cast<int>(static_cast<long long>(ngrp) * rank / C);
  const int g_end = static_cast<int>(static_cast<long long>(ngrp) * (rank + 1) / C);
  const int ng = g_end - g_beg;
  const float2 no_vec[E2] = {};

  // ---- the shift M = max_i |k_i|^2 over the pair; d_i = exp(scale |k_i|^2 - scale M)
  float mx = 0.f;
  for (int g = g_beg + warp; g < g_end; g += WC_NW) {
    const float sq = wc_dots<T, D, true>(Kb, g * 32, n, no_vec, lane);
    const int i = g * 32 + lane;
    if (i < n) {
      d[i] = sq;
      mx = fmaxf(mx, sq);
    }
  }
  mx = warp_max(mx);
  if (lane == 0) sh.wsum[warp] = mx;
  __syncthreads();
  if (tid < C) {
    float cm = 0.f;
    for (int q = 0; q < WC_NW; ++q) cm = fmaxf(cm, sh.wsum[q]);
    cluster.map_shared_rank(sh.cmax, tid)[rank] = cm;
  }
  cluster.sync();
  float M = 0.f;
  for (int c = 0; c < C; ++c) M = fmaxf(M, sh.cmax[c]);
  const float sM = scale * M;
  for (int g = g_beg + warp; g < g_end; g += WC_NW) {
    const int i = g * 32 + lane;
    float x = 0.f;
    if (i < n) {
      x = __expf(scale * d[i] - sM);
      d[i] = x;
    }
    x = warp_sum(x);
    if (lane == 0) gsum[g - g_beg] = x;
  }
  __syncthreads();

  const int per = (ng + WC_THREADS - 1) / WC_THREADS;  // contiguous groups per thread in the draw
  const int r_lo = min(ng, tid * per), r_hi = min(ng, r_lo + per);
  int taken = 0;
  for (int t = 0; t < m; ++t) {
    // ---- 1. the draw: the first token whose running sum of d reaches u_t * total
    float part = 0.f;
    for (int r = r_lo; r < r_hi; ++r) part += gsum[r];
    float ctot;
    const float incl = wc_scan(part, sh.wsum, &ctot);
    if (tid < C) cluster.map_shared_rank(sh.ctot, tid)[rank] = ctot;
    cluster.sync();
    float total = 0.f;
    for (int c = 0; c < C; ++c) total += sh.ctot[c];
    if (!(total > 0.f)) break;  // uniform: the residual is zero (or n = 0)
    const float target = ub[t] * total;
    int owner = -1, owner_fb = -1;
    float owner_pre = 0.f, fb_pre = 0.f;
    {
      float acc = 0.f;
      for (int c = 0; c < C; ++c) {
        const float x = sh.ctot[c];
        if (x > 0.f) {
          owner_fb = c;
          fb_pre = acc;
        }
        const float before = acc;
        acc += x;
        if (owner < 0 && x > 0.f && acc >= target) {
          owner = c;
          owner_pre = before;
        }
      }
    }
    if (owner < 0) {  // rounding kept every running sum short: the last CTA holding residual
      owner = owner_fb;
      owner_pre = fb_pre;
    }
    if (owner < 0) break;  // uniform (no positive total)
    if (rank == owner) {
      if (tid == 0) {
        sh.pg = INT_MAX;
        sh.pg_fb = -1;
      }
      __syncthreads();
      const float pre = owner_pre + (incl - part);
      {
        // the smallest group whose running sum reaches the target; the minimum
        // over threads keeps the choice deterministic where rounding lets two reach it
        float acc = pre;
        int last_pos = -1;
        for (int r = r_lo; r < r_hi; ++r) {
          const float x = gsum[r];
          if (x > 0.f) last_pos = r;
          acc += x;
          if (x > 0.f && acc >= target) {
            atomicMin(&sh.pg, r);
            break;
          }
        }
        if (last_pos >= 0) atomicMax(&sh.pg_fb, last_pos);
      }
      __syncthreads();
      if (tid == 0 && sh.pg == INT_MAX) sh.pg = sh.pg_fb;  // else the last group holding residual
      __syncthreads();
      const int gsel = sh.pg;
      if (gsel >= r_lo && gsel < r_hi) {
        float acc = pre;
        for (int r = r_lo; r < gsel; ++r) acc += gsum[r];
        sh.base = acc;
      }
      __syncthreads();
      if (warp == 0) {
        int pick = -1;
        if (gsel >= 0) {
          const int i = (g_beg + gsel) * 32 + lane;
          const float x = i < n ? d[i] : 0.f;
          float sc = x;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(FULL_MASK, sc, o);
            if (lane >= o) sc += y;
          }
          const unsigned hit = __ballot_sync(FULL_MASK, x > 0.f && sh.base + sc >= target);
          const unsigned pos = __ballot_sync(FULL_MASK, x > 0.f);
          if (pos) pick = (g_beg + gsel) * 32 + (hit ? __ffs(hit) - 1 : 31 - __clz(pos));
        }
        if (lane < C) *cluster.map_shared_rank(&sh.piv, lane) = pick;
      }
    }
    cluster.sync();
    const int s = sh.piv;
    if (s < 0 || s >= n) break;  // (no positive entry in the drawn group: not reached for finite keys)

    // ---- 2. the pivot's key slice, its factor row, and the residual at the pivot
    float2 ks[E2];
    wc_slice2<T, D>(Kb + static_cast<size_t>(s) * D, lane, ks);
    for (int j = tid; j < t; j += WC_THREADS) sh.fs[j] = __ldcg(F + wc_fidx(j, s, m));
    if (tid == 0) sh.piv_list[t] = s;
    __syncthreads();
    if (warp == 0) {
      // the same computation as the pivot's lane in the column pass, so bit-identical
      const float g = wc_column<T, D>(Kb, s & ~31, n, ks, F, m, sh.fs, t, scale, sM, lane);
      const float gs = __shfl_sync(FULL_MASK, g, s & 31);
      if (lane == 0) sh.gpiv = gs;
    }
    __syncthreads();
    const float gp = sh.gpiv;
    if (!(gp > 0.f)) break;  // uniform: no residual left at the pivot
    const float inv = rsqrtf(gp);

    // ---- 3. the fused pass: factor column t, the downdate of d, group sums, column sum
    float csum = 0.f;
    for (int g = g_beg + warp; g < g_end; g += WC_NW) {
      const int i = g * 32 + lane;
      const float di = i < n ? d[i] : 0.f;  // issued ahead of the column's loads
      const float gi = wc_column<T, D>(Kb, g * 32, n, ks, F, m, sh.fs, t, scale, sM, lane);
      float dn = 0.f;
      if (i < n) {
        const float f = gi * inv;
        F[wc_fidx(t, i, m)] = f;
        dn = i == s ? 0.f : fmaxf(di - f * f, 0.f);
        d[i] = dn;
        csum += f;
      }
      dn = warp_sum(dn);
      if (lane == 0) gsum[g - g_beg] = dn;
    }
    csum = wc_sum(csum, sh.wsum);
    if (tid == 0) cs[static_cast<size_t>(rank) * m + t] = csum;
    taken = t + 1;
    __syncthreads();
  }
  cluster.sync();  // every CTA's factor columns and column sums are written
  if (rank != 0) return;

  // ---- weights: F_S^T w = F^T 1 (F_S[r][c] = F[c][S_r], lower triangular), the
  // right-hand side the rank-ordered sum of the CTAs' column sums; one back
  // substitution by warp 0
  int32_t* idx_out = tok_idx + static_cast<size_t>(bh) * m;
  float* w_out = w + static_cast<size_t>(bh) * m;
  for (int r = tid; r < taken; r += WC_THREADS) {
    float acc = 0.f;
    for (int c = 0; c < C; ++c) acc += __ldcg(cs + static_cast<size_t>(c) * m + r);
    sh.fs[r] = acc;
  }
  __syncthreads();
  if (warp == 0) {
    for (int c = taken - 1; c >= 0; --c) {
      // w_c = (rhs_c - sum_{r > c} F_S[r][c] w_r) / F_S[c][c]
      float acc = 0.f;
      for (int r = c + 1 + lane; r < taken; r += 32) acc = fmaf(__ldcg(F + wc_fidx(c, sh.piv_list[r], m)), sh.fs[r], acc);
      acc = warp_sum(acc);
      if (lane == 0) sh.fs[c] = (sh.fs[c] - acc) / __ldcg(F + wc_fidx(c, sh.piv_list[c], m));
      __syncwarp();
    }
  }
  __syncthreads();
  for (int r = tid; r < m; r += WC_THREADS) {
    if (r < taken) {
      idx_out[r] = sh.piv_list[r];
      w_out[r] = fmaxf(sh.fs[r], 0.f);
    } else {
      idx_out[r] = 0;
      w_out[r] = 0.f;
    }
  }
  if (tid == 0 && n_sel) n_sel[bh] = taken;
}

template <typename T, int D>
static cudaError_t wildcat_launch(const kv_shape* s, const void* K, float scale, int m, int C, const float* u,
                                  int32_t* tok_idx, float* w, int32_t* n_sel, float* ws, cudaStream_t st) {
  auto kern = wildcat_kernel<T, D>;
  const int groups = (s->Ncap + 31) / 32;
  const size_t smem = static_cast<size_t>((groups + C - 1) / C) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(s->B * s->Hkv * C));
  cfg.blockDim = dim3(WC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(C);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(K), s->seq_lens, s->Hkv, s->Ncap, m, scale, u, tok_idx,
                            w, n_sel, ws);
}
}  // namespace kvs

extern "C" size_t kv_wildcat_workspace_bytes(const kv_shape* shape, int m) {
  if (!shape || m < 1 || shape->B < 0 || shape->Hkv < 1 || shape->Ncap < 1) return 0;
  const size_t n32 = static_cast<size_t>((shape->Ncap + 31) & ~31);
  const size_t per_pair = (static_cast<size_t>(m) + 1) * n32 + static_cast<size_t>(kvs::WC_MAX_C) * m;
  return static_cast<size_t>(shape->B) * shape->Hkv * per_pair * sizeof(float);
}

extern "C" kv_status kv_build_wildcat_coreset(const kv_shape* shape, const void* K, float scale, int m,
                                              int ctas_per_pair, const float* u, int32_t* tok_idx, float* w,
                                              int32_t* n_sel, void* workspace, size_t ws_bytes, kv_stream_t stream) {
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
  if (shape->Ncap > kvs::WC_MAX_NCAP) {
    kvs::set_last_error("kv_build_wildcat_coreset: Ncap above 2^20");
    return KV_ERR_UNSUPPORTED;
  }
  if (shape->dtype != KV_BF16 && shape->dtype != KV_F32) return bad("kv_build_wildcat_coreset: unknown dtype");
  if (m < 1 || m > kvs::WC_MAX_M || m > shape->Ncap) return bad("kv_build_wildcat_coreset: m outside 1..min(4096, Ncap)");
  if (ctas_per_pair < 0 || ctas_per_pair > kvs::WC_MAX_C)
    return bad("kv_build_wildcat_coreset: ctas_per_pair outside 0..8");
  if (!std::isfinite(scale) || scale <= 0.f) return bad("kv_build_wildcat_coreset: scale must be finite and > 0");
  auto al = [](const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (shape->B > 0 && !al(shape->seq_lens, 4)) return bad("kv_build_wildcat_coreset: seq_lens NULL or misaligned");
  if (!al(K, 16)) return bad("kv_build_wildcat_coreset: K NULL or not 16-byte aligned");
  if (!al(u, 4) || !al(tok_idx, 4) || !al(w, 4)) return bad("kv_build_wildcat_coreset: u, tok_idx, w NULL or misaligned");
  if (n_sel && !al(n_sel, 4)) return bad("kv_build_wildcat_coreset: n_sel misaligned");
  if (!al(workspace, 16)) return bad("kv_build_wildcat_coreset: workspace NULL or not 16-byte aligned");
  if (ws_bytes < kv_wildcat_workspace_bytes(shape, m)) return bad("kv_build_wildcat_coreset: workspace too small");
  const long long pairs = static_cast<long long>(shape->B) * shape->Hkv;
  if (pairs == 0) return KV_OK;
  int C = ctas_per_pair;
  if (C == 0) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();
      kvs::set_last_error("kv_build_wildcat_coreset: no current CUDA device");
      return KV_ERR_CUDA;
    }
    C = static_cast<int>(std::max(1LL, std::min<long long>(kvs::WC_MAX_C, sms / pairs)));
  }
  if (pairs * C > INT_MAX) return bad("kv_build_wildcat_coreset: too many (sequence, KV head) pairs");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  cudaError_t e;
  if (shape->dtype == KV_BF16)
    e = shape->D == 64 ? kvs::wildcat_launch<__nv_bfloat16, 64>(shape, K, scale, m, C, u, tok_idx, w, n_sel, ws, st)
                       : kvs::wildcat_launch<__nv_bfloat16, 128>(shape, K, scale, m, C, u, tok_idx, w, n_sel, ws, st);
  else
    e = shape->D == 64 ? kvs::wildcat_launch<float, 64>(shape, K, scale, m, C, u, tok_idx, w, n_sel, ws, st)
                       : kvs::wildcat_launch<float, 128>(shape, K, scale, m, C, u, tok_idx, w, n_sel, ws, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    kvs::set_last_error("kv_build_wildcat_coreset: launch failed");
    return KV_ERR_CUDA;
  }
  return KV_OK;
}
