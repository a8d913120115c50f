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
// The key dot products are warp-cooperative: every lane holds D/32 of the pivot's
// key, a warp loads one whole row per instruction (coalesced) for 32 rows, and a
// transpose reduction leaves row r's dot product in lane r, which owns token r for
// the coalesced factor, d and output traffic. The factor lives in the workspace as
// F[t][i] (token index fastest). With the pivots' rows F_S (lower triangular in
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

// A lane's slice of a key row (D/32 elements) as loaded, and its fp32 values.
template <typename T, int E>
struct WcRaw;
template <>
struct WcRaw<__nv_bfloat16, 2> {
  using type = unsigned int;
  __device__ __forceinline__ static void unpack(type r, float (&x)[2]) {
    x[0] = __uint_as_float(r << 16);
    x[1] = __uint_as_float(r & 0xffff0000u);
  }
};
template <>
struct WcRaw<__nv_bfloat16, 4> {
  using type = uint2;
  __device__ __forceinline__ static void unpack(type r, float (&x)[4]) {
    x[0] = __uint_as_float(r.x << 16);
    x[1] = __uint_as_float(r.x & 0xffff0000u);
    x[2] = __uint_as_float(r.y << 16);
    x[3] = __uint_as_float(r.y & 0xffff0000u);
  }
};
template <>
struct WcRaw<float, 2> {
  using type = float2;
  __device__ __forceinline__ static void unpack(type r, float (&x)[2]) {
    x[0] = r.x;
    x[1] = r.y;
  }
};
template <>
struct WcRaw<float, 4> {
  using type = float4;
  __device__ __forceinline__ static void unpack(type r, float (&x)[4]) {
    x[0] = r.x;
    x[1] = r.y;
    x[2] = r.z;
    x[3] = r.w;
  }
};

template <typename T, int D>
struct WcRow {
  static constexpr int E = D / 32;
  using R = WcRaw<T, E>;
  using raw = typename R::type;
  // rows whose slices are loaded before any is used (64 registers of loads)
  static constexpr int RB = sizeof(raw) >= 16 ? 16 : 32;
  __device__ __forceinline__ static raw load(const T* row, int lane) {
    return __ldcs(reinterpret_cast<const raw*>(row) + lane);  // keys stream: evict first
  }
};

// Dot products of the 32 key rows i0 .. i0+31 with the lane-split vector ks
// (SELF: each row with itself); lane j returns row i0+j's. Rows at or past n
// read row n-1 (in bounds) and their results are ignored by the caller.
template <typename T, int D, bool SELF>
__device__ __forceinline__ float wc_dots(const T* Kb, int i0, int n, const float (&ks)[D / 32], int lane) {
  using W = WcRow<T, D>;
  constexpr int E = W::E, RB = W::RB;
  float v[32];
#pragma unroll
  for (int r0 = 0; r0 < 32; r0 += RB) {
    typename W::raw raw[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) raw[r] = W::load(Kb + static_cast<size_t>(min(i0 + r0 + r, n - 1)) * D, lane);
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      float x[E];
      W::R::unpack(raw[r], x);
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) a = fmaf(x[e], SELF ? x[e] : ks[e], a);
      v[r0 + r] = a;
    }
  }
  transpose_reduce<32, 16>(v, lane);
  return v[0];
}

// Residual kernel column at token i0 + lane: exp(scale k_i.k_s - sM) minus the
// factor rows so far times fs (fs[j] = F[j][s]). The factor is read through L2
// (it is written by every CTA of the cluster).
template <typename T, int D>
__device__ __forceinline__ float wc_column(const T* Kb, int i0, int n, const float (&ks)[D / 32], const float* F,
                                           int Ncap, const float* fs, int t, float scale, float sM, int lane) {
  const float dot = wc_dots<T, D, false>(Kb, i0, n, ks, lane);
  float g = __expf(scale * dot - sM);
  const int i = i0 + lane;
  if (i < n) {
    // 32 factor rows per batch, all loads issued before the first use (one
    // round trip per 32 rows); rows past t load nothing and add nothing
    const float* Fi = F + i;
    for (int j0 = 0; j0 < t; j0 += 32) {
      float f[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) f[k] = j0 + k < t ? __ldcg(Fi + static_cast<size_t>(j0 + k) * Ncap) : 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k)
        if (j0 + k < t) g = fmaf(-f[k], fs[j0 + k], g);
    }
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

struct WcShared {
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
  constexpr int E = D / 32;
  __shared__ WcShared sh;
  extern __shared__ float gsum[];  // this CTA's group sums of d
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.x / C, b = bh / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = max(0, min(seq_lens[b], Ncap));
  const T* Kb = K + static_cast<size_t>(bh) * Ncap * D;
  const size_t stride = (static_cast<size_t>(m) + 1) * Ncap + static_cast<size_t>(WC_MAX_C) * m;
  float* F = ws + static_cast<size_t>(bh) * stride;  // F[t][i], t < m
  float* d = F + static_cast<size_t>(m) * Ncap;      // residual diagonal
  float* cs = d + Ncap;                              // column sums [C][m]
  const float* ub = u + static_cast<size_t>(bh) * m;
  const int ngrp = (n + 31) / 32;
  const int g_beg = static_cast<int>(static_cast<long long>(ngrp) * rank / C);
  const int g_end = static_cast<int>(static_cast<long long>(ngrp) * (rank + 1) / C);
  const int ng = g_end - g_beg;
  const float no_vec[E] = {};

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
    float ks[E];
    WcRow<T, D>::R::unpack(WcRow<T, D>::load(Kb + static_cast<size_t>(s) * D, lane), ks);
    for (int j = tid; j < t; j += WC_THREADS) sh.fs[j] = __ldcg(F + static_cast<size_t>(j) * Ncap + s);
    if (tid == 0) sh.piv_list[t] = s;
    __syncthreads();
    if (warp == 0) {
      // the same computation as the pivot's lane in the column pass, so bit-identical
      const float g = wc_column<T, D>(Kb, s & ~31, n, ks, F, Ncap, sh.fs, t, scale, sM, lane);
      const float gs = __shfl_sync(FULL_MASK, g, s & 31);
      if (lane == 0) sh.gpiv = gs;
    }
    __syncthreads();
    const float gp = sh.gpiv;
    if (!(gp > 0.f)) break;  // uniform: no residual left at the pivot
    const float inv = rsqrtf(gp);

    // ---- 3. the fused pass: factor column t, the downdate of d, group sums, column sum
    float csum = 0.f;
    float* Ft = F + static_cast<size_t>(t) * Ncap;
    for (int g = g_beg + warp; g < g_end; g += WC_NW) {
      const int i = g * 32 + lane;
      const float di = i < n ? d[i] : 0.f;  // issued ahead of the column's loads
      const float gi = wc_column<T, D>(Kb, g * 32, n, ks, F, Ncap, sh.fs, t, scale, sM, lane);
      float dn = 0.f;
      if (i < n) {
        const float f = gi * inv;
        Ft[i] = f;
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
      const float* Fc = F + static_cast<size_t>(c) * Ncap;
      float acc = 0.f;
      for (int r = c + 1 + lane; r < taken; r += 32) acc = fmaf(__ldcg(Fc + sh.piv_list[r]), sh.fs[r], acc);
      acc = warp_sum(acc);
      if (lane == 0) sh.fs[c] = (sh.fs[c] - acc) / __ldcg(Fc + sh.piv_list[c]);
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
  const size_t per_pair = (static_cast<size_t>(m) + 1) * shape->Ncap + static_cast<size_t>(kvs::WC_MAX_C) * m;
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
