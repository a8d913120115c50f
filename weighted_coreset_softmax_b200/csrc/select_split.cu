// Block selection for few (sequence, KV head) pairs: each pair's blocks split over a
// thread-block cluster of S CTAs, so that a batch with fewer pairs than SMs still
// streams its block summaries with every SM. Same result as select_kernel in the
// summary and bf16-mean modes with k_top <= 16 (the per-warp top-k path), only the
// order of the normaliser's additions differs.
//
// CTA r of the cluster scores the blocks [r * seg, min(nbv, (r + 1) * seg)) with the
// scorer of select_kernel (score_summary, given row and count pointers shifted to the
// range), so its log2-domain logits are the one-CTA kernel's. The per-head (max, sum)
// partials of Equation 5's normaliser go to every CTA through distributed shared
// memory and each CTA adds them in rank order; each CTA then forms its blocks' group
// scores and ranking keys (score bits, inverted global index; forced blocks 0), writes
// its scores, and takes its k_top largest keys; rank 0 takes the k_top largest of the
// S * k_top candidates, adds the forced blocks and writes the kept list ascending.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <atomic>

#include "launch.h"
#include "select.cuh"

namespace cg = cooperative_groups;

namespace kvs {

constexpr int SPLIT_MAX_S = 8;

struct SplitMisc {
  float pmx[SPLIT_MAX_S][8], psm[SPLIT_MAX_S][8];          // per-CTA normaliser partials (written by every CTA)
  unsigned long long cand[SPLIT_MAX_S][SEL_TOPK];          // rank 0: every CTA's top keys
  int ncand[SPLIT_MAX_S];                                  // rank 0: every CTA's candidate count
  float lse[8];
};

template <typename T, int D, int G, int MODE>
__global__ void __launch_bounds__(SEL_THREADS, 2) select_split_kernel(const SelParams p, int segcap) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  __shared__ SplitMisc sp;
  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int nbp = sel_nbp(segcap);
  float* lg = reinterpret_cast<float*>(sel_smem);
  unsigned long long* key = reinterpret_cast<unsigned long long*>(sel_smem + static_cast<size_t>(G) * nbp * 4);
  SelMisc& ms = *reinterpret_cast<SelMisc*>(sel_smem + static_cast<size_t>(G) * nbp * 4 + static_cast<size_t>(nbp) * 8);
  const int bh = blockIdx.x / S;
  const int b = bh / p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dep_wait();
  grid_dep_launch();
  const int n = max(0, min(p.seq_lens[b], p.Ncap));
  const int nbv = (n + p.L - 1) / p.L;
  const int seg = (nbv + S - 1) / S;
  const int lo = min(nbv, rank * seg), hi = min(nbv, lo + seg);
  const int len = hi - lo;  // <= segcap

  // ---- the range's logits, by the one-CTA scorer on shifted rows
  if (tid == 0) {
#pragma unroll
    for (int w = 0; w < SEL_NW; ++w)
#pragma unroll
      for (int st = 0; st < SEL_STAGES; ++st) mbar_init(reinterpret_cast<uint64_t*>(&ms.rbar[w][st]), 1);
    fence_mbar_init();
  }
  if (warp < SEL_NW && lane < 8) {
    ms.pm[warp][lane] = -INFINITY;
    ms.ps[warp][lane] = 0.f;
  }
  __syncthreads();
  constexpr int ROWK = MODE == SEL_MEAN16 ? ROW_MEAN16 : ROW_SUM32;
  constexpr int RB = D * (ROWK == ROW_MEAN16 ? 2 : 4);
  if (len > 0) {
    SelParams ps = p;
    if constexpr (ROWK == ROW_MEAN16)
      ps.k_mean16 = static_cast<const unsigned char*>(p.k_mean16) + static_cast<size_t>(lo) * RB;
    else
      ps.k_sum = p.k_sum + static_cast<size_t>(lo) * D;
    ps.counts = p.counts + lo;
    int* cnt = reinterpret_cast<int*>(sel_smem + sel_smem_bytes(G, segcap));
    float4* ring = reinterpret_cast<float4*>(
        sel_smem + ((sel_smem_bytes(G, segcap) + static_cast<size_t>(nbp) * 4 + 15) & ~static_cast<size_t>(15)));
    score_summary<T, D, G, ROWK>(ps, lg, nbp, bh, len, ring, cnt, ms);
  }
  __syncthreads();

  // ---- Equation 5's normalisers: this CTA's (max, sum) per head to every CTA
  if (warp == 0 && lane < G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < SEL_NW; ++w) M = fmaxf(M, ms.pm[w][lane]);
    float Ssum = 0.f;
    if (M != -INFINITY)
#pragma unroll
      for (int w = 0; w < SEL_NW; ++w)
        if (ms.pm[w][lane] != -INFINITY) Ssum += ms.ps[w][lane] * exp2f(ms.pm[w][lane] - M);
    for (int r = 0; r < S; ++r) {
      SplitMisc* rem = cluster.map_shared_rank(&sp, r);
      rem->pmx[rank][lane] = M;
      rem->psm[rank][lane] = Ssum;
    }
  }
  cluster.sync();
  if (tid < G) {
    float M = -INFINITY;
    for (int r = 0; r < S; ++r) M = fmaxf(M, sp.pmx[r][tid]);
    float Ssum = 0.f;
    if (M != -INFINITY)
      for (int r = 0; r < S; ++r)
        if (sp.pmx[r][tid] != -INFINITY) Ssum += sp.psm[r][tid] * exp2f(sp.pmx[r][tid] - M);
    sp.lse[tid] = (M == -INFINITY || Ssum <= 0.f) ? -INFINITY : M + log2f(Ssum);
  }
  __syncthreads();

  // ---- group scores and keys of the range
  int ncand = 0;
  for (int i = tid; i < len; i += SEL_THREADS) {
    const int blk = lo + i;
    float Sg = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (sp.lse[g] != -INFINITY) Sg += exp2f(lg[g * nbp + i] - sp.lse[g]);
    if (p.scores) p.scores[static_cast<size_t>(bh) * p.NBcap + blk] = Sg;
    const bool forced = (p.force_first && blk == 0) || (p.force_last && blk == nbv - 1);
    key[i] = forced ? 0ull
                    : ((static_cast<unsigned long long>(__float_as_uint(Sg)) << 32) |
                       static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(blk)));
    ncand += !forced;
  }
  if (p.scores && rank == S - 1)
    for (int i = nbv + tid; i < p.NBcap; i += SEL_THREADS) p.scores[static_cast<size_t>(bh) * p.NBcap + i] = 0.f;
  ncand = sel_block_sum(ncand, ms.wsum);  // also orders the key writes

  // ---- this CTA's k_top largest keys (k rounds of "largest key below the previous
  // one": per warp over its share, then over the warps), to rank 0
  const int k = p.k_top;
  {
    const int per = (len + SEL_NW - 1) / SEL_NW;
    const int wlo = warp * per, whi = min(len, wlo + per);
    unsigned long long prev = ~0ull;
    for (int r = 0; r < k; ++r) {
      unsigned long long best = 0ull;
      for (int i = wlo + lane; i < whi; i += 32) {
        const unsigned long long x = key[i];
        if (x < prev && x > best) best = x;
      }
      best = warp_max_key(best);
      if (lane == 0) ms.wtop[warp * SEL_TOPK + r] = best;
      prev = best;
    }
    __syncthreads();
    if (warp == 0) {
      unsigned long long cand[SEL_NW];
#pragma unroll
      for (int w = 0; w < SEL_NW; ++w) cand[w] = lane < k ? ms.wtop[w * SEL_TOPK + lane] : 0ull;
      prev = ~0ull;
      SplitMisc* r0 = cluster.map_shared_rank(&sp, 0);
      for (int r = 0; r < k; ++r) {
        unsigned long long best = 0ull;
#pragma unroll
        for (int w = 0; w < SEL_NW; ++w)
          if (cand[w] < prev && cand[w] > best) best = cand[w];
        best = warp_max_key(best);
        if (lane == 0) r0->cand[rank][r] = best;  // 0: no more candidates in this range
        prev = best;
      }
      if (lane == 0) r0->ncand[rank] = ncand;
    }
  }
  cluster.sync();

  // ---- rank 0: the k largest of the candidates, the forced blocks, ascending
  if (rank == 0 && warp == 0) {
    int total = 0;
    for (int r = 0; r < S; ++r) total += sp.ncand[r];
    int32_t* out = p.block_idx + static_cast<size_t>(bh) * p.kmax;
    if (k >= total) {
      // every block is kept (nbv <= k + forced <= kmax)
      for (int i = lane; i < nbv; i += 32) out[i] = i;
      if (lane == 0) p.n_kept[bh] = nbv;
    } else {
      unsigned long long prev = ~0ull;
      int won = -1;  // lane r: the global index of the (r+1)-th largest
      for (int r = 0; r < k; ++r) {
        unsigned long long best = 0ull;
        for (int c = lane; c < S * SEL_TOPK; c += 32) {
          const int cr = c / SEL_TOPK, ci = c - cr * SEL_TOPK;
          if (ci < k) {
            const unsigned long long x = sp.cand[cr][ci];
            if (x < prev && x > best) best = x;
          }
        }
        best = warp_max_key(best);
        if (lane == r) won = static_cast<int>(0xffffffffu - static_cast<uint32_t>(best));
        prev = best;
      }
      // forced blocks in lanes k and k + 1
      const int f0 = (p.force_first && nbv > 0) ? 0 : -1;
      const int f1 = (p.force_last && nbv > 1) ? nbv - 1 : -1;
      if (lane == k) won = f0;
      if (lane == k + 1) won = f1;
      if (lane == k + 1 && f1 == f0) won = -1;  // nbv == 1 with both forced: one block
      // ascending: position = how many kept indices are smaller
      int pos = 0, tot = 0;
      for (int j = 0; j < 32; ++j) {
        const int o = __shfl_sync(FULL_MASK, won, j);
        pos += (o >= 0 && o < won);
        tot += (o >= 0);
      }
      if (won >= 0 && pos < p.kmax) out[pos] = won;
      if (lane == 0) p.n_kept[bh] = min(tot, p.kmax);
    }
  }
  cluster.sync();  // no CTA leaves while rank 0 may still read its candidates
}

template <typename T, int D, int G, int MODE>
static cudaError_t split_one(const SelParams& p, int NBH, int S, cudaStream_t st) {
  const int segcap = (p.NBcap + S - 1) / S;
  const size_t smem = sel_summary_smem_bytes(G, segcap);
  static std::atomic<int> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured.load() & (1 << (dev & 31)))) {
    size_t most = sel_summary_smem_bytes(G, (SEL_MAXNB + 1) / 2);
    if (most > 200 * 1024) most = 200 * 1024;
    const cudaError_t e = cudaFuncSetAttribute(select_split_kernel<T, D, G, MODE>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(most));
    if (e != cudaSuccess) return e;
    configured.fetch_or(1 << (dev & 31));
  }
  if (smem > 200 * 1024) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(NBH * S));
  cfg.blockDim = dim3(SEL_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(S);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, select_split_kernel<T, D, G, MODE>, p, segcap);
}

template <typename T, int D, int MODE>
static cudaError_t split_g(int G, const SelParams& p, int NBH, int S, cudaStream_t st) {
  switch (G) {
    case 1: return split_one<T, D, 1, MODE>(p, NBH, S, st);
    case 2: return split_one<T, D, 2, MODE>(p, NBH, S, st);
    case 3: return split_one<T, D, 3, MODE>(p, NBH, S, st);
    case 4: return split_one<T, D, 4, MODE>(p, NBH, S, st);
    case 5: return split_one<T, D, 5, MODE>(p, NBH, S, st);
    case 6: return split_one<T, D, 6, MODE>(p, NBH, S, st);
    case 7: return split_one<T, D, 7, MODE>(p, NBH, S, st);
    case 8: return split_one<T, D, 8, MODE>(p, NBH, S, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_select_split(int dtype, int D, int G, int mode, const SelParams& p, int NBH, int S,
                                cudaStream_t st) {
  if (S < 2 || S > SPLIT_MAX_S || p.k_top > SEL_TOPK) return cudaErrorInvalidValue;
  if (mode == SEL_MEAN16) {
    if (dtype != KV_BF16) return cudaErrorInvalidValue;
    return D == 64 ? split_g<__nv_bfloat16, 64, SEL_MEAN16>(G, p, NBH, S, st)
                   : split_g<__nv_bfloat16, 128, SEL_MEAN16>(G, p, NBH, S, st);
  }
  if (mode != SEL_SUMMARY) return cudaErrorInvalidValue;
  if (dtype == KV_BF16)
    return D == 64 ? split_g<__nv_bfloat16, 64, SEL_SUMMARY>(G, p, NBH, S, st)
                   : split_g<__nv_bfloat16, 128, SEL_SUMMARY>(G, p, NBH, S, st);
  return D == 64 ? split_g<float, 64, SEL_SUMMARY>(G, p, NBH, S, st)
                 : split_g<float, 128, SEL_SUMMARY>(G, p, NBH, S, st);
}
}  // namespace kvs
