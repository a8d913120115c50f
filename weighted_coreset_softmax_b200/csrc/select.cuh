// Per-KV-head block choice for one decode step.
//
// Sources: "COBS: Cumulant Order Block Sparse Attention" -- Equation (5): a KV
// head's shared block set is ranked by the group score, the sum over its G query
// heads of per-head block softmax probabilities m_b / Z^(g,h); the first-order
// (mean-pool) estimate of ln m_b, s = q . (block mean key) + ln n_b (text after
// Equation (8) and the affine score (18)); OSA computes the exact masses from all
// block keys instead (the OSA paragraph).
//
// Design (sm_100a). One 256-thread CTA per (sequence, KV head), two per SM.
//  scoring: summary mode is a GEMV over the fp32 block key sums -- each warp
//  streams rows with 16-byte loads, several rows in flight per lane, and finishes
//  the G dot products of a row batch with a transpose reduction; exact mode
//  streams every key of a block and keeps an online log-sum-exp per head. The
//  block logits (log2 domain) stay in shared memory.
//  normalisers: one warp per query head reduces max and sum over the blocks.
//  ranking: each block gets a 64-bit key (score bits, then the inverted block
//  index, so larger keys win and ties go to the lower index); a most-significant-
//  digit-first radix select over those keys, with warp-aggregated shared-memory
//  histograms, finds the k-th largest key and stops as soon as the remaining
//  digit bucket is taken whole.
//  output: a CTA-wide prefix sum over the selected flags writes the kept blocks in
//  ascending order.
#pragma once

#include "common.cuh"
#include "rank.cuh"

#include <cuda_fp16.h>
#include <cuda_fp4.h>

namespace kvs {

constexpr int SEL_THREADS = 256;
constexpr int SEL_NW = SEL_THREADS / 32;
constexpr int SEL_MAXNB = 4096;  // NBcap limit

enum SelMode { SEL_SUMMARY = 0, SEL_EXACT = 1, SEL_QUEST = 2, SEL_COBS = 3, SEL_MEAN16 = 4, SEL_COBS4 = 5 };
// Row kinds of the summary-style scorer: fp32 key sums, Quest (min, max) bf16
// pairs (both four bytes a channel), bf16 block means (two bytes a channel).
enum SelRow { ROW_SUM32 = 0, ROW_QUEST = 1, ROW_MEAN16 = 2 };

struct SelParams {
  const void* q;
  const float* k_sum;
  const void* k_bounds;  // Quest mode: [B][Hkv][NBcap][D][2] bf16 (min, max)
  const void* k_mean16;  // bf16-mean mode: [B][Hkv][NBcap][D] bf16 block mean keys
  const float* k_xi;     // second-order mode: [B][Hkv][NBcap][cobs_r][D] fp32 scaled eigenvectors
  int cobs_r;
  // stored-descriptor second-order mode: [B][Hkv][NBcap][cobs_r][SP / 2] E2M1 codes
  // (element 2j in the low nibble), [B][Hkv][NBcap][cobs_r] fp32 scales, and the
  // query basis U [Hkv][s_dim][D] (NULL: the full space, s_dim = D); SP = s_dim
  // rounded up to 32
  const uint8_t* xi4;
  const float* xi4_scale;
  const float* Uq;
  int s_dim, SP;
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

// Shared memory beyond the dynamic arrays.
constexpr int SEL_STAGES = 3;
// k_top up to this takes the per-warp top-k path, larger k the radix select
constexpr int SEL_TOPK = 16;
constexpr int COV_MAX_RANK_SEL = 8;  // largest rank of the second-order factors

struct SelMisc {
  float lse[8];
  float pm[SEL_NW][8], ps[SEL_NW][8];  // per-warp (max, sum) of the normalisers (summary mode)
  union {
    unsigned hist[256];                          // radix select
    unsigned long long wtop[SEL_NW * SEL_TOPK];  // per-warp largest keys (k <= SEL_TOPK)
  };
  unsigned long long prefix, mask;
  int krem, digit, above, bucket;
  int wsum[SEL_NW];
  unsigned long long rbar[SEL_NW][SEL_STAGES];  // scorer ring: one mbarrier per warp and stage
};

// Dynamic shared memory: lg[G][NBP] floats | key[NBP] u64 | misc; summary mode
// adds cnt[NBP] i32 | the row ring (sel_ring_bytes, 16-byte aligned).
__host__ __device__ inline int sel_nbp(int NBcap) { return (NBcap + 31) & ~31; }
__host__ __device__ inline size_t sel_smem_bytes(int G, int NBcap) {
  const int nbp = sel_nbp(NBcap);
  return static_cast<size_t>(G) * nbp * 4 + static_cast<size_t>(nbp) * 8 + sizeof(SelMisc);
}

// Sum of one int per thread over the CTA; every thread gets the result.
__device__ __forceinline__ int sel_block_sum(int v, int* wsum) {
  v = __reduce_add_sync(FULL_MASK, v);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int w = 0; w < SEL_NW; ++w) s += wsum[w];
  __syncthreads();
  return s;
}

// Summary mode: lg[g][b] = (q_g * qscale) . k_sum_b / n_b + log2 n_b.
// Each warp takes 8-row batches (warp, warp + 8, ...); every lane moves its own
// 16-byte pieces of a batch (one column chunk of RS rows) into a lane-private
// three-stage ring with cp.async, so three batches per warp are in flight with
// no register staging and no synchronisation between lanes.
__host__ __device__ inline size_t sel_ring_bytes(int G) {
  const int GP = G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8));
  const int RS = GP >= 4 ? 32 / GP : 8;  // rows per lane per batch (D = 128; D = 64 needs fewer)
  return static_cast<size_t>(SEL_STAGES) * RS * SEL_THREADS * 16;
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t"
      "@p cp.async.cg.shared.global [%0], [%1], 16;\n\t}" ::"r"(smem_u32(dst)),
      "l"(src), "r"(static_cast<int>(pred))
      : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Dynamic shared memory of a summary-mode selector CTA.
__host__ __device__ inline size_t sel_summary_smem_bytes(int G, int NBcap) {
  return ((sel_smem_bytes(G, NBcap) + static_cast<size_t>(sel_nbp(NBcap)) * 4 + 15) & ~static_cast<size_t>(15)) +
         sel_ring_bytes(G);
}

// ROW_QUEST: the rows are the Quest bounds -- per channel a (min, max) bf16 pair,
// also four bytes per channel -- and a lane's logit part is sum_j max(q_j min_j,
// q_j max_j) over its four channels, with no count term ("COBS: Cumulant Order
// Block Sparse Attention", the Quest paragraph: the largest inner product any
// point of the block's bounding box can reach).
// ROW_MEAN16: the rows are the block mean keys at bf16 precision (the same
// page's quantisation paragraph keeps the block mean at bf16), two bytes a
// channel: a lane covers eight channels with one 16-byte piece, a 512-byte ring
// slot holds two rows at D = 128, and the logit is the dot plus log2 n_b (no
// division: the row is already the mean).
template <typename T, int D, int G, int ROWK = ROW_SUM32>
__device__ void score_summary(const SelParams& p, float* lg, int nbp, int bh, int nbv, float4* ring, int* cnt,
                              SelMisc& ms) {
  constexpr bool QUEST = ROWK == ROW_QUEST;
  constexpr bool M16 = ROWK == ROW_MEAN16;
  constexpr int CPL = M16 ? 8 : 4;        // channels per lane (one 16-byte piece)
  constexpr int RB = D * (M16 ? 2 : 4);   // bytes per row
  constexpr int LPR = D / CPL;            // lanes per row
  constexpr int RPW = 32 / LPR;
  constexpr int GP = pow2ceil(G);
  constexpr int RS0 = (D / 4) / GP;       // ring bytes as for fp32 rows (sel_ring_bytes)
  constexpr int RS = RS0 < 1 ? 1 : (RS0 > 8 ? 8 : RS0);  // row slots per lane per batch
  constexpr int NV = RS * GP;
  constexpr int BATCH = RPW * RS;                         // rows per warp per batch
  using HV = HeldValues<NV, LPR, GP>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rg = lane / LPR, c = lane % LPR;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  // RB bytes a row: fp32 sums, (min, max) bf16 pairs, or bf16 means
  const unsigned char* krows =
      static_cast<const unsigned char*>(QUEST ? p.k_bounds : (M16 ? p.k_mean16 : static_cast<const void*>(p.k_sum))) +
      static_cast<size_t>(bh) * p.NBcap * RB;
  const int nbt = (nbv + BATCH - 1) / BATCH;               // batches of the bh
  const int nmine = nbt > warp ? (nbt - warp + SEL_NW - 1) / SEL_NW : 0;  // batches of this warp
  // The ring is filled by bulk copies with an L2 evict-first policy (the rows are
  // read once a step; they should not push the next kernels' code and data out
  // of L2). Stage s, slot i of a warp is 512 contiguous bytes -- rows
  // rb + i * RPW .. + RPW - 1 -- at ring[(s * RS + i) * SEL_THREADS + warp * 32],
  // so lane (rg, c) finds its 16 bytes where its own copy would have put them.
  // Completion is counted in bytes on the warp's mbarrier of the stage.
  uint64_t* rbar = reinterpret_cast<uint64_t*>(ms.rbar[warp]);
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int m) {
    if (m >= nmine) return;  // warp-uniform
    const int st = m % SEL_STAGES;
    const int rb = (warp + m * SEL_NW) * BATCH;
    const int nvalid = min(BATCH, nbv - rb);  // >= 1: batch rb starts below nbv
    if (lane == 0) mbar_arrive_expect_tx(rbar + st, static_cast<uint32_t>(nvalid) * RB);
    __syncwarp();
    if (lane < RS) {
      const int r0 = rb + lane * RPW;
      const int nr = min(RPW, nbv - r0);
      if (nr > 0)
        bulk_g2s(ring + (st * RS + lane) * SEL_THREADS + warp * 32, krows + static_cast<size_t>(r0) * RB,
                 static_cast<uint32_t>(nr) * RB, rbar + st, pol);
    }
  };
#pragma unroll
  for (int m = 0; m < SEL_STAGES; ++m) issue(m);
  // counts and q while the first batches are in flight
  if constexpr (!QUEST) {
    const int32_t* cn = p.counts + static_cast<size_t>(b) * p.NBcap;
    for (int i = tid; i < nbv; i += SEL_THREADS) cnt[i] = __ldg(cn + i);
  }
  const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * D + c * CPL;
  float4 qf[G];
  float q8[M16 ? G : 1][8];
  if constexpr (M16) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) q8[g][e] = load_as_float(qrow + g * D + e) * p.qscale;
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g)
      qf[g] = make_float4(load_as_float(qrow + g * D) * p.qscale, load_as_float(qrow + g * D + 1) * p.qscale,
                          load_as_float(qrow + g * D + 2) * p.qscale, load_as_float(qrow + g * D + 3) * p.qscale);
  }
  // QUEST: max(q min, q max) = max(q, 0) max + min(q, 0) min (max >= min), two FMAs
  float qa[QUEST ? G : 1][4], qb[QUEST ? G : 1][4];
  if constexpr (QUEST) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float qv[4] = {qf[g].x, qf[g].y, qf[g].z, qf[g].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qa[g][e] = fmaxf(qv[e], 0.f);
        qb[g][e] = fminf(qv[e], 0.f);
      }
    }
  }
  __syncthreads();  // cnt
  // running (max, sum of 2^(x - max)) of the logits this lane holds: the Eq. 5
  // normalisers come out of the scoring pass
  float om[HV::NH], os[HV::NH];
#pragma unroll
  for (int j = 0; j < HV::NH; ++j) {
    om[j] = -INFINITY;
    os[j] = 0.f;
  }
  for (int m = 0; m < nmine; ++m) {
    const int st = m % SEL_STAGES;
    if (!mbar_wait(rbar + st, static_cast<uint32_t>((m / SEL_STAGES) & 1), nullptr))
      mbar_wait(rbar + st, static_cast<uint32_t>((m / SEL_STAGES) & 1), nullptr);  // bounded: let a late copy land

    const int rb = (warp + m * SEL_NW) * BATCH;
    float part[NV];
#pragma unroll
    for (int i = 0; i < RS; ++i) {
      const int row = rb + i * RPW + rg;
      const float4 k4 = row < nbv ? ring[(st * RS + i) * SEL_THREADS + tid] : make_float4(0.f, 0.f, 0.f, 0.f);
      if constexpr (M16) {
        // bf16 means of channels 8c .. 8c + 7
        float2 kf[4];
        Chunk<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(&k4), kf);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (g < G) {
            float d = q8[g][0] * kf[0].x;
            d = fmaf(q8[g][1], kf[0].y, d);
            d = fmaf(q8[g][2], kf[1].x, d);
            d = fmaf(q8[g][3], kf[1].y, d);
            d = fmaf(q8[g][4], kf[2].x, d);
            d = fmaf(q8[g][5], kf[2].y, d);
            d = fmaf(q8[g][6], kf[3].x, d);
            d = fmaf(q8[g][7], kf[3].y, d);
            part[i * GP + g] = d;
          } else {
            part[i * GP + g] = 0.f;
          }
        }
      } else if constexpr (QUEST) {
        // (min, max) pairs of channels 4c .. 4c + 3
        const __nv_bfloat162* mm = reinterpret_cast<const __nv_bfloat162*>(&k4);
        float lo[4], hi[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          lo[e] = __low2float(mm[e]);
          hi[e] = __high2float(mm[e]);
        }
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (g < G) {
            float d = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) d = fmaf(qa[g][e], hi[e], fmaf(qb[g][e], lo[e], d));
            part[i * GP + g] = d;
          } else {
            part[i * GP + g] = 0.f;
          }
        }
      } else {
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
    }
    // refill this stage: its values are in registers now; order those reads before
    // the copies that overwrite the slots
    __syncwarp();
    fence_proxy_async_smem();
    issue(m + SEL_STAGES);
    transpose_reduce<NV, LPR / 2>(part, lane);
#pragma unroll
    for (int j = 0; j < HV::NH; ++j) {
      const int vi = HV::index(c, j);
      const int ri = vi / GP, g = vi % GP;
      const int row = rb + ri * RPW + rg;
      if (g < G && row < nbv) {
        float x;
        if constexpr (QUEST) {
          x = part[j];  // the box bound, in the log2 domain through qscale
        } else if constexpr (M16) {
          const int nb = cnt[row];
          x = nb > 0 ? part[j] + log2f(static_cast<float>(nb)) : -INFINITY;
        } else {
          const int nb = cnt[row];
          x = nb > 0 ? part[j] / static_cast<float>(nb) + log2f(static_cast<float>(nb)) : -INFINITY;
        }
        lg[g * nbp + row] = x;
        if (x != -INFINITY) {
          if (x > om[j]) {
            os[j] = os[j] * exp2f(om[j] - x) + 1.f;
            om[j] = x;
          } else {
            os[j] += exp2f(x - om[j]);
          }
        }
      }
    }
  }
  // every copy issued was waited for above (batches m >= nmine issue none)
  // merge the pairs of the lanes that hold the same head (every lane bit that
  // changes the row), then one lane per head writes this warp's pair
#pragma unroll
  for (int j = 0; j < HV::NH; ++j) {
#pragma unroll
    for (int mask = HV::ROW_MASK_LO; mask < 32; mask <<= 1) {
      const float m2 = __shfl_xor_sync(FULL_MASK, om[j], mask), s2 = __shfl_xor_sync(FULL_MASK, os[j], mask);
      const float M = fmaxf(om[j], m2);
      os[j] = (om[j] == -INFINITY ? 0.f : os[j] * exp2f(om[j] - M)) + (m2 == -INFINITY ? 0.f : s2 * exp2f(m2 - M));
      om[j] = M;
    }
    const int vi = HV::index(c, j);
    const int ri = vi / GP, g = vi % GP;
    const bool holder = NV >= LPR || (c % (NV >= LPR ? 1 : LPR / NV)) == 0;
    if (ri == 0 && rg == 0 && holder && g < G) {
      ms.pm[warp][g] = om[j];
      ms.ps[warp][g] = os[j];
    }
  }
}

// Exact mode: lg[g][b] = log2 sum_{r in block} exp2((q_g * qscale) . k_r).
template <typename T, int D, int G>
__device__ void score_exact(const SelParams& p, float* lg, int nbp, int bh, int nbv, int n) {
  constexpr int ES = sizeof(T);
  constexpr int RB = D * ES;
  constexpr int LPR = RB / 16;
  constexpr int RPW = 32 / LPR;
  constexpr int CH2 = 8 / ES;
  constexpr int R = 4;
  constexpr int GP = pow2ceil(G);
  constexpr int NV = R * GP;
  constexpr int BATCH = RPW * R;
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
  for (int i = warp; i < nbv; i += SEL_NW) {
    const int t0 = i * p.L;
    const int cnt = min(p.L, n - t0);
    float M[HV::NH], S[HV::NH];
#pragma unroll
    for (int j = 0; j < HV::NH; ++j) {
      M[j] = -INFINITY;
      S[j] = 0.f;
    }
    for (int rb = 0; rb < cnt; rb += 2 * BATCH) {
      uint4 raw[2][R];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int row = rb + u * BATCH + r * RPW + rg;
          raw[u][r] = row < cnt ? __ldcs(reinterpret_cast<const uint4*>(Kb + static_cast<size_t>(t0 + row) * RB))
                                : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (rb + u * BATCH >= cnt) break;  // warp-uniform
        float part[NV];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float2 kf[CH2];
          Chunk<T>::unpack(raw[u][r], kf);
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
          const int row = rb + u * BATCH + ri * RPW + rg;
          const float sv = row < cnt ? part[j] : -INFINITY;
          // reduce over every lane bit that changes the row: the row bits inside
          // a row group and the row-group bits above them
          float cm = sv;
#pragma unroll
          for (int mask = HV::ROW_MASK_LO; mask < 32; mask <<= 1)
            cm = fmaxf(cm, __shfl_xor_sync(FULL_MASK, cm, mask));
          const float Mn = fmaxf(M[j], cm);  // finite: the batch's first row is valid
          float e = exp2f(sv - Mn);
#pragma unroll
          for (int mask = HV::ROW_MASK_LO; mask < 32; mask <<= 1) e += __shfl_xor_sync(FULL_MASK, e, mask);
          S[j] = S[j] * exp2f(M[j] - Mn) + e;
          M[j] = Mn;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < HV::NH; ++j) {
      const int g = HV::index(c, j) % GP;
      if (g < G) lg[g * nbp + i] = cnt > 0 ? M[j] + log2f(S[j]) : -INFINITY;
    }
  }
}

// Second-order term ("COBS: Cumulant Order Block Sparse Attention", text after
// Equation (8) and the low-rank form (13)): adds (sigma^2 / 2) sum_i (q . xi_i)^2
// to the first-order block logits in lg. In the log2 domain, with qs = q sigma
// log2(e), that is (ln 2 / 2) sum_i (qs . xi_i)^2. A warp takes NBW groups of RPW
// blocks at a time (D / 4 lanes per row, a float4 each) and issues all their
// factor-row loads (up to RMAX rows a block) before reducing, so NBW * RMAX loads
// per lane are in flight.
template <int D, int G, int NBW, int RMAX>
__device__ void cobs_second_order(const SelParams& p, float* lg, int nbp, int bh, int nbv, const float4 (&qf)[G]) {
  constexpr int LPR = D / 4;
  constexpr int RPW = 32 / LPR;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane / LPR;
  const int r = p.cobs_r;
  const float* base = p.k_xi + static_cast<size_t>(bh) * p.NBcap * r * D + (lane % LPR) * 4;
  for (int b0 = warp * RPW * NBW; b0 < nbv; b0 += SEL_NW * RPW * NBW) {
    float4 x[NBW][RMAX];
#pragma unroll
    for (int j = 0; j < NBW; ++j) {
      const int b = b0 + j * RPW + rg;
#pragma unroll
      for (int i = 0; i < RMAX; ++i)
        x[j][i] = (b < nbv && i < r)
                      ? __ldg(reinterpret_cast<const float4*>(base + (static_cast<size_t>(b) * r + i) * D))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < NBW; ++j) {
      const int b = b0 + j * RPW + rg;
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = 0.f;
#pragma unroll
      for (int i = 0; i < RMAX; ++i) {
        if (i >= r) break;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float d = qf[g].x * x[j][i].x;
          d = fmaf(qf[g].y, x[j][i].y, d);
          d = fmaf(qf[g].z, x[j][i].z, d);
          d = fmaf(qf[g].w, x[j][i].w, d);
#pragma unroll
          for (int o = LPR / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(FULL_MASK, d, o);
          acc[g] = fmaf(d, d, acc[g]);
        }
      }
      if (b < nbv && (lane % LPR) == 0)
#pragma unroll
        for (int g = 0; g < G; ++g) lg[g * nbp + b] += 0.34657359027997264f * acc[g];  // ln 2 / 2
    }
  }
}

// The same second-order term for D = 128 streamed through the scorer's ring (free
// once the first-order pass has drained it), filled the same way: one 512-byte
// bulk copy per slot with an L2 evict-first policy, completion counted on the
// warp's mbarrier of the stage (re-initialised after the first pass). A batch is
// BPB = RSC / r whole blocks (RSC rows a stage, consecutive in memory), SEL_STAGES
// batches in flight per warp, the warps taking batches in turn. Needs r <= RSC.
template <int G, int RSC>
__device__ void cobs_second_order_ring(const SelParams& p, float* lg, int nbp, int bh, int nbv, const float4 (&qf)[G],
                                       float4* ring, uint64_t* rbar) {
  constexpr int D = 128;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = p.cobs_r;
  const int bpb = RSC / r;
  const int nbt = (nbv + bpb - 1) / bpb;
  const int nmine = nbt > warp ? (nbt - warp + SEL_NW - 1) / SEL_NW : 0;
  const float* base = p.k_xi + static_cast<size_t>(bh) * p.NBcap * r * D;
  const uint64_t pol = l2_evict_first_policy();
  auto issue = [&](int m) {
    if (m >= nmine) return;  // warp-uniform
    const int st = m % SEL_STAGES;
    const int b0 = (warp + m * SEL_NW) * bpb;
    const int nrows = min(bpb, nbv - b0) * r;  // >= r: batch b0 starts below nbv
    if (lane == 0) mbar_arrive_expect_tx(rbar + st, static_cast<uint32_t>(nrows) * D * 4);
    __syncwarp();
    if (lane < nrows)  // row `lane` of the batch: factor lane % r of block b0 + lane / r
      bulk_g2s(ring + (st * RSC + lane) * SEL_THREADS + warp * 32, base + (static_cast<size_t>(b0) * r + lane) * D,
               D * 4, rbar + st, pol);
  };
#pragma unroll
  for (int m = 0; m < SEL_STAGES; ++m) issue(m);
  for (int m = 0; m < nmine; ++m) {
    const int st = m % SEL_STAGES;
    if (!mbar_wait(rbar + st, static_cast<uint32_t>((m / SEL_STAGES) & 1), nullptr))
      mbar_wait(rbar + st, static_cast<uint32_t>((m / SEL_STAGES) & 1), nullptr);  // bounded: let a late copy land
    const int b0 = (warp + m * SEL_NW) * bpb;
    float4 xs[RSC];
#pragma unroll
    for (int i = 0; i < RSC; ++i) xs[i] = ring[(st * RSC + i) * SEL_THREADS + tid];
    // refill this stage: its values are in registers now; order those reads before
    // the copies that overwrite the slots
    __syncwarp();
    fence_proxy_async_smem();
    issue(m + SEL_STAGES);
    // RSC rows x GP heads of partial dots, summed across the warp by halving
    // exchanges (NV - 1 shuffles): lane c then holds value c / SPAN (row * GP + head)
    constexpr int GP = pow2ceil(G);
    constexpr int NV = RSC * GP;  // <= 32
    constexpr int SPAN = 32 / NV;
    float part[NV];
#pragma unroll
    for (int i = 0; i < RSC; ++i)
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float d = 0.f;
        if (g < G) {
          d = qf[g].x * xs[i].x;
          d = fmaf(qf[g].y, xs[i].y, d);
          d = fmaf(qf[g].z, xs[i].z, d);
          d = fmaf(qf[g].w, xs[i].w, d);
        }
        part[i * GP + g] = d;
      }
    transpose_reduce<NV, 16>(part, lane);
    const int vi = lane / SPAN;
    const int row = vi / GP, g = vi - (vi / GP) * GP;
    const float sq = part[0] * part[0];
    float tot = sq;
    for (int t = 1; t < r; ++t) tot += __shfl_down_sync(FULL_MASK, sq, t * GP * SPAN);  // the block's later rows
    const int blk = b0 + row / r;
    if ((lane % SPAN) == 0 && g < G && row % r == 0 && row < bpb * r && blk < nbv)
      lg[g * nbp + blk] += 0.34657359027997264f * tot;  // ln 2 / 2
  }
  // every copy issued was waited for above (batches m >= nmine issue none)
}

// Second-order term from the stored descriptor ("COBS: Cumulant Order Block Sparse
// Attention", the subspace and quantisation paragraphs): adds (sigma^2 / 2)
// sum_i (q~ . xi_i)^2 to lg, q~ = U q the projected query (qt: the log2-domain q~ of
// the G heads, [G][SP] in shared memory, zero past s) and xi_i = scale_i *
// e2m1(codes_i), on the tensor cores (mma.sync m16n8k16, f16 inputs, fp32
// accumulation). A warp takes 4 blocks at a time: the 16 rows of A are (block j,
// factor i) = row 4j + i, the K dimension the SP subspace columns (SP / 16 steps); the
// 8 columns of B are the projected queries split into f16 high and low parts (heads
// 0..3 high, then low; for G > 4 two column tiles, all high then all low). A thread of
// the mma layout needs byte tig of every 32-bit word of its two rows (E2M1 codes, 2j in
// the low nibble): the E2M1 -> f16x2 conversion of that byte is exactly its A register
// for columns (2 tig, 2 tig + 1), or (+8, +9) for the odd words. E2M1 values are exact
// in f16, and high + low carries the query to about 22 bits. Epilogue: the high and low
// columns added (xor 2), squared, times scale^2, summed over the 4 factor rows (xor 4,
// 8), and (ln 2 / 2) times that added to the block's logits.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo_k, float hi_k) {
  const __half a = __float2half_rn(lo_k), b = __float2half_rn(hi_k);
  return static_cast<uint32_t>(__half_as_ushort(a)) | (static_cast<uint32_t>(__half_as_ushort(b)) << 16);
}

template <int G>
__device__ void cobs_fp4_second_order_tc(const SelParams& p, float* lg, int nbp, int bh, int nbv, const float* qt) {
  constexpr int NT = G <= 4 ? 1 : 2;  // column tiles of B
  constexpr int KMAX = 8;             // SP <= 128
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, tig = lane & 3;
  const int r = p.cobs_r, SP = p.SP, KS = SP / 16, WPR = SP / 8;  // k steps, words a row
  // B fragments: column n = grp of each tile; rows k = 16 ks + 2 tig (+1) and (+8, +9)
  uint32_t bq[NT][KMAX][2];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    // tile t, column grp: head and part
    int g, part;
    if constexpr (NT == 1) {
      g = grp & 3;
      part = grp >> 2;  // 0 high, 1 low
    } else {
      g = grp;
      part = t;
    }
#pragma unroll
    for (int ks = 0; ks < KMAX; ++ks) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float v[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int k = ks * 16 + tig * 2 + hh * 8 + e;
          const float x = (ks < KS && g < G) ? qt[g * SP + k] : 0.f;
          const float hi = __half2float(__float2half_rn(x));
          v[e] = part == 0 ? hi : x - hi;
        }
        bq[t][ks][hh] = pack_f16x2(v[0], v[1]);
      }
    }
  }
  const size_t fbytes = static_cast<size_t>(SP) / 2;
  const size_t base = static_cast<size_t>(bh) * p.NBcap * r;
  constexpr int U = 2;  // block quads a warp loads before converting any
  for (int f0 = 0; f0 < r; f0 += 4) {
    for (int bq0 = warp * 4; bq0 < nbv; bq0 += SEL_NW * 4 * U) {  // warp-uniform
      // per quad u: this thread's rows grp -> (block + grp / 4, factor f0 + grp % 4),
      // grp + 8 -> block + 2; whole rows (every thread of a quad loads them, keeping
      // different bytes)
      uint32_t w[U][2][12];
      float sc[U][2];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int b0 = bq0 + u * SEL_NW * 4;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int rb = b0 + (grp >> 2) + 2 * h2, rf = f0 + (grp & 3);
          const bool live = rb < nbv && rf < r;
          const size_t row = base + static_cast<size_t>(rb) * r + rf;
          const uint4* src = reinterpret_cast<const uint4*>(p.xi4 + row * fbytes);
#pragma unroll
          for (int q4 = 0; q4 < 3; ++q4) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (live && q4 < WPR / 4) v = __ldg(src + q4);
            w[u][h2][4 * q4] = v.x;
            w[u][h2][4 * q4 + 1] = v.y;
            w[u][h2][4 * q4 + 2] = v.z;
            w[u][h2][4 * q4 + 3] = v.w;
          }
          sc[u][h2] = live ? __ldg(p.xi4_scale + row) : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int b0 = bq0 + u * SEL_NW * 4;
        if (b0 >= nbv) break;  // warp-uniform
        float acc[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 6; ++ks) {
          if (ks < KS) {
            uint32_t a[4];
            a[0] = e2m1x2_to_f16x2((w[u][0][2 * ks] >> (8 * tig)) & 0xffu);
            a[1] = e2m1x2_to_f16x2((w[u][1][2 * ks] >> (8 * tig)) & 0xffu);
            a[2] = e2m1x2_to_f16x2((w[u][0][2 * ks + 1] >> (8 * tig)) & 0xffu);
            a[3] = e2m1x2_to_f16x2((w[u][1][2 * ks + 1] >> (8 * tig)) & 0xffu);
#pragma unroll
            for (int t = 0; t < NT; ++t) mma_f16_16816(acc[t], a, bq[t][ks][0], bq[t][ks][1]);
          }
        }
        if (KS > 6) {  // SP = 112 or 128: the last words, loaded here
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int rb = b0 + (grp >> 2) + 2 * h2, rf = f0 + (grp & 3);
            const bool live = rb < nbv && rf < r;
            const uint4* src =
                reinterpret_cast<const uint4*>(p.xi4 + (base + static_cast<size_t>(rb) * r + rf) * fbytes);
            const uint4 v = (live && WPR > 12) ? __ldg(src + 3) : make_uint4(0u, 0u, 0u, 0u);
            w[u][h2][0] = v.x;
            w[u][h2][1] = v.y;
            w[u][h2][2] = v.z;
            w[u][h2][3] = v.w;
          }
#pragma unroll
          for (int ks = 6; ks < KMAX; ++ks) {
            if (ks < KS) {
              uint32_t a[4];
              a[0] = e2m1x2_to_f16x2((w[u][0][2 * (ks - 6)] >> (8 * tig)) & 0xffu);
              a[1] = e2m1x2_to_f16x2((w[u][1][2 * (ks - 6)] >> (8 * tig)) & 0xffu);
              a[2] = e2m1x2_to_f16x2((w[u][0][2 * (ks - 6) + 1] >> (8 * tig)) & 0xffu);
              a[3] = e2m1x2_to_f16x2((w[u][1][2 * (ks - 6) + 1] >> (8 * tig)) & 0xffu);
#pragma unroll
              for (int t = 0; t < NT; ++t) mma_f16_16816(acc[t], a, bq[t][ks][0], bq[t][ks][1]);
            }
          }
        }
        // dots: acc[t][e] is row grp (e < 2) or grp + 8 (e >= 2), column 2 tig + (e & 1)
        float dot[4];
        if constexpr (NT == 1) {
#pragma unroll
          for (int e = 0; e < 4; ++e) dot[e] = acc[0][e] + __shfl_xor_sync(FULL_MASK, acc[0][e], 2);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) dot[e] = acc[0][e] + acc[1][e];
        }
        // squares times scale^2, summed over the 4 factor rows (lane bits 2, 3)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float s2 = sc[u][e >> 1] * sc[u][e >> 1];
          float v = dot[e] * dot[e] * s2;
          v += __shfl_xor_sync(FULL_MASK, v, 4);
          v += __shfl_xor_sync(FULL_MASK, v, 8);
          dot[e] = v;
        }
        // lanes with grp % 4 == 0 hold blocks b0 + grp / 4 (e < 2) and + 2 (e >= 2)
        if ((grp & 3) == 0 && (NT == 2 || tig < 2)) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int g = 2 * tig + (e & 1);
            const int blk = b0 + (grp >> 2) + 2 * (e >> 1);
            if (g < G && blk < nbv) lg[g * nbp + blk] += 0.34657359027997264f * dot[e];  // ln 2 / 2
          }
        }
      }
    }
  }
}

template <typename T, int D, int G, int MODE>
__global__ void __launch_bounds__(SEL_THREADS, 2) select_kernel(const SelParams p) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int nbp = sel_nbp(p.NBcap);
  float* lg = reinterpret_cast<float*>(sel_smem);
  unsigned long long* key = reinterpret_cast<unsigned long long*>(sel_smem + static_cast<size_t>(G) * nbp * 4);
  SelMisc& ms = *reinterpret_cast<SelMisc*>(sel_smem + static_cast<size_t>(G) * nbp * 4 + static_cast<size_t>(nbp) * 8);
  const int bh = blockIdx.x;
  const int b = bh / p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dep_wait();    // inputs may come from the kernel before this one
  grid_dep_launch();  // every CTA of this grid is resident: the next kernel may be scheduled
  const int n = max(0, min(p.seq_lens[b], p.Ncap));
  const int nbv = (n + p.L - 1) / p.L;

  if (MODE == SEL_SUMMARY || MODE == SEL_QUEST || MODE == SEL_COBS || MODE == SEL_MEAN16 || MODE == SEL_COBS4) {
    // the scorer ring's mbarriers (one per warp and stage)
    if (tid == 0) {
#pragma unroll
      for (int w = 0; w < SEL_NW; ++w)
#pragma unroll
        for (int st = 0; st < SEL_STAGES; ++st) mbar_init(reinterpret_cast<uint64_t*>(&ms.rbar[w][st]), 1);
      fence_mbar_init();
    }
    __syncthreads();
    int* cnt = reinterpret_cast<int*>(sel_smem + sel_smem_bytes(G, p.NBcap));
    float4* ring = reinterpret_cast<float4*>(sel_smem + ((sel_smem_bytes(G, p.NBcap) + static_cast<size_t>(nbp) * 4 + 15) & ~static_cast<size_t>(15)));
    score_summary<T, D, G,
                  MODE == SEL_QUEST ? ROW_QUEST : ((MODE == SEL_MEAN16 || MODE == SEL_COBS4) ? ROW_MEAN16 : ROW_SUM32)>(
        p, lg, nbp, bh, nbv, ring, cnt, ms);
  }
  else
    score_exact<T, D, G>(p, lg, nbp, bh, nbv, n);
  __syncthreads();
  if constexpr (MODE == SEL_COBS) {
    // the first-order logits are in lg; add the second-order term
    const int h = bh - b * p.Hkv;
    const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * D + (lane % (D / 4)) * 4;
    float4 qf[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
      qf[g] = make_float4(load_as_float(qrow + g * D) * p.qscale, load_as_float(qrow + g * D + 1) * p.qscale,
                          load_as_float(qrow + g * D + 2) * p.qscale, load_as_float(qrow + g * D + 3) * p.qscale);
    constexpr int RSC = pow2ceil(G) >= 4 ? 32 / pow2ceil(G) : 8;  // ring rows a stage (sel_ring_bytes)
    if constexpr (D == 128) {
      if (p.cobs_r <= RSC) {
        float4* ring = reinterpret_cast<float4*>(
            sel_smem + ((sel_smem_bytes(G, p.NBcap) + static_cast<size_t>(nbp) * 4 + 15) & ~static_cast<size_t>(15)));
        // fresh ring barriers: the first pass left them at different phases
        if (tid == 0) {
#pragma unroll
          for (int w = 0; w < SEL_NW; ++w)
#pragma unroll
            for (int st = 0; st < SEL_STAGES; ++st) {
              mbar_inval(reinterpret_cast<uint64_t*>(&ms.rbar[w][st]));
              mbar_init(reinterpret_cast<uint64_t*>(&ms.rbar[w][st]), 1);
            }
          fence_mbar_init();
        }
        __syncthreads();
        cobs_second_order_ring<G, RSC>(p, lg, nbp, bh, nbv, qf, ring, reinterpret_cast<uint64_t*>(ms.rbar[warp]));
      } else {
        cobs_second_order<D, G, 1, COV_MAX_RANK_SEL>(p, lg, nbp, bh, nbv, qf);
      }
    } else if (p.cobs_r <= 4) {
      cobs_second_order<D, G, 4, 4>(p, lg, nbp, bh, nbv, qf);
    } else {
      cobs_second_order<D, G, 1, COV_MAX_RANK_SEL>(p, lg, nbp, bh, nbv, qf);
    }
    __syncthreads();
  }

  if constexpr (MODE == SEL_COBS4) {
    // the first-order (bf16-mean) logits are in lg; the projected queries go where the
    // scorer's ring was
    float* qt = reinterpret_cast<float*>(
        sel_smem + ((sel_smem_bytes(G, p.NBcap) + static_cast<size_t>(nbp) * 4 + 15) & ~static_cast<size_t>(15)));
    const int h = bh - b * p.Hkv;
    const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * D;
    if (p.Uq) {
      // q~[g][j] = U_j . q_g: a warp per basis row j (coalesced), the group's queries
      // in registers (D / 32 channels a lane)
      constexpr int CPL = D / 32;
      float qreg[G][CPL];
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int k = 0; k < CPL; ++k) qreg[g][k] = load_as_float(qrow + g * D + lane * CPL + k);
      // the warp's basis rows, eight at a time, all eight loaded before the first
      // reduction, so their latencies overlap
      constexpr int RB8 = 8;
      for (int j0 = warp; j0 < p.SP; j0 += RB8 * SEL_NW) {  // warp-uniform
        float u[RB8][CPL];
#pragma unroll
        for (int jj = 0; jj < RB8; ++jj) {
          const int j = j0 + jj * SEL_NW;
#pragma unroll
          for (int k = 0; k < CPL; ++k)
            u[jj][k] = j < p.s_dim ? __ldg(p.Uq + (static_cast<size_t>(h) * p.s_dim + j) * D + lane * CPL + k) : 0.f;
        }
#pragma unroll
        for (int jj = 0; jj < RB8; ++jj) {
          const int j = j0 + jj * SEL_NW;
          if (j >= p.SP) break;  // warp-uniform
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float v = 0.f;
#pragma unroll
            for (int k = 0; k < CPL; ++k) v = fmaf(u[jj][k], qreg[g][k], v);
            v = warp_sum(v);
            if (lane == 0) qt[g * p.SP + j] = v * p.qscale;
          }
        }
      }
    } else {
      for (int e = tid; e < G * p.SP; e += SEL_THREADS) {
        const int g = e / p.SP, j = e - (e / p.SP) * p.SP;
        qt[e] = (j < p.s_dim ? load_as_float(qrow + g * D + j) : 0.f) * p.qscale;
      }
    }
    __syncthreads();
    cobs_fp4_second_order_tc<G>(p, lg, nbp, bh, nbv, qt);  // SP <= D <= 128
    __syncthreads();
  }

  // per-head normaliser log2 sum_b 2^lg (Equation 5's Z, log2 domain): in summary
  // and Quest modes from the warps' (max, sum) pairs of the scoring pass, else
  // (exact and second-order modes) a pass over lg
  if (MODE == SEL_SUMMARY || MODE == SEL_QUEST || MODE == SEL_MEAN16) {
    if (warp == 0 && lane < G) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < SEL_NW; ++w) M = fmaxf(M, ms.pm[w][lane]);
      float S = 0.f;
      if (M != -INFINITY)
#pragma unroll
        for (int w = 0; w < SEL_NW; ++w)
          if (ms.pm[w][lane] != -INFINITY) S += ms.ps[w][lane] * exp2f(ms.pm[w][lane] - M);
      ms.lse[lane] = (M == -INFINITY || S <= 0.f) ? -INFINITY : M + log2f(S);
    }
  } else if (warp < G) {
    float M = -INFINITY;
    for (int i = lane; i < nbv; i += 32) M = fmaxf(M, lg[warp * nbp + i]);
    M = warp_max(M);
    float S = 0.f;
    if (M != -INFINITY)
      for (int i = lane; i < nbv; i += 32) S += exp2f(lg[warp * nbp + i] - M);
    S = warp_sum(S);
    if (lane == 0) ms.lse[warp] = (M == -INFINITY || S <= 0.f) ? -INFINITY : M + log2f(S);
  }
  __syncthreads();

  // group score and ranking keys
  int ncand = 0;
  for (int i = tid; i < nbv; i += SEL_THREADS) {
    float Sg = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (ms.lse[g] != -INFINITY) Sg += exp2f(lg[g * nbp + i] - ms.lse[g]);
    if (p.scores) p.scores[static_cast<size_t>(bh) * p.NBcap + i] = Sg;
    const bool forced = (p.force_first && i == 0) || (p.force_last && i == nbv - 1);
    key[i] = forced ? 0ull
                    : ((static_cast<unsigned long long>(__float_as_uint(Sg)) << 32) |
                       static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(i)));
    ncand += !forced;
  }
  if (p.scores)
    for (int i = nbv + tid; i < p.NBcap; i += SEL_THREADS) p.scores[static_cast<size_t>(bh) * p.NBcap + i] = 0.f;
  ncand = sel_block_sum(ncand, ms.wsum);  // also orders the key writes

  if (p.k_top > 0 && p.k_top < ncand && p.k_top <= SEL_TOPK) {
    // Small k: each warp extracts the k largest keys of its share of the blocks
    // (k rounds of "largest key below the previous one"); warp 0 takes the k
    // largest of those, adds the forced blocks and writes the kept list in
    // ascending order. Keys of candidates are distinct and nonzero (the inverted
    // index is in the low bits), and ncand > k >= 1 means nbv >= 2, so the two
    // forced blocks are distinct.
    const int per = (nbv + SEL_NW - 1) / SEL_NW;
    const int lo = warp * per, hi = min(nbv, lo + per);
    unsigned long long prev = ~0ull;
    for (int r = 0; r < p.k_top; ++r) {
      unsigned long long best = 0ull;
      for (int i = lo + lane; i < hi; i += 32) {
        const unsigned long long x = key[i];
        if (x < prev && x > best) best = x;
      }
      best = warp_max_key(best);
      if (lane == 0) ms.wtop[warp * SEL_TOPK + r] = best;  // 0: no more candidates here
      prev = best;
    }
    __syncthreads();
    if (warp == 0) {
      unsigned long long cand[SEL_NW];
#pragma unroll
      for (int w = 0; w < SEL_NW; ++w) cand[w] = lane < p.k_top ? ms.wtop[w * SEL_TOPK + lane] : 0ull;
      unsigned long long won = 0ull;  // lane r: the (r+1)-th largest key
      prev = ~0ull;
      for (int r = 0; r < p.k_top; ++r) {
        unsigned long long best = 0ull;
#pragma unroll
        for (int w = 0; w < SEL_NW; ++w)
          if (cand[w] < prev && cand[w] > best) best = cand[w];
        best = warp_max_key(best);
        if (lane == r) won = best;
        prev = best;
      }
      int blk = lane < p.k_top ? static_cast<int>(0xffffffffu - static_cast<uint32_t>(won)) : -1;
      int nsel = p.k_top;
      if (p.force_first) {
        if (lane == nsel) blk = 0;
        ++nsel;
      }
      if (p.force_last) {
        if (lane == nsel) blk = nbv - 1;
        ++nsel;
      }
      int rank = 0;  // position in ascending order (indices are distinct)
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const int o = __shfl_sync(FULL_MASK, blk, j);
        rank += (o >= 0 && o < blk);
      }
      if (blk >= 0 && rank < p.kmax) p.block_idx[static_cast<size_t>(bh) * p.kmax + rank] = blk;
      if (lane == 0) p.n_kept[bh] = min(nsel, p.kmax);
    }
    return;
  }

  // threshold: select keys with (key & mask) >= prefix
  unsigned long long prefix = 1ull, mask = ~0ull;  // default: every candidate
  if (p.k_top <= 0) {
    prefix = ~0ull;  // nothing competes successfully
  } else if (p.k_top < ncand) {
    if (tid == 0) {
      ms.prefix = 0ull;
      ms.mask = 0ull;
      ms.krem = p.k_top;
    }
    for (int shift = 56; shift >= 0; shift -= 8) {
      if (tid < 256) ms.hist[tid] = 0u;
      __syncthreads();
      const unsigned long long pf = ms.prefix, mk = ms.mask;
      for (int i0 = 0; i0 < nbv; i0 += SEL_THREADS) {
        const int i = i0 + tid;
        int d = -1;
        if (i < nbv) {
          const unsigned long long x = key[i];
          if (x != 0ull && (x & mk) == pf) d = static_cast<int>((x >> shift) & 0xffull);
        }
        // warp-aggregated histogram update
        const unsigned peers = __match_any_sync(FULL_MASK, d);
        if (d >= 0 && (__ffs(peers) - 1) == lane) atomicAdd(&ms.hist[d], static_cast<unsigned>(__popc(peers)));
      }
      __syncthreads();
      if (warp == 0) {
        // lane l covers digits 255-8l .. 248-8l (descending)
        unsigned h8[8];
        unsigned tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          h8[j] = ms.hist[255 - 8 * lane - j];
          tot += h8[j];
        }
        unsigned incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned v = __shfl_up_sync(FULL_MASK, incl, o);
          if (lane >= o) incl += v;
        }
        const unsigned before = incl - tot;  // keys in higher digits than this lane's
        const unsigned krem = static_cast<unsigned>(ms.krem);
        if (before < krem && krem <= incl) {
          unsigned run = before;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (run < krem && krem <= run + h8[j]) {
              ms.digit = 255 - 8 * lane - j;
              ms.above = static_cast<int>(run);
              ms.bucket = static_cast<int>(h8[j]);
            }
            run += h8[j];
          }
        }
      }
      __syncthreads();
      if (tid == 0) {
        ms.krem -= ms.above;
        ms.prefix |= static_cast<unsigned long long>(ms.digit) << shift;
        ms.mask |= 0xffull << shift;
      }
      __syncthreads();
      if (ms.bucket == ms.krem) break;  // the whole bucket is taken: done (uniform)
    }
    prefix = ms.prefix;
    mask = ms.mask;
  }

  // ascending compaction of the selected blocks (forced ones included)
  const int per = (nbv + SEL_THREADS - 1) / SEL_THREADS;
  const int a0 = min(nbv, tid * per), a1 = min(nbv, a0 + per);
  int mine = 0;
  for (int i = a0; i < a1; ++i) {
    const unsigned long long x = key[i];
    const bool forced = (p.force_first && i == 0) || (p.force_last && i == nbv - 1);
    mine += forced || (x != 0ull && (x & mask) >= prefix);
  }
  // exclusive scan over the CTA
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(FULL_MASK, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) ms.wsum[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
#pragma unroll
  for (int w = 0; w < SEL_NW; ++w) {
    const int v = ms.wsum[w];
    if (w < warp) wbase += v;
    total += v;
  }
  int pos = wbase + incl - mine;
  for (int i = a0; i < a1; ++i) {
    const unsigned long long x = key[i];
    const bool forced = (p.force_first && i == 0) || (p.force_last && i == nbv - 1);
    if (forced || (x != 0ull && (x & mask) >= prefix)) {
      if (pos < p.kmax) p.block_idx[static_cast<size_t>(bh) * p.kmax + pos] = i;
      ++pos;
    }
  }
  if (tid == 0) p.n_kept[bh] = min(total, p.kmax);
}

}  // namespace kvs
