// Split-K gather attention for decode: exact softmax attention over the kept
// blocks' tokens plus the count-aware tail proxy (block mode), over a weighted
// coreset (weighted mode), or over every cached token (dense mode).
//
// Method sources:
//  * "OpenAttention reads 1% of the KV cache -- Count-aware tail proxy", section
//    "Skipping reviews without losing the verdict": the unread tail enters the
//    softmax as one token whose value is the tail's mean value and whose logit is
//    its mean logit plus ln(count); it is handled like an ordinary token, so here
//    it is one more partial result merged with the others.
//  * "WildCat: Near-Linear Attention in Theory and Practice", abstract: weighted
//    coreset attention, logit + ln w_i.
//  * "COBS: Cumulant Order Block Sparse Attention", read-traffic accounting:
//    dense attention reads the whole cache.
//
// Design (sm_100a). All (sequence, KV head) pairs ("bh") lay their P token slots
// end to end on one axis; the grid (about two CTAs per SM) splits that axis into
// equal contiguous ranges, so every CTA streams the same number of bytes whatever
// the per-head work. In each CTA one producer warp walks its range in chunks of
// TR rows and moves the K and V rows of each chunk into a 4-stage shared-memory
// ring with cp.async.bulk (one copy per contiguous run; one per row when rows are
// gathered), completion tracked by mbarrier transaction counts. Four consumer
// warps compute q.k for all G query heads of the group in fp32 (16-byte row
// chunks per lane, packed f32x2 FMAs, a transpose reduction across the lanes of a
// row), keep an online softmax per row group in the log2 domain, and accumulate
// p * v. When the range leaves a bh (or ends) the consumers merge their states
// into one partial record (m, l, acc) in the workspace and take an arrival ticket
// for that bh; whichever CTA arrives last merges all of the bh's records (and the
// proxy record) into the output. No CTA ever waits for another.
#pragma once

#include "common.cuh"

namespace kvs {

enum AttnMode { ATTN_BLOCKS = 0, ATTN_WEIGHTED = 1, ATTN_DENSE = 2 };

struct AttnParams {
  const void* q;
  const void* K;
  const void* V;
  const int32_t* seq_lens;
  const int32_t* block_idx;
  const int32_t* n_kept;
  int kmax;
  const float* k_sum;
  const float* v_sum;
  const int32_t* counts;
  const float* k_tot;
  const float* v_tot;
  const int32_t* tok_idx;
  const float* w;
  int m;
  float* out;
  float* lse;
  uint32_t* status;
  uint32_t* counters;
  float* recs;
  float* proxy_recs;
  int B, Hq, Hkv, Ncap, L, NBcap;
  int mode;
  int use_proxy;
  float qscale;  // softmax scale * log2(e): logits are kept in the log2 domain
  Partition part;
};

template <typename T, int D, int G>
struct AttnCfg {
  static constexpr int ES = sizeof(T);
  static constexpr int RB = D * ES;        // bytes per cached row
  static constexpr int LPR = RB / 16;      // lanes per row (16 bytes each)
  static constexpr int RPW = 32 / LPR;     // row groups per warp
  static constexpr int CH = 16 / ES;       // elements per lane chunk
  static constexpr int CH2 = CH / 2;       // float2 pairs per lane chunk
  static constexpr int R = 4;              // rows per lane per chunk
  static constexpr int NCW = 4;            // consumer warps
  static constexpr int NTHREADS = (NCW + 1) * 32;
  static constexpr int TR = NCW * RPW * R;  // rows per chunk (8 KB of K, 8 KB of V)
  static constexpr int GP = pow2ceil(G);
  static constexpr int NV = R * GP;        // partial dots per lane per chunk
  // Up to G = 4 two CTAs share an SM; larger groups need more registers, so one
  // CTA per SM runs with a deeper ring to keep as many bytes in flight.
  static constexpr int CPS = G <= 4 ? 2 : 1;          // CTAs per SM
  static constexpr int S = G <= 4 ? 4 : 8;            // pipeline stages
  using HV = HeldValues<NV, LPR, GP>;
  static constexpr int NH = HV::NH;
  static constexpr int QBYTES = G * D * ES;
  static constexpr int QB = (QBYTES + 15) & ~15;
  static constexpr int PSTR = GP < 4 ? 4 : GP;  // floats per P row (16-byte rows)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TR * RB;
  static constexpr int OFF_Q = 2 * TR * RB;
  static constexpr int OFF_BIAS = OFF_Q + QB;
  static constexpr int OFF_HDR = OFF_BIAS + TR * 4;
  static constexpr int STAGE = (OFF_HDR + 16 + 127) & ~127;
  static constexpr int OFF_BARS = S * STAGE;
  static constexpr int OFF_P = OFF_BARS + 128;
  static constexpr int PW_FLOATS = RPW * (R + 1) * PSTR;  // per consumer warp
  static constexpr int OFF_MERGE = OFF_P + NCW * PW_FLOATS * 4;
  static constexpr int MERGE_FLOATS = NCW * G * D + 2 * NCW * G;
  static constexpr int SMEM = OFF_MERGE + MERGE_FLOATS * 4;
  static constexpr int RECF = (G * D + 2 * G + 3) & ~3;
  static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "row layout");
  static_assert(TR <= 64, "producer covers at most 64 rows per chunk");
  static_assert(2 * S * 8 <= 128, "barrier area");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ float safe_max_ref(float m) { return m == -INFINITY ? 0.f : m; }

// Walks [cur, end) of the token axis in chunks that stay inside one bh, hold at
// most TR rows, and (block mode) stay inside one kept block.
struct ChunkIter {
  int64_t cur, end;
  __device__ __forceinline__ bool next(int P, int L, int TR, int mode, int& bh, int& j0, int& rows) {
    if (cur >= end) return false;
    bh = static_cast<int>(cur / P);
    j0 = static_cast<int>(cur - static_cast<int64_t>(bh) * P);
    int64_t lim = min(end, static_cast<int64_t>(bh + 1) * P) - cur;
    int r = static_cast<int>(min(lim, static_cast<int64_t>(TR)));
    if (mode == ATTN_BLOCKS) r = min(r, L - (j0 % L));
    rows = r;
    cur += r;
    return true;
  }
};

// Per-chunk metadata the producer loads one ring cycle ahead.
struct ChunkMeta {
  int has, bh, j0, rows, first;
  int n, nk, blk;   // seq_len; block mode: n_kept and block index of the slot
  int i0, i1;       // weighted mode: token index of rows lane, lane + 32
  float w0, w1;
};

__device__ __forceinline__ int expected_arrivals(const Partition& pt, int bh, int use_proxy) {
  const int64_t a = static_cast<int64_t>(bh) * pt.P;
  const int cf = part_cta_of(pt, a);
  const int cl = part_cta_of(pt, a + pt.P - 1);
  return cl - cf + 1 + (use_proxy ? 1 : 0);
}

// Merges every partial record of one bh into out / lse. One warp.
template <int D, int G>
__device__ void finalize_bh(const AttnParams& p, int bh, int lane) {
  constexpr int RECF = (G * D + 2 * G + 3) & ~3;
  constexpr int VEC = D / 32;
  const int64_t a = static_cast<int64_t>(bh) * p.part.P;
  const int cf = part_cta_of(p.part, a);
  const int cl = part_cta_of(p.part, a + p.part.P - 1);
  const int nrec = cl - cf + 1 + (p.use_proxy ? 1 : 0);
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  auto rec_ptr = [&](int j) -> const float* {
    return (j <= cl - cf) ? p.recs + static_cast<size_t>(cf + j + bh) * RECF
                          : p.proxy_recs + static_cast<size_t>(bh) * RECF;
  };
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
    for (int j = 0; j < nrec; ++j) M = fmaxf(M, __ldcg(rec_ptr(j) + G * D + g));
    const float Ms = safe_max_ref(M);
    float Lsum = 0.f;
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    for (int j = 0; j < nrec; ++j) {
      const float* r = rec_ptr(j);
      const float mj = __ldcg(r + G * D + g);
      const float wj = exp2f(mj - Ms);
      Lsum = fmaf(wj, __ldcg(r + G * D + G + g), Lsum);
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = fmaf(wj, __ldcg(r + g * D + lane * VEC + v), acc[v]);
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    float* o = p.out + (static_cast<size_t>(b) * p.Hq + h * G + g) * D + lane * VEC;
#pragma unroll
    for (int v = 0; v < VEC; ++v) o[v] = acc[v] * inv;
    if (p.lse && lane == 0)
      p.lse[static_cast<size_t>(b) * p.Hq + h * G + g] =
          Lsum > 0.f ? (M + log2f(Lsum)) * LN2 : -INFINITY;
  }
}

// Arrival ticket for bh; the last arriver merges. Called by one whole warp after
// its writes are complete and fenced.
template <int D, int G>
__device__ __forceinline__ void arrive_bh(const AttnParams& p, int bh, int lane) {
  int last = 0;
  if (lane == 0) {
    const int E = expected_arrivals(p.part, bh, p.use_proxy);
    const uint32_t old = atomicAdd(p.counters + bh, 1u);
    last = (old + 1 == static_cast<uint32_t>(E));
    if (last) p.counters[bh] = 0u;  // ready for the next launch
  }
  last = __shfl_sync(FULL_MASK, last, 0);
  if (last) {
    __threadfence();
    finalize_bh<D, G>(p, bh, lane);
  }
}

// The tail proxy of one bh as a partial record (m = its log2 logit, l = 1,
// acc = its value). One warp.
template <typename T, int D, int G>
__device__ void build_proxy(const AttnParams& p, int bh, int lane) {
  constexpr int RECF = (G * D + 2 * G + 3) & ~3;
  constexpr int VEC = D / 32;
  const int b = bh / p.Hkv, h = bh % p.Hkv;
  int n = p.seq_lens[b];
  if (n < 0 || n > p.Ncap) {
    if (lane == 0) atomicOr(p.status, KV_DEV_BAD_SEQ_LEN);
    n = max(0, min(n, p.Ncap));
  }
  const int nbv = (n + p.L - 1) / p.L;
  int nk = p.n_kept[bh];
  if (nk < 0 || nk > p.kmax) {
    if (lane == 0) atomicOr(p.status, KV_DEV_BAD_N_KEPT);
    nk = max(0, min(nk, p.kmax));
  }
  float ks[VEC], vs[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) ks[v] = vs[v] = 0.f;
  int cnt = 0, prev = -1;
  for (int s0 = 0; s0 < nk; s0 += 32) {
    const int mine = (s0 + lane < nk) ? p.block_idx[static_cast<size_t>(bh) * p.kmax + s0 + lane] : -1;
    const int lim = min(32, nk - s0);
    for (int jj = 0; jj < lim; ++jj) {
      const int blk = __shfl_sync(FULL_MASK, mine, jj);
      if (blk <= prev || blk >= nbv) {
        if (lane == 0) atomicOr(p.status, KV_DEV_BAD_BLOCK_INDEX);
        continue;
      }
      prev = blk;
      const size_t row = (static_cast<size_t>(bh) * p.NBcap + blk) * D + lane * VEC;
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        ks[v] += p.k_sum[row + v];
        vs[v] += p.v_sum[row + v];
      }
      cnt += p.counts[static_cast<size_t>(b) * p.NBcap + blk];
    }
  }
  const int nT = n - cnt;
  float* rec = p.proxy_recs + static_cast<size_t>(bh) * RECF;
  const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * D;
  if (nT > 0) {
    const float inv = 1.f / static_cast<float>(nT);
    float kb[VEC], vb[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      kb[v] = (p.k_tot[static_cast<size_t>(bh) * D + lane * VEC + v] - ks[v]) * inv;
      vb[v] = (p.v_tot[static_cast<size_t>(bh) * D + lane * VEC + v] - vs[v]) * inv;
    }
    const float lc = log2f(static_cast<float>(nT));
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
      float dot = 0.f;
#pragma unroll
      for (int v = 0; v < VEC; ++v) dot = fmaf(load_as_float(qrow + g * D + lane * VEC + v), kb[v], dot);
      dot = warp_sum(dot);
#pragma unroll
      for (int v = 0; v < VEC; ++v) rec[g * D + lane * VEC + v] = vb[v];
      if (lane == 0) {
        rec[G * D + g] = dot * p.qscale + lc;
        rec[G * D + G + g] = 1.f;
      }
    }
  } else {
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int v = 0; v < VEC; ++v) rec[g * D + lane * VEC + v] = 0.f;
      if (lane == 0) {
        rec[G * D + g] = -INFINITY;
        rec[G * D + G + g] = 0.f;
      }
    }
  }
  __threadfence();
  __syncwarp();
  arrive_bh<D, G>(p, bh, lane);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(AttnCfg<T, D, G>::NTHREADS, AttnCfg<T, D, G>::CPS)
    attn_kernel(const AttnParams p) {
  using C = AttnCfg<T, D, G>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int cta = blockIdx.x;
  const int64_t t0 = part_t0(p.part, cta);
  const int64_t t1 = part_t0(p.part, cta + 1);
  const int P = p.part.P;

  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  uint64_t* empty = full + C::S;
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < C::S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, C::NCW);
    }
    fence_mbar_init();
  }
  // Rows a chunk does not fill keep stale (finite) data; zero the K/V buffers
  // once so that no uninitialised pattern can ever be multiplied by p = 0.
  for (int s = 0; s < C::S; ++s) {
    uint4* b4 = reinterpret_cast<uint4*>(smem + s * C::STAGE);
    for (int i = tid; i < 2 * C::TR * C::RB / 16; i += C::NTHREADS) b4[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  __syncthreads();

  if (warp == C::NCW) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_evict_first_policy();
    const unsigned char* Kb = static_cast<const unsigned char*>(p.K);
    const unsigned char* Vb = static_cast<const unsigned char*>(p.V);
    const unsigned char* Qb = static_cast<const unsigned char*>(p.q);
    ChunkIter ahead{t0, t1};
    int prev_bh = -1;
    auto fetch = [&](ChunkMeta& mt) {
      int bh, j0, rows;
      mt.has = ahead.next(P, p.L, C::TR, p.mode, bh, j0, rows);
      if (!mt.has) return;
      mt.bh = bh;
      mt.j0 = j0;
      mt.rows = rows;
      mt.first = (bh != prev_bh);
      prev_bh = bh;
      const int b = bh / p.Hkv;
      mt.n = p.seq_lens[b];
      if (p.mode == ATTN_BLOCKS) {
        // with kmax = 0 the axis still has one (empty) slot per bh: read nothing
        const int slot = j0 / p.L;
        mt.nk = p.n_kept[bh];
        mt.blk = slot < p.kmax ? p.block_idx[static_cast<size_t>(bh) * p.kmax + slot] : -1;
      } else if (p.mode == ATTN_WEIGHTED) {
        // rows past m (m = 0 leaves one empty row per bh) are never read
        const size_t base = static_cast<size_t>(bh) * p.m + j0;
        const bool r0 = lane < rows && j0 + lane < p.m, r1 = lane + 32 < rows && j0 + lane + 32 < p.m;
        mt.i0 = r0 ? p.tok_idx[base + lane] : -1;
        mt.w0 = r0 ? p.w[base + lane] : 0.f;
        mt.i1 = r1 ? p.tok_idx[base + lane + 32] : -1;
        mt.w1 = r1 ? p.w[base + lane + 32] : 0.f;
      }
    };
    ChunkMeta ring[C::S];
    bool gave_up = false;  // after one timed-out wait, wait no more
#pragma unroll
    for (int s = 0; s < C::S; ++s) fetch(ring[s]);
    for (int base = 0;; base += C::S) {
      bool done = false;
#pragma unroll
      for (int s = 0; s < C::S; ++s) {
        ChunkMeta& mt = ring[s];
        if (!done && !mt.has) done = true;
        if (done) continue;
        const uint32_t phase = static_cast<uint32_t>(base / C::S) & 1u;
        if (base > 0 && !gave_up && !mbar_wait(empty + s, phase ^ 1u, p.status)) gave_up = true;
        unsigned char* stg = smem + s * C::STAGE;
        float* bias = reinterpret_cast<float*>(stg + C::OFF_BIAS);
        int* hdr = reinterpret_cast<int*>(stg + C::OFF_HDR);
        const int b = mt.bh / p.Hkv, h = mt.bh % p.Hkv;
        int n = mt.n;
        if (n < 0 || n > p.Ncap) {
          if (lane == 0) atomicOr(p.status, KV_DEV_BAD_SEQ_LEN);
          n = max(0, min(n, p.Ncap));
        }
        int nvalid = 0;
        int64_t tok0 = 0;
        bool v0 = false, v1 = false;
        if (p.mode == ATTN_WEIGHTED) {
          const bool in0 = mt.i0 >= 0 && mt.i0 < n, in1 = mt.i1 >= 0 && mt.i1 < n;
          v0 = lane < mt.rows && in0 && mt.w0 > 0.f;
          v1 = lane + 32 < mt.rows && in1 && mt.w1 > 0.f;
          if ((lane < mt.rows && mt.w0 > 0.f && !in0) || (lane + 32 < mt.rows && mt.w1 > 0.f && !in1))
            atomicOr(p.status, KV_DEV_BAD_TOKEN_INDEX);
          nvalid = __popc(__ballot_sync(FULL_MASK, v0)) + __popc(__ballot_sync(FULL_MASK, v1));
          if (lane < C::TR) bias[lane] = v0 ? log2f(mt.w0) : -INFINITY;
          if (lane + 32 < C::TR) bias[lane + 32] = v1 ? log2f(mt.w1) : -INFINITY;
        } else {
          if (p.mode == ATTN_BLOCKS) {
            const int nbv = (n + p.L - 1) / p.L;
            const int slot = mt.j0 / p.L;
            const int nk = mt.nk;
            if ((nk < 0 || nk > p.kmax) && lane == 0) atomicOr(p.status, KV_DEV_BAD_N_KEPT);
            const bool ok = slot < max(0, min(nk, p.kmax));
            if (ok && (mt.blk < 0 || mt.blk >= nbv) && lane == 0) atomicOr(p.status, KV_DEV_BAD_BLOCK_INDEX);
            if (ok && mt.blk >= 0 && mt.blk < nbv) {
              tok0 = static_cast<int64_t>(mt.blk) * p.L + (mt.j0 % p.L);
              nvalid = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(mt.rows), n - tok0)));
            }
          } else {
            tok0 = mt.j0;
            nvalid = max(0, min(mt.rows, n - mt.j0));
          }
          if (lane < C::TR) bias[lane] = lane < nvalid ? 0.f : -INFINITY;
          if (lane + 32 < C::TR) bias[lane + 32] = lane + 32 < nvalid ? 0.f : -INFINITY;
        }
        if (lane == 0) hdr[0] = nvalid;
        const uint32_t tx = (mt.first ? C::QBYTES : 0) + 2u * nvalid * C::RB;
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(full + s, tx);
        __syncwarp();
        if (mt.first && lane == 0)
          bulk_g2s(stg + C::OFF_Q, Qb + (static_cast<size_t>(b) * p.Hq + h * G) * C::RB, C::QBYTES, full + s,
                   pol);
        if (p.mode == ATTN_WEIGHTED) {
          const size_t hb = static_cast<size_t>(mt.bh) * p.Ncap;
          if (v0) {
            bulk_g2s(stg + C::OFF_K + lane * C::RB, Kb + (hb + mt.i0) * C::RB, C::RB, full + s, pol);
            bulk_g2s(stg + C::OFF_V + lane * C::RB, Vb + (hb + mt.i0) * C::RB, C::RB, full + s, pol);
          }
          if (v1) {
            bulk_g2s(stg + C::OFF_K + (lane + 32) * C::RB, Kb + (hb + mt.i1) * C::RB, C::RB, full + s, pol);
            bulk_g2s(stg + C::OFF_V + (lane + 32) * C::RB, Vb + (hb + mt.i1) * C::RB, C::RB, full + s, pol);
          }
        } else if (nvalid > 0) {
          const size_t off = (static_cast<size_t>(mt.bh) * p.Ncap + tok0) * C::RB;
          if (lane == 1) bulk_g2s(stg + C::OFF_K, Kb + off, nvalid * C::RB, full + s, pol);
          if (lane == 2) bulk_g2s(stg + C::OFF_V, Vb + off, nvalid * C::RB, full + s, pol);
        }
        fetch(mt);
      }
      if (done) break;
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int w = warp;
  const int rg = lane / C::LPR;
  const int c = lane % C::LPR;
  using HV = typename C::HV;

  if (p.mode == ATTN_BLOCKS && p.use_proxy) {
    const int64_t bh_lo = (t0 + P - 1) / P;
    const int64_t bh_hi = min(static_cast<int64_t>(p.part.NBH), (t1 + P - 1) / P);
    for (int64_t bh = bh_lo + w; bh < bh_hi; bh += C::NCW) build_proxy<T, D, G>(p, static_cast<int>(bh), lane);
  }

  float* Pw = reinterpret_cast<float*>(smem + C::OFF_P) + w * C::PW_FLOATS + rg * (C::R + 1) * C::PSTR;
  float* MA = reinterpret_cast<float*>(smem + C::OFF_MERGE);  // [NCW][G][D]
  float* MM = MA + C::NCW * G * D;                             // [NCW][G]
  float* ML = MM + C::NCW * G;                                 // [NCW][G]

  float2 qf[G][C::CH2];
  float2 acc[G][C::CH2];
  float mrun[G], lrun[G];
  auto reset_state = [&]() {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mrun[g] = -INFINITY;
      lrun[g] = 0.f;
#pragma unroll
      for (int e = 0; e < C::CH2; ++e) acc[g][e] = make_float2(0.f, 0.f);
    }
  };

  auto flush = [&](int bh) {
    // 1) merge the row groups of this warp (lanes with the same channel chunk)
#pragma unroll
    for (int mask = C::LPR; mask < 32; mask <<= 1) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mo = __shfl_xor_sync(FULL_MASK, mrun[g], mask);
        const float lo = __shfl_xor_sync(FULL_MASK, lrun[g], mask);
        const float M = fmaxf(mrun[g], mo);
        const float Ms = safe_max_ref(M);
        const float a = exp2f(mrun[g] - Ms), bw = exp2f(mo - Ms);
        lrun[g] = lrun[g] * a + lo * bw;
#pragma unroll
        for (int e = 0; e < C::CH2; ++e) {
          const float ox = __shfl_xor_sync(FULL_MASK, acc[g][e].x, mask);
          const float oy = __shfl_xor_sync(FULL_MASK, acc[g][e].y, mask);
          acc[g][e].x = acc[g][e].x * a + ox * bw;
          acc[g][e].y = acc[g][e].y * a + oy * bw;
        }
        mrun[g] = M;
      }
    }
    // 2) one row group per warp publishes its state
    if (rg == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2* dst = reinterpret_cast<float2*>(MA + (w * G + g) * D + c * C::CH);
#pragma unroll
        for (int e = 0; e < C::CH2; ++e) dst[e] = acc[g][e];
      }
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          MM[w * G + g] = mrun[g];
          ML[w * G + g] = lrun[g];
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(C::NCW * 32) : "memory");
    // 3) the four warp states -> one partial record
    float* rec = p.recs + static_cast<size_t>(cta + bh) * C::RECF;
    const int ctid = w * 32 + lane;
    for (int it = ctid; it < G * D / 4; it += C::NCW * 32) {
      const int g = it / (D / 4), d4 = it % (D / 4);
      float M = -INFINITY;
#pragma unroll
      for (int ww = 0; ww < C::NCW; ++ww) M = fmaxf(M, MM[ww * G + g]);
      const float Ms = safe_max_ref(M);
      float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int ww = 0; ww < C::NCW; ++ww) {
        const float a = exp2f(MM[ww * G + g] - Ms);
        const float4 x = *reinterpret_cast<const float4*>(MA + (ww * G + g) * D + d4 * 4);
        r.x = fmaf(a, x.x, r.x);
        r.y = fmaf(a, x.y, r.y);
        r.z = fmaf(a, x.z, r.z);
        r.w = fmaf(a, x.w, r.w);
      }
      *reinterpret_cast<float4*>(rec + g * D + d4 * 4) = r;
    }
    if (ctid < G) {
      const int g = ctid;
      float M = -INFINITY;
#pragma unroll
      for (int ww = 0; ww < C::NCW; ++ww) M = fmaxf(M, MM[ww * G + g]);
      const float Ms = safe_max_ref(M);
      float Ls = 0.f;
#pragma unroll
      for (int ww = 0; ww < C::NCW; ++ww) Ls = fmaf(exp2f(MM[ww * G + g] - Ms), ML[ww * G + g], Ls);
      rec[G * D + g] = M;
      rec[G * D + G + g] = Ls;
    }
    __threadfence();
    asm volatile("bar.sync 1, %0;" ::"n"(C::NCW * 32) : "memory");
    if (w == 0) arrive_bh<D, G>(p, bh, lane);
  };

  ChunkIter it{t0, t1};
  int cur_bh = -1;
  bool timed_out = false;
  int bh, j0, rows;
  int i = 0;
  reset_state();
#pragma unroll 1
  while (it.next(P, p.L, C::TR, p.mode, bh, j0, rows)) {
    const int s = i % C::S;
    const uint32_t phase = static_cast<uint32_t>(i / C::S) & 1u;
    const bool first = (bh != cur_bh);
    if (first) {
      if (cur_bh >= 0) flush(cur_bh);
      cur_bh = bh;
      reset_state();
    }
    if (!timed_out && !mbar_wait(full + s, phase, p.status)) timed_out = true;
    const unsigned char* stg = smem + s * C::STAGE;
    if (first) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint4 raw = lds128(stg + C::OFF_Q + g * C::RB + c * 16);
        float2 f[C::CH2];
        Chunk<T>::unpack(raw, f);
#pragma unroll
        for (int e = 0; e < C::CH2; ++e) qf[g][e] = make_float2(f[e].x * p.qscale, f[e].y * p.qscale);
      }
    }
    const int nvalid = *reinterpret_cast<const int*>(stg + C::OFF_HDR);
    if (nvalid > 0) {
      const float* bias = reinterpret_cast<const float*>(stg + C::OFF_BIAS);
      // q . k for R rows x G heads, finished by a transpose reduction
      float part[C::NV];
#pragma unroll
      for (int r = 0; r < C::R; ++r) {
        const int row = w * (C::RPW * C::R) + r * C::RPW + rg;
        const uint4 raw = lds128(stg + C::OFF_K + row * C::RB + c * 16);
        float2 kf[C::CH2];
        Chunk<T>::unpack(raw, kf);
#pragma unroll
        for (int g = 0; g < C::GP; ++g) {
          if (g < G) {
            float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < C::CH2; ++e) a2 = ffma2(qf[g][e], kf[e], a2);
            part[r * C::GP + g] = a2.x + a2.y;
          } else {
            part[r * C::GP + g] = 0.f;
          }
        }
      }
      transpose_reduce<C::NV, C::LPR / 2>(part, lane);
      // held values -> logits, chunk maxima, probabilities
#pragma unroll
      for (int j = 0; j < C::NH; ++j) {
        const int vi = HV::index(c, j);
        const int ri = vi / C::GP, g = vi % C::GP;
        const int row = w * (C::RPW * C::R) + ri * C::RPW + rg;
        float sj = g < G ? part[j] + bias[row] : -INFINITY;
        float cm = sj;
#pragma unroll
        for (int mask = HV::ROW_MASK_LO; mask < C::LPR; mask <<= 1)
          cm = fmaxf(cm, __shfl_xor_sync(FULL_MASK, cm, mask));
        float mold = mrun[0];
#pragma unroll
        for (int gg = 1; gg < G; ++gg)
          if (g == gg) mold = mrun[gg];
        const float mnew = fmaxf(mold, cm);
        const float pj = exp2f(sj - safe_max_ref(mnew));
        if (g < G) {
          Pw[ri * C::PSTR + g] = pj;
          Pw[C::R * C::PSTR + g] = mnew;
        }
      }
      __syncwarp();
      // rescale, then accumulate p * v
      float sc[G];
      {
        float mn[C::PSTR];
#pragma unroll
        for (int g4 = 0; g4 < C::PSTR; g4 += 4) {
          const float4 x = *reinterpret_cast<const float4*>(Pw + C::R * C::PSTR + g4);
          mn[g4] = x.x;
          mn[g4 + 1] = x.y;
          mn[g4 + 2] = x.z;
          mn[g4 + 3] = x.w;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          sc[g] = exp2f(mrun[g] - safe_max_ref(mn[g]));
          mrun[g] = mn[g];
          lrun[g] *= sc[g];
#pragma unroll
          for (int e = 0; e < C::CH2; ++e) acc[g][e] = fmul2(acc[g][e], make_float2(sc[g], sc[g]));
        }
      }
#pragma unroll
      for (int r = 0; r < C::R; ++r) {
        const int row = w * (C::RPW * C::R) + r * C::RPW + rg;
        const uint4 raw = lds128(stg + C::OFF_V + row * C::RB + c * 16);
        float2 vf[C::CH2];
        Chunk<T>::unpack(raw, vf);
        float pr[C::PSTR];
#pragma unroll
        for (int g4 = 0; g4 < C::PSTR; g4 += 4) {
          const float4 x = *reinterpret_cast<const float4*>(Pw + r * C::PSTR + g4);
          pr[g4] = x.x;
          pr[g4 + 1] = x.y;
          pr[g4 + 2] = x.z;
          pr[g4 + 3] = x.w;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          lrun[g] += pr[g];
          const float2 pp = make_float2(pr[g], pr[g]);
#pragma unroll
          for (int e = 0; e < C::CH2; ++e) acc[g][e] = ffma2(pp, vf[e], acc[g][e]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + s);
    ++i;
  }
  if (cur_bh >= 0) flush(cur_bh);
  if (timed_out) {
    // Give copies that may still be in flight a last bounded chance to land
    // before this CTA's shared memory is released.
    for (int s = 0; s < C::S; ++s) {
      const int last_use = (i - 1 - s) >= 0 ? (i - 1 - s) / C::S : -1;
      if (last_use >= 0) mbar_wait(full + ((i - 1 - s) % C::S), static_cast<uint32_t>(last_use) & 1u, nullptr);
    }
  }
}

}  // namespace kvs
