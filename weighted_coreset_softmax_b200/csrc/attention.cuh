// Split-K gather attention for decode: exact softmax attention over the kept
// blocks' tokens plus the count-aware tail proxy (block mode), over a weighted
// coreset (weighted mode), or over every cached token (dense mode).
//
// Method sources:
//  * "OpenAttention reads 1% of the KV cache -- Count-aware tail proxy", section
//    "Skipping reviews without losing the verdict": the unread tail enters the
//    softmax as one token whose value is the tail's mean value and whose logit is
//    its mean logit plus ln(count); it has the form of an ordinary token, so here
//    it is one more partial result merged with the others.
//  * "WildCat: Near-Linear Attention in Theory and Practice", abstract: weighted
//    coreset attention, logit + ln w_i.
//  * "COBS: Cumulant Order Block Sparse Attention", read-traffic accounting:
//    dense attention reads the whole cache.
//
// Design (sm_100a). All (sequence, KV head) pairs ("bh") lay their P token slots
// end to end on one axis; the launch cuts that axis into equal contiguous ranges,
// one per warp ("worker"), so every SM streams the same bytes whatever the
// per-head work. A worker walks its range in chunks of TR rows that stay inside
// one bh (and, in block mode, one kept block). Each worker is an independent
// pipeline: it moves its chunks' K and V (and, at the start of a bh, the group's
// q) into its own two-slot shared-memory ring with bulk copies, tracked by its
// own mbarriers, and refills a slot as soon as it has consumed it; the per-chunk
// indices are loaded 32 chunks at a time, one batch ahead.
//  q.k: four lanes share a group of two tokens (each lane reads a quarter of
//  each row); q is held once per warp in fp32, prescaled by scale*log2(e), split
//  into two 16-byte planes per chunk; every lane visits its row chunks in a
//  rotated order chosen so that the eight lanes of each quarter-warp (the unit
//  in which 16-byte shared loads are served) hit eight different bank groups,
//  for the K rows and for q alike; packed f32x2 FMAs; a 4-lane all-reduce
//  finishes the dots and the first two lanes of each group then own one token's
//  logits each.
//  softmax: per warp, in the log2 domain; the running maximum is uniform across
//  the warp, so partial states merge without rescaling.
//  p.v: lanes own 16-byte channel chunks of V rows, packed f32x2 FMAs.
// For bf16 caches in block and dense modes a tensor-core consumer replaces the
// CUDA-core one: warp-chunks of 32 rows move with tiled tensor copies (two boxes
// of 32 rows x 128 bytes per tensor for d = 128) into 128-byte-swizzled tiles, so
// the 8x8 ldmatrix reads are conflict-free; q.k is mma.sync m16n8k16 with the 16
// tokens of a tile as M and the G <= 8 query heads as N (q^T fragments stay in
// registers for the whole bh), so the bf16 products are exact and accumulate in
// fp32; the softmax runs on the accumulator fragments; P is split into a bf16
// high part and a bf16 remainder (about 16 significant bits together), moved
// into B-operand layout with movmatrix, and p.v is two mma.sync per 16x16 tile of
// V^T. The q.k and p.v of a kept token then cost a few instructions instead of
// a few dozen, which leaves the kernel bound by HBM rather than by issue.
// When a warp's chunk sequence leaves a bh it writes one partial record
// (acc, m, l) to the workspace and takes an arrival ticket for that bh; the last
// arriver merges all records of the bh (and the proxy record) into the output.
// No warp ever waits for another.
#pragma once

#include <cuda.h>

#include <climits>

#include "common.cuh"
#include "rank.cuh"

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
  int B, Hq, Hkv, Ncap, L, log2L, NBcap;
  int mode;
  int use_proxy;
  float qscale;  // softmax scale * log2(e): logits are kept in the log2 domain
  Partition part;
  // fused decode step only: block selection inside the CTA (summary scoring)
  int k_top, force_first, force_last;
  int32_t* sel_block_idx;  // the selection's outputs (block_idx / n_kept above alias them)
  int32_t* sel_n_kept;
  float* sel_scores;       // optional [B][Hkv][NBcap]
};

// Shape constants of one instantiation. MMA selects the tensor-core consumer
// (bf16 caches, block and dense modes): 32 rows per warp-chunk, K and V moved by
// tiled tensor copies into 128-byte-swizzled tiles; otherwise the CUDA-core
// consumer: 16 rows per warp-chunk in dense rows.
template <typename T, int D, int G, bool MMA>
struct AttnCfg {
  static constexpr int ES = sizeof(T);
  static constexpr int RB = D * ES;          // bytes per cached row
  static constexpr int CPR = RB / 16;        // 16-byte chunks per row
  static constexpr int CH = 16 / ES;         // elements per chunk
  static constexpr int CH2 = CH / 2;         // float2 pairs per chunk
  static constexpr int LPT = 4;              // lanes per token group (CUDA-core q.k)
  static constexpr int CPL = CPR / LPT;      // chunks per lane per row (CUDA-core q.k)
  static constexpr int TPL = 2;              // tokens per token group (CUDA-core q.k)
  static constexpr int TPW = MMA ? 32 : 8 * TPL;  // rows per warp per chunk
  static constexpr int NW = ATTN_NW;         // worker warps per CTA
  static constexpr int NTHREADS = (NW + 1) * 32;  // + one helper warp (tail proxies, merges)
  static constexpr int TR = TPW;             // rows per chunk (one worker)
  static constexpr int VR = 32 / CPR;        // V rows per p.v step (CUDA-core)
  static constexpr int KS = D / 16;          // k-steps of q.k and d-tiles of p.v (MMA)
  static constexpr int KH = MMA ? RB / 128 : 1;   // 128-byte column boxes per row (MMA)
  static constexpr int BOX = TPW * 128;      // bytes of one swizzled box (MMA)
  static constexpr int QPL = CH / 4;         // 16-byte planes of fp32 q per chunk
  static constexpr int QPLANE = CPR * 16;    // bytes of one plane of one head
  static constexpr int QHEAD = QPL * QPLANE; // bytes of one head of q (fp32)
  static constexpr int QBYTES = G * RB;      // q of one KV head's group, input type
  static constexpr int PSTR = G <= 4 ? 4 : 8;
  // one ring slot: K rows | V rows | raw q | bias | header (1024-byte aligned
  // for the swizzled tiles)
  static constexpr int SL_K = 0;
  static constexpr int SL_V = TPW * RB;
  static constexpr int SL_Q = 2 * TPW * RB;
  static constexpr int SL_BIAS = SL_Q + QBYTES;
  static constexpr int SL_HDR = SL_BIAS + TPW * 4;
  static constexpr int SLOT = MMA ? (SL_HDR + 16 + 1023) & ~1023 : (SL_HDR + 16 + 127) & ~127;
  // ring slots per worker: three where two CTAs of three-slot workers still fit
  // in an SM's 228 KB (1 KB of it reserved per CTA), else two
  static constexpr int S = (MMA && 2 * (NW * (3 * SLOT + 1024) + 1024 + 1024) <= 228 * 1024) ? 3 : 2;
  // one warp: S slots | q fp32 | p | barriers (q fp32 and p: CUDA-core only)
  static constexpr int W_Q = S * SLOT;
  static constexpr int W_P = W_Q + (MMA ? 0 : G * QHEAD);
  static constexpr int W_BAR = W_P + (MMA ? 0 : TPW * PSTR * 4);
  static constexpr int W_BYTES = MMA ? (W_BAR + S * 8 + 1023) & ~1023 : (W_BAR + S * 8 + 127) & ~127;
  static constexpr int ALIGN_SLACK = MMA ? 1024 : 0;
  static constexpr int CTA_EXTRA = 64;      // per-CTA: the workers' record-ready barriers
  static constexpr int SMEM = NW * W_BYTES + CTA_EXTRA + ALIGN_SLACK;
  static constexpr int RECF = (G * D + 2 * G + 3) & ~3;
  static_assert(MMA || CPL == 2 || CPL == 4 || CPL == 8, "chunks per lane");
  static_assert(MMA || (VR >= 1 && 32 % CPR == 0 && TPW % VR == 0), "p.v row layout");
  static_assert(!MMA || (ES == 2 && G <= 8 && RB % 128 == 0), "tensor-core consumer: bf16, G <= 8");
  static_assert(TPW <= 32, "one row per lane when issuing copies");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  // CUDA-core q.k: rotation of the chunk a lane reads at step st. Within a
  // quarter-warp the lanes are (ts & 1) x pq; rows sit 128-byte aligned, so the
  // bank group of chunk c is c mod 8 -- this choice gives the eight lanes eight
  // different groups.
  __device__ __forceinline__ static int chunk_at(int st, int ts, int pq) {
    const int rot = CPL == 2 ? 0 : (CPL == 4 ? 2 * (pq >> 1) : 2 * pq);
    return pq * CPL + ((st + (ts & 1) + rot) & (CPL - 1));
  }
  // Tensor core: byte offset of 16-byte chunk c of row r in a slot's K or V
  // tiles (128-byte swizzle: chunk c of a 128-byte line sits at c ^ (r mod 8)).
  __device__ __forceinline__ static int swz(int r, int c) {
    return (c >> 3) * BOX + r * 128 + (((c & 7) ^ (r & 7)) << 4);
  }
};

// ---- tensor-core helpers (warp-wide, bf16 operands, fp32 accumulate)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma_bf16(float& d0, float& d1, float& d2, float& d3, const uint32_t (&a)[4],
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// two floats -> bf16x2 (lo in the low half), round to nearest
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float safe_max_ref(float m) { return m == -INFINITY ? 0.f : m; }

// Walks [cur, end) of the token axis in chunks that stay inside one bh, hold at
// most TR rows and, in block mode, stay inside one kept block. Incremental: no
// division after init.
struct ChunkIter {
  int64_t cur, end;
  int bh, j0;
  __device__ __forceinline__ void init(int64_t t0, int64_t t1, int P) {
    cur = t0;
    end = t1;
    bh = t0 <= 0x7fffffff ? static_cast<int>(static_cast<unsigned>(t0) / static_cast<unsigned>(P))
                          : static_cast<int>(t0 / P);
    j0 = static_cast<int>(t0 - static_cast<int64_t>(bh) * P);
  }
  __device__ __forceinline__ bool next(int P, int L, int TR, int mode, int& obh, int& oj0, int& rows) {
    if (cur >= end) return false;
    int r = P - j0;
    const int64_t left = end - cur;
    if (left < r) r = static_cast<int>(left);
    if (r > TR) r = TR;
    if (mode == ATTN_BLOCKS) r = min(r, L - (j0 & (L - 1)));
    obh = bh;
    oj0 = j0;
    rows = r;
    cur += r;
    j0 += r;
    if (j0 == P) {
      ++bh;
      j0 = 0;
    }
    return true;
  }
};

// What a warp needs to issue one chunk's copies. Held one chunk per lane, a
// batch of 32 chunks at a time.
struct ChunkMeta {
  int has, bh, j0, rows, first;
  int n;       // seq_len of the sequence
  int nk;      // block mode: n_kept of the bh
  int blk;     // block mode: block index of the chunk's slot
};

__device__ __forceinline__ int first_worker(const Partition& pt, int bh) {
  return part_worker_of(pt, static_cast<int64_t>(bh) * pt.P);
}
__device__ __forceinline__ int last_worker(const Partition& pt, int bh) {
  return part_worker_of(pt, static_cast<int64_t>(bh) * pt.P + pt.P - 1);
}

// Merges every partial record of one bh into out / lse. One warp. With at most
// R records (the usual case: a bh spans a few workers, plus the proxy) each
// lane requests its channels of all of them together with the records' maxima
// and sums, so the merge costs one memory round trip; more records are folded
// 32 at a time (maxima and sums by one lane each, then the channels streamed).
template <int D, int G>
__device__ void finalize_bh(const AttnParams& p, int bh, int lane) {
  constexpr int RECF = (G * D + 2 * G + 3) & ~3;
  constexpr int VEC = D / 32;
  constexpr int R = G <= 4 ? 4 : 2;
  const int cf = first_worker(p.part, bh), cl = last_worker(p.part, bh);
  const int nattn = cl - cf + 1;
  const int nrec = nattn + (p.use_proxy ? 1 : 0);
  const int b = bh / p.Hkv, h = bh - (bh / p.Hkv) * p.Hkv;
  const float* base = p.recs + static_cast<size_t>(cf + bh) * RECF;
  auto rec_ptr = [&](int j) -> const float* {
    return j < nattn ? base + static_cast<size_t>(j) * RECF : p.proxy_recs + static_cast<size_t>(bh) * RECF;
  };
  auto load_vec = [&](const float* r, float (&x)[VEC]) {
    if constexpr (VEC == 4) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(r));
      x[0] = f.x;
      x[1] = f.y;
      x[2] = f.z;
      x[3] = f.w;
    } else {
#pragma unroll
      for (int v = 0; v < VEC; ++v) x[v] = __ldcg(r + v);
    }
  };
  float* o = p.out + (static_cast<size_t>(b) * p.Hq + h * G) * D + lane * VEC;
  float Mg[G], Lg[G], acc[G][VEC];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    Mg[g] = -INFINITY;
    Lg[g] = 0.f;
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[g][v] = 0.f;
  }
  if (nrec <= R) {
    float x[R][G][VEC];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (r < nrec) {
          load_vec(rec_ptr(r) + g * D + lane * VEC, x[r][g]);
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) x[r][g][v] = 0.f;
        }
      }
    float mj[G], lj[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mj[g] = lane < nrec ? __ldcg(rec_ptr(lane) + G * D + g) : -INFINITY;
      lj[g] = lane < nrec ? __ldcg(rec_ptr(lane) + G * D + G + g) : 0.f;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      Mg[g] = warp_max(mj[g]);
      const float wj = fast_exp2(mj[g] - safe_max_ref(Mg[g]));
      Lg[g] = warp_sum(wj * lj[g]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float wr = __shfl_sync(FULL_MASK, wj, r);
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[g][v] = fmaf(wr, x[r][g][v], acc[g][v]);
      }
    }
  } else {
    for (int j0 = 0; j0 < nrec; j0 += 32) {
      const int j = j0 + lane;
      float mj[G], lj[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        mj[g] = j < nrec ? __ldcg(rec_ptr(j) + G * D + g) : -INFINITY;
        lj[g] = j < nrec ? __ldcg(rec_ptr(j) + G * D + G + g) : 0.f;
      }
      float wj[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float Mn = fmaxf(Mg[g], warp_max(mj[g]));
        const float Ms = safe_max_ref(Mn);
        const float rescale = fast_exp2(Mg[g] - Ms);
        wj[g] = fast_exp2(mj[g] - Ms);
        Lg[g] = Lg[g] * rescale + warp_sum(wj[g] * lj[g]);
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[g][v] *= rescale;
        Mg[g] = Mn;
      }
      const int cnt = min(32, nrec - j0);
#pragma unroll 4
      for (int k = 0; k < cnt; ++k) {
        const float* r = rec_ptr(j0 + k) + lane * VEC;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float wk = __shfl_sync(FULL_MASK, wj[g], k);
          float x[VEC];
          load_vec(r + g * D, x);
#pragma unroll
          for (int v = 0; v < VEC; ++v) acc[g][v] = fmaf(wk, x[v], acc[g][v]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float inv = Lg[g] > 0.f ? 1.f / Lg[g] : 0.f;
#pragma unroll
    for (int v = 0; v < VEC; ++v) o[g * D + v] = acc[g][v] * inv;
    if (p.lse && lane == 0)
      p.lse[static_cast<size_t>(b) * p.Hq + h * G + g] = Lg[g] > 0.f ? (Mg[g] + log2f(Lg[g])) * LN2 : -INFINITY;
  }
}

// Arrival ticket for bh; the last arriver merges. Called by one whole warp after
// its record writes are complete and fenced.
template <int D, int G>
__device__ __forceinline__ void arrive_bh(const AttnParams& p, int bh, int lane) {
  int last = 0;
  if (lane == 0) {
    const int E = (last_worker(p.part, bh) - first_worker(p.part, bh) + 1) + (p.use_proxy ? 1 : 0);
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

// The tail proxy of one bh: this lane's VEC channels of its value (the mean
// unread value) and the G log2 logits (q_g . mean unread key * scale*log2(e) +
// log2 of the unread count; -inf with no unread token). One warp. All kept
// block indices are read in one round trip and the key/value sums of the kept
// blocks are then requested together, so the proxy costs two dependent memory
// round trips (up to 32 kept blocks).
template <typename T, int D, int G>
__device__ void proxy_values(const AttnParams& p, int bh, int lane, float (&vb)[D / 32], float (&pm)[G]) {
  constexpr int VEC = D / 32;
  constexpr int UNR = 8;  // kept blocks whose sums are in flight together
  const int b = bh / p.Hkv, h = bh - (bh / p.Hkv) * p.Hkv;
  // independent first loads: length, count, indices, q, totals
  int n = p.seq_lens[b];
  int nk = p.n_kept[bh];
  const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * D;
  float qv[G][VEC];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int v = 0; v < VEC; ++v) qv[g][v] = load_as_float(qrow + g * D + lane * VEC + v);
  float kt[VEC], vt[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    kt[v] = p.k_tot[static_cast<size_t>(bh) * D + lane * VEC + v];
    vt[v] = p.v_tot[static_cast<size_t>(bh) * D + lane * VEC + v];
  }
  if (n < 0 || n > p.Ncap) {
    if (lane == 0) atomicOr(p.status, KV_DEV_BAD_SEQ_LEN);
    n = max(0, min(n, p.Ncap));
  }
  if (nk < 0 || nk > p.kmax) {
    if (lane == 0) atomicOr(p.status, KV_DEV_BAD_N_KEPT);
    nk = max(0, min(nk, p.kmax));
  }
  const int nbv = (n + p.L - 1) >> p.log2L;
  float ks[VEC], vs[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) ks[v] = vs[v] = 0.f;
  int cnt = 0;
  int prev_last = -1;  // last block index of the previous group of 32
  // the first 32 index slots are read before n_kept is known (they are in bounds)
  const int first32 = lane < p.kmax ? p.block_idx[static_cast<size_t>(bh) * p.kmax + lane] : INT_MAX;
  for (int s0 = 0; s0 < nk; s0 += 32) {
    int mine = s0 == 0 ? first32 : ((s0 + lane < nk) ? p.block_idx[static_cast<size_t>(bh) * p.kmax + s0 + lane] : INT_MAX);
    if (s0 + lane >= nk) mine = INT_MAX;
    // a kept index must lie in [0, nbv) and exceed the one before it
    int before = __shfl_up_sync(FULL_MASK, mine, 1);
    if (lane == 0) before = prev_last;
    const bool in_list = s0 + lane < nk;
    const bool ok = in_list && mine >= 0 && mine < nbv && mine > before;
    if (__any_sync(FULL_MASK, in_list && !ok) && lane == 0) atomicOr(p.status, KV_DEV_BAD_BLOCK_INDEX);
    const unsigned okmask = __ballot_sync(FULL_MASK, ok);
    prev_last = __shfl_sync(FULL_MASK, mine, 31);
    // the counts of this group of kept blocks, one per lane
    int c = ok ? p.counts[static_cast<size_t>(b) * p.NBcap + mine] : 0;
    c = __reduce_add_sync(FULL_MASK, c);
    cnt += c;
    const int lim = min(32, nk - s0);
    for (int j0 = 0; j0 < lim; j0 += UNR) {
      float kr[UNR][VEC], vr[UNR][VEC];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u;
        const int blk = __shfl_sync(FULL_MASK, mine, j & 31);
        const bool use = j < lim && ((okmask >> (j & 31)) & 1u);
        const size_t row = (static_cast<size_t>(bh) * p.NBcap + (use ? blk : 0)) * D + lane * VEC;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          kr[u][v] = use ? p.k_sum[row + v] : 0.f;
          vr[u][v] = use ? p.v_sum[row + v] : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u)
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          ks[v] += kr[u][v];
          vs[v] += vr[u][v];
        }
    }
  }
  const int nT = n - cnt;
  if (nT > 0) {
    const float inv = 1.f / static_cast<float>(nT);
    float kb[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      kb[v] = (kt[v] - ks[v]) * inv;
      vb[v] = (vt[v] - vs[v]) * inv;
    }
    const float lc = log2f(static_cast<float>(nT));
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float d = 0.f;
#pragma unroll
      for (int v = 0; v < VEC; ++v) d = fmaf(qv[g][v], kb[v], d);
      pm[g] = d;
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
      for (int g = 0; g < G; ++g) pm[g] += __shfl_xor_sync(FULL_MASK, pm[g], m);
#pragma unroll
    for (int g = 0; g < G; ++g) pm[g] = pm[g] * p.qscale + lc;
  } else {
#pragma unroll
    for (int v = 0; v < VEC; ++v) vb[v] = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) pm[g] = -INFINITY;
  }
}

// The tail proxy as one more partial record of the bh (m = its logit, l = 1,
// acc = its value) in the workspace, followed by its arrival ticket.
template <typename T, int D, int G>
__device__ void build_proxy(const AttnParams& p, int bh, int lane) {
  constexpr int RECF = (G * D + 2 * G + 3) & ~3;
  constexpr int VEC = D / 32;
  float vb[VEC], pm[G];
  proxy_values<T, D, G>(p, bh, lane, vb, pm);
  float* rec = p.proxy_recs + static_cast<size_t>(bh) * RECF;
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) rec[g * D + lane * VEC + v] = pm[g] == -INFINITY ? 0.f : vb[v];
    if (lane == 0) {
      rec[G * D + g] = pm[g];
      rec[G * D + G + g] = pm[g] == -INFINITY ? 0.f : 1.f;
    }
  }
  __threadfence();
  __syncwarp();
  arrive_bh<D, G>(p, bh, lane);
}

// Merge of one bh whose partial records all live in this CTA: nw records in
// shared memory (written by the workers, layout as in the workspace) and the
// proxy held in registers (pm = -inf: none). One warp.
template <int D, int G>
__device__ void merge_local(const AttnParams& p, int bh, int lane, const float* const* recs, int nw,
                            const float (&vb)[D / 32], const float (&pm)[G]) {
  constexpr int VEC = D / 32;
  const int b = bh / p.Hkv, h = bh - (bh / p.Hkv) * p.Hkv;
  float* o = p.out + (static_cast<size_t>(b) * p.Hq + h * G) * D + lane * VEC;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float M = pm[g];
    for (int j = 0; j < nw; ++j) M = fmaxf(M, recs[j][G * D + g]);
    const float Ms = safe_max_ref(M);
    const float wp = fast_exp2(pm[g] - Ms);
    float Lsum = pm[g] == -INFINITY ? 0.f : wp;
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = pm[g] == -INFINITY ? 0.f : wp * vb[v];
    for (int j = 0; j < nw; ++j) {
      const float wj = fast_exp2(recs[j][G * D + g] - Ms);
      Lsum = fmaf(wj, recs[j][G * D + G + g], Lsum);
      const float* r = recs[j] + g * D + lane * VEC;
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = fmaf(wj, r[v], acc[v]);
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll
    for (int v = 0; v < VEC; ++v) o[g * D + v] = acc[v] * inv;
    if (p.lse && lane == 0)
      p.lse[static_cast<size_t>(b) * p.Hq + h * G + g] = Lsum > 0.f ? (M + log2f(Lsum)) * LN2 : -INFINITY;
  }
}

// Selection phase of the fused decode step: one CTA holds one bh (its workers
// split the bh's kept tokens later). Summary scoring of every block ("COBS:
// Cumulant Order Block Sparse Attention", text after Equation (8): the mean-pool
// estimate s = q . k_mean + ln n_b), then the Eq. 5 ranking. The workers stream
// the bh's fp32 key-sum rows through their ring slots (32 rows a slot, bulk
// copies, chunks interleaved between the workers) and write the block logits
// into worker 0's last slot; the helper loads the block counts; keys, counts and
// the ranking's scratch live in worker 1's last slot (those two slots do not
// stream). Every warp of the CTA calls this once (same barrier sequence);
// afterwards block_idx / n_kept of the bh are in global memory, visible to the
// whole CTA, and the workers' ring barriers are fresh.
template <typename T, int D, int G, typename C>
__device__ void fused_select(const AttnParams& p, unsigned char* smem, int bh, int warp, int lane, uint64_t pol) {
  constexpr int LPR = D / 4;            // lanes per fp32 row (float4 each)
  constexpr int RPW = 32 / LPR;         // rows one warp load covers
  constexpr int GR = 8;                 // rows per reduction group
  constexpr int RS = GR / RPW;          // rows per lane per group
  constexpr int GP = pow2ceil(G);
  constexpr int NV = RS * GP;
  constexpr int ROWB = D * 4;
  constexpr int CROWS = 2 * C::TPW * C::RB / ROWB;  // rows in a slot's K+V region (32)
  using HV = HeldValues<NV, LPR, GP>;
  static_assert(CROWS % GR == 0 && C::NW >= 2, "fused selection layout");
  {
  const int b = bh / p.Hkv, h = bh - (bh / p.Hkv) * p.Hkv;
  const int n = max(0, min(p.seq_lens[b], p.Ncap));
  const int nbv = (n + p.L - 1) >> p.log2L;
  const int nbp = (p.NBcap + 31) & ~31;
  float* lg = reinterpret_cast<float*>(smem + (C::S - 1) * C::SLOT);  // worker 0, last slot
  unsigned char* x1 = smem + C::W_BYTES + (C::S - 1) * C::SLOT;       // worker 1, last slot
  unsigned long long* key = reinterpret_cast<unsigned long long*>(x1);
  int* cnt = reinterpret_cast<int*>(x1 + static_cast<size_t>(nbp) * 8);
  RankMisc<C::NTHREADS>& ms = *reinterpret_cast<RankMisc<C::NTHREADS>*>(x1 + ((static_cast<size_t>(nbp) * 12 + 15) & ~15));
  const int nch = (nbv + CROWS - 1) / CROWS;
  unsigned char* wb = smem + warp * C::W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(wb + C::W_BAR);
  const float* ks = p.k_sum + static_cast<size_t>(bh) * p.NBcap * D;
  const int nslots = warp < 2 ? C::S - 1 : C::S;  // streaming slots of this worker
  auto issue = [&](int c, int s) {  // chunk c into slot s (lane 0)
    const int rows = min(CROWS, nbv - c * CROWS);
    const uint32_t bytes = static_cast<uint32_t>(rows * ROWB);
    mbar_arrive_expect_tx(bars + s, bytes);
    bulk_g2s(wb + s * C::SLOT, ks + static_cast<size_t>(c) * CROWS * D, bytes, bars + s, pol);
  };
  const int rg = lane / LPR, c4 = lane % LPR;
  float4 qf[G];
  if (warp == C::NW) {
    const int32_t* cn = p.counts + static_cast<size_t>(b) * p.NBcap;
    for (int i = lane; i < nbv; i += 32) cnt[i] = cn[i];
  } else {
    if (lane == 0)
      for (int j = 0; j < nslots && warp + j * C::NW < nch; ++j) issue(warp + j * C::NW, j);
    const T* qrow = static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.Hq + h * G) * D + c4 * 4;
#pragma unroll
    for (int g = 0; g < G; ++g)
      qf[g] = make_float4(load_as_float(qrow + g * D) * p.qscale, load_as_float(qrow + g * D + 1) * p.qscale,
                          load_as_float(qrow + g * D + 2) * p.qscale, load_as_float(qrow + g * D + 3) * p.qscale);
  }
  __syncthreads();  // counts
  if (warp < C::NW) {
    bool ok = true;
    int j = 0;
    for (int c = warp; c < nch; c += C::NW, ++j) {
      const int s = j % nslots;
      if (ok && !mbar_wait(bars + s, static_cast<uint32_t>(j / nslots) & 1u, p.status)) ok = false;
      const float* chunk = reinterpret_cast<const float*>(wb + s * C::SLOT);
#pragma unroll 1
      for (int g0 = 0; g0 < CROWS; g0 += GR) {
        float part[NV];
#pragma unroll
        for (int i = 0; i < RS; ++i) {
          const int lr = g0 + i * RPW + rg;
          const float4 k4 = c * CROWS + lr < nbv ? *reinterpret_cast<const float4*>(chunk + lr * D + c4 * 4)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
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
        for (int jj = 0; jj < HV::NH; ++jj) {
          const int vi = HV::index(c4, jj);
          const int ri = vi / GP, g = vi % GP;
          const int row = c * CROWS + g0 + ri * RPW + rg;
          const bool holder = NV >= LPR || (c4 % (NV >= LPR ? 1 : LPR / NV)) == 0;
          if (holder && g < G && row < nbv) {
            const int nb = cnt[row];
            lg[g * nbp + row] =
                nb > 0 ? part[jj] / static_cast<float>(nb) + log2f(static_cast<float>(nb)) : -INFINITY;
          }
        }
      }
      __syncwarp();
      fence_proxy_async_smem();  // the slot is refilled by the async proxy
      if (lane == 0 && ok && c + nslots * C::NW < nch) issue(c + nslots * C::NW, s);
    }
    // fresh ring barriers for the attention phase (every copy above was consumed)
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < C::S; ++s) {
        mbar_inval(bars + s);
        mbar_init(bars + s, 1);
      }
      fence_mbar_init();
    }
    __syncwarp();
  }
  __syncthreads();  // every block logit is in lg
  rank_in_cta<G, C::NTHREADS>(lg, nbp, nbv, p.NBcap, p.k_top, p.force_first != 0, p.force_last != 0, p.kmax,
                              p.sel_scores ? p.sel_scores + static_cast<size_t>(bh) * p.NBcap : nullptr,
                              p.sel_block_idx + static_cast<size_t>(bh) * p.kmax, p.sel_n_kept + bh, key, ms);
  __syncthreads();  // the kept list is written (visible to this CTA) and the scratch is free
  }
}

template <typename T, int D, int G, bool MMA, bool FUSED>
__global__ void __launch_bounds__(AttnCfg<T, D, G, MMA>::NTHREADS)
    attn_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  using C = AttnCfg<T, D, G, MMA>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // swizzled tiles need 1024-byte alignment
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u) * (MMA ? 1 : 0);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int P = p.part.P;
  constexpr int VEC = D / 32;
  // Worker ranges of this CTA. When the CTA's range starts and ends on bh
  // boundaries and each worker's range lies inside one bh ("local" CTA), every
  // partial record of those bh is produced here: the workers leave their
  // records in shared memory and the helper warp merges them with the proxy,
  // with no workspace round trip, fence or ticket.
  int64_t wa[C::NW + 1];
#pragma unroll
  for (int w = 0; w <= C::NW; ++w) wa[w] = part_t0(p.part, blockIdx.x * C::NW + w);
  auto bh_of = [&](int64_t x) -> int64_t {
    return p.part.TT <= 0x7fffffff ? static_cast<int64_t>(static_cast<unsigned>(x) / static_cast<unsigned>(P)) : x / P;
  };
  bool local = bh_of(wa[0]) * P == wa[0] && bh_of(wa[C::NW]) * P == wa[C::NW];
#pragma unroll
  for (int w = 0; w < C::NW; ++w)
    if (wa[w] < wa[w + 1] && bh_of(wa[w]) != bh_of(wa[w + 1] - 1)) local = false;
  uint64_t* ready = reinterpret_cast<uint64_t*>(smem + C::NW * C::W_BYTES);
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 0; w < C::NW; ++w) mbar_init(ready + w, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == C::NW) {
    // helper warp: the tail proxies of the bh whose first token lies in this
    // CTA's range, built while the workers stream (its memory round trips stay
    // off their critical path); in a local CTA also the final merges
    grid_dep_wait();
    if constexpr (FUSED) fused_select<T, D, G, C>(p, smem, static_cast<int>(bh_of(wa[0])), warp, lane, 0ull);
    const int64_t bh_lo = bh_of(wa[0] + P - 1);
    const int64_t bh_hi = min(static_cast<int64_t>(p.part.NBH), bh_of(wa[C::NW] + P - 1));
    const bool proxy = p.mode == ATTN_BLOCKS && p.use_proxy;
    if (local) {
      for (int64_t pbh = bh_lo; pbh < bh_hi; ++pbh) {
        float vb[VEC], pm[G];
        if (proxy) {
          proxy_values<T, D, G>(p, static_cast<int>(pbh), lane, vb, pm);
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) vb[v] = 0.f;
#pragma unroll
          for (int g = 0; g < G; ++g) pm[g] = -INFINITY;
        }
        const float* recs[C::NW];
        int nw = 0;
#pragma unroll
        for (int w = 0; w < C::NW; ++w)
          if (wa[w] < wa[w + 1] && bh_of(wa[w]) == pbh) recs[nw++] = reinterpret_cast<const float*>(smem + w * C::W_BYTES);
        // a first pass of the merge over whatever the slots hold now, while the
        // workers stream: it brings the merge's instructions into the SM's
        // instruction cache off the critical path (the merge runs once a launch,
        // so it would otherwise start cold); the merge after the waits rewrites
        // every output this pass writes, in this thread
        merge_local<D, G>(p, static_cast<int>(pbh), lane, recs, nw, vb, pm);
#pragma unroll
        for (int w = 0; w < C::NW; ++w)
          if (wa[w] < wa[w + 1] && bh_of(wa[w]) == pbh) mbar_wait(ready + w, 0u, p.status);
        merge_local<D, G>(p, static_cast<int>(pbh), lane, recs, nw, vb, pm);
      }
    } else if (proxy) {
      for (int64_t pbh = bh_lo; pbh < bh_hi; ++pbh) build_proxy<T, D, G>(p, static_cast<int>(pbh), lane);
    }
    return;
  }
  const int wk = blockIdx.x * C::NW + warp;  // this worker
  const int64_t t0 = wa[warp];
  const int64_t t1 = wa[warp + 1];
  unsigned char* wb = smem + warp * C::W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(wb + C::W_BAR);
  float* q32 = reinterpret_cast<float*>(wb + C::W_Q);
  float* pbuf = reinterpret_cast<float*>(wb + C::W_P);

  if (lane == 0) {
    if constexpr (MMA) {
      prefetch_tensor_map(&tmK);
      prefetch_tensor_map(&tmV);
    }
#pragma unroll
    for (int s = 0; s < C::S; ++s) mbar_init(bars + s, 1);
    fence_mbar_init();
  }
  if constexpr (!MMA) {
    // Rows a chunk does not fill keep stale (finite) data; zero the ring once so
    // that no uninitialised pattern is ever multiplied by p = 0. (The tiled
    // copies of the tensor-core consumer always fill whole boxes.)
    for (int i = lane; i < C::S * C::SLOT / 16; i += 32) reinterpret_cast<uint4*>(wb)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  __syncwarp();

  const uint64_t pol = l2_evict_first_policy();
  const unsigned char* Kg = static_cast<const unsigned char*>(p.K);
  const unsigned char* Vg = static_cast<const unsigned char*>(p.V);
  const unsigned char* Qg = static_cast<const unsigned char*>(p.q);

  // ---- chunk metadata, 32 chunks per batch (lane j holds chunk j) ---------
  // Each lane finds its own chunk and loads that chunk's sequence length, kept
  // count and block index, so one memory round trip covers the next 32 copies.
  // When every chunk has the same TE rows (P a multiple of TE; ranges start on
  // multiples of 32) chunk j starts at the batch start + j TE, one division per
  // lane; otherwise each lane walks the chunk sequence up to its chunk.
  const int TE = (p.mode == ATTN_BLOCKS && p.L < C::TR) ? p.L : C::TR;
  const bool uniform = (P % TE) == 0;
  ChunkIter bstart;
  bstart.init(t0, t1, P);
  int batch_prev_bh = -1;
  auto load_batch = [&](ChunkMeta& lc) {
    int bh = -1, j0 = 0, rows = 0;
    bool has = false;
    if (uniform) {
      const int64_t cs = bstart.cur + static_cast<int64_t>(lane) * TE;
      has = cs < bstart.end;
      const int off = bstart.j0 + lane * TE;  // < P + 32 TE
      const int qd = static_cast<int>(static_cast<unsigned>(off) / static_cast<unsigned>(P));
      bh = bstart.bh + qd;
      j0 = off - qd * P;
      rows = static_cast<int>(min(static_cast<int64_t>(TE), bstart.end - cs));
      bstart.cur += 32 * TE;
      const int nj = bstart.j0 + 32 * TE;
      const int nq = static_cast<int>(static_cast<unsigned>(nj) / static_cast<unsigned>(P));
      bstart.bh += nq;
      bstart.j0 = nj - nq * P;
    } else {
      ChunkIter c = bstart;
      for (int k = 0; k <= lane; ++k) {
        has = c.next(P, p.L, C::TR, p.mode, bh, j0, rows);
        if (!has) break;
      }
      // the next batch starts where lane 31 stopped
      bstart.cur = __shfl_sync(FULL_MASK, c.cur, 31);
      bstart.bh = __shfl_sync(FULL_MASK, c.bh, 31);
      bstart.j0 = __shfl_sync(FULL_MASK, c.j0, 31);
    }
    lc.has = has;
    lc.bh = has ? bh : -1;
    lc.j0 = j0;
    lc.rows = rows;
    int prev = __shfl_up_sync(FULL_MASK, lc.bh, 1);
    if (lane == 0) prev = batch_prev_bh;
    lc.first = has && lc.bh != prev;
    batch_prev_bh = __shfl_sync(FULL_MASK, lc.bh, 31);
    lc.n = has ? p.seq_lens[lc.bh / p.Hkv] : 0;
    lc.nk = 0;
    lc.blk = -1;
    if (has && p.mode == ATTN_BLOCKS) {
      const int slot = j0 >> p.log2L;
      lc.nk = p.n_kept[lc.bh];
      lc.blk = slot < p.kmax ? p.block_idx[static_cast<size_t>(lc.bh) * p.kmax + slot] : -1;
    }
  };
  // weighted mode: this lane's row (token index, weight) of one chunk
  auto load_rows = [&](int bh, int j0, int rows, int& idx, float& w) {
    const int row = j0 + lane;
    const bool in = bh >= 0 && lane < C::TPW && lane < rows && row < p.m;
    const size_t at = static_cast<size_t>(in ? bh : 0) * p.m + (in ? row : 0);
    idx = in ? p.tok_idx[at] : -1;
    w = in ? p.w[at] : 0.f;
  };
  // bcur is loaded after the warm-up pass below, bnext once the ring is full
  ChunkMeta bcur, bnext;
  bcur.has = 0;
  int widx = -1, widx_n = -1;
  float ww = 0.f, ww_n = 0.f;

  // issue the copies of chunk c (its metadata sits in lane c & 31 of bcur)
  auto issue = [&](int c, int s) {
    const int src = c & 31;
    const int mbh = __shfl_sync(FULL_MASK, bcur.bh, src);
    const int mj0 = __shfl_sync(FULL_MASK, bcur.j0, src);
    const int mrows = __shfl_sync(FULL_MASK, bcur.rows, src);
    const int mfirst = __shfl_sync(FULL_MASK, bcur.first, src);
    int n = __shfl_sync(FULL_MASK, bcur.n, src);
    const int mnk = __shfl_sync(FULL_MASK, bcur.nk, src);
    const int mblk = __shfl_sync(FULL_MASK, bcur.blk, src);
    unsigned char* sl = wb + s * C::SLOT;
    float* bias = reinterpret_cast<float*>(sl + C::SL_BIAS);
    if (n < 0 || n > p.Ncap) {
      if (lane == 0) atomicOr(p.status, KV_DEV_BAD_SEQ_LEN);
      n = max(0, min(n, p.Ncap));
    }
    const int nr = min(C::TPW, mrows);  // rows of this chunk
    bool vrow = false;
    int64_t tok = 0;
    float bz = -INFINITY;
    int nvalid = 0;
    if (p.mode == ATTN_WEIGHTED) {
      const bool inb = widx >= 0 && widx < n;
      vrow = lane < nr && ww > 0.f && inb;
      if (lane < nr && ww > 0.f && !inb) atomicOr(p.status, KV_DEV_BAD_TOKEN_INDEX);
      tok = widx;
      if (vrow) bz = log2f(ww);
      nvalid = __popc(__ballot_sync(FULL_MASK, vrow));
    } else {
      int64_t tok0 = 0;
      if (p.mode == ATTN_BLOCKS) {
        const int nbv = (n + p.L - 1) >> p.log2L;
        const int slot = mj0 >> p.log2L;
        if ((mnk < 0 || mnk > p.kmax) && lane == 0) atomicOr(p.status, KV_DEV_BAD_N_KEPT);
        const bool kept = slot < max(0, min(mnk, p.kmax));
        if (kept && (mblk < 0 || mblk >= nbv) && lane == 0) atomicOr(p.status, KV_DEV_BAD_BLOCK_INDEX);
        if (kept && mblk >= 0 && mblk < nbv) {
          tok0 = (static_cast<int64_t>(mblk) << p.log2L) + (mj0 & (p.L - 1));
          nvalid = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(nr), n - tok0)));
        }
      } else {
        tok0 = mj0;
        nvalid = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(nr), n - tok0)));
      }
      vrow = lane < nvalid;
      tok = tok0 + lane;
      if (vrow) bz = 0.f;
    }
    if (lane < C::TPW) bias[lane] = bz;
    if (lane == 0) *reinterpret_cast<int*>(sl + C::SL_HDR) = nvalid;
    const uint32_t tx = (mfirst ? C::QBYTES : 0u) + (MMA ? (nvalid > 0 ? 2u * C::KH * C::BOX : 0u) : 2u * nvalid * C::RB);
    __syncwarp();
    if (lane == 0) mbar_arrive_expect_tx(bars + s, tx);
    __syncwarp();
    const int b = mbh / p.Hkv, h = mbh - b * p.Hkv;
    if (mfirst && lane == 0)
      bulk_g2s(sl + C::SL_Q, Qg + (static_cast<size_t>(b) * p.Hq + h * G) * C::RB, C::QBYTES, bars + s, pol);
    if constexpr (MMA) {
      if (p.mode == ATTN_WEIGHTED) {
        // gathered rows: gather4 tensor copies (the maps' box is one row high),
        // four rows each, into the same swizzled tiles; a row that takes no part
        // reads the bh's first token instead and is masked by its bias
        if (nvalid > 0) {
          const int yrow = static_cast<int>(static_cast<int64_t>(mbh) * p.Ncap + (vrow ? tok : 0));
          const int g4 = (lane & 7) * 4;
          const int y0 = __shfl_sync(FULL_MASK, yrow, g4), y1 = __shfl_sync(FULL_MASK, yrow, g4 + 1);
          const int y2 = __shfl_sync(FULL_MASK, yrow, g4 + 2), y3 = __shfl_sync(FULL_MASK, yrow, g4 + 3);
          if (lane < C::TPW / 4) {
#pragma unroll
            for (int hx = 0; hx < C::KH; ++hx) {
              tma_gather4(sl + C::SL_K + hx * C::BOX + lane * 4 * 128, &tmK, hx * 64, y0, y1, y2, y3, bars + s);
              tma_gather4(sl + C::SL_V + hx * C::BOX + lane * 4 * 128, &tmV, hx * 64, y0, y1, y2, y3, bars + s);
            }
          }
        }
      } else if (nvalid > 0 && lane == 0) {
        // two tiled tensor copies (K, V) per 128-byte column box, 32 rows each; rows
        // past the valid ones are read but masked by their bias
        const int y = static_cast<int>(static_cast<int64_t>(mbh) * p.Ncap + (tok - lane));
#pragma unroll
        for (int hx = 0; hx < C::KH; ++hx) {
          tma_load_2d(sl + C::SL_K + hx * C::BOX, &tmK, hx * 64, y, bars + s, pol);
          tma_load_2d(sl + C::SL_V + hx * C::BOX, &tmV, hx * 64, y, bars + s, pol);
        }
      }
    } else if (p.mode == ATTN_WEIGHTED) {
      // one copy per gathered row
      if (vrow) {
        const size_t off = (static_cast<size_t>(mbh) * p.Ncap + tok) * C::RB;
        bulk_g2s(sl + C::SL_K + lane * C::RB, Kg + off, C::RB, bars + s, pol);
        bulk_g2s(sl + C::SL_V + lane * C::RB, Vg + off, C::RB, bars + s, pol);
      }
    } else if (nvalid > 0) {
      const size_t off = (static_cast<size_t>(mbh) * p.Ncap + (tok - lane)) * C::RB;
      if (lane == 1) bulk_g2s(sl + C::SL_K, Kg + off, nvalid * C::RB, bars + s, pol);
      if (lane == 2) bulk_g2s(sl + C::SL_V, Vg + off, nvalid * C::RB, bars + s, pol);
    }
  };
  // advance the issue cursor past chunk c: roll batches, prefetch weighted rows
  auto issued_one = [&](int c) {
    const int nc = c + 1;
    if ((nc & 31) == 0) {
      bcur = bnext;
      load_batch(bnext);
    }
    if (p.mode == ATTN_WEIGHTED) {
      widx = widx_n;
      ww = ww_n;
      // rows of chunk nc + 1 (it lies in bcur, or at lane 0 of bnext)
      const int c2 = nc + 1;
      const bool in_cur = (c2 >> 5) == (nc >> 5);
      const int src = c2 & 31;
      const int rbh = in_cur ? __shfl_sync(FULL_MASK, bcur.bh, src) : __shfl_sync(FULL_MASK, bnext.bh, src);
      const int rj0 = in_cur ? __shfl_sync(FULL_MASK, bcur.j0, src) : __shfl_sync(FULL_MASK, bnext.j0, src);
      const int rrows = in_cur ? __shfl_sync(FULL_MASK, bcur.rows, src) : __shfl_sync(FULL_MASK, bnext.rows, src);
      load_rows(rbh, rj0, rrows, widx_n, ww_n);
    }
  };

  // ---- per-warp softmax state --------------------------------------------
  // CUDA-core: mrun/lrun per head (warp-uniform max), acc[g] = channel chunk vc
  //   of rows owned in p.v.
  // Tensor core: this lane's heads are h0 = 2 (lane & 3) and h0 + 1; o[i] is the
  //   fragment of O^T rows 16 i + lane / 4 (+ 8) for those two heads.
  constexpr int NA = MMA ? 2 : G;                 // heads tracked per lane
  constexpr int ACC = MMA ? C::KS * 4 : G * C::CH;  // accumulator floats per lane
  float mrun[NA], lrun[NA];
  float acc[ACC];
  uint32_t qb[MMA ? C::KS * 2 : 1];               // q^T fragments (tensor core)
  auto reset_state = [&]() {
#pragma unroll
    for (int g = 0; g < NA; ++g) {
      mrun[g] = -INFINITY;
      lrun[g] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < ACC; ++e) acc[e] = 0.f;
  };

  auto flush = [&](int bh) {
    // local CTA: the record goes to ring slot 0 (this is the worker's last bh and
    // every copy it issued has been consumed); otherwise to the workspace
    float* rec = local ? reinterpret_cast<float*>(wb) : p.recs + static_cast<size_t>(wk + bh) * C::RECF;
    if constexpr (MMA) {
      const int h0 = 2 * (lane & 3);
      float lt[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float v = lrun[u];
        v += __shfl_xor_sync(FULL_MASK, v, 4);
        v += __shfl_xor_sync(FULL_MASK, v, 8);
        v += __shfl_xor_sync(FULL_MASK, v, 16);
        lt[u] = v;
      }
      const int dr = lane >> 2;
#pragma unroll
      for (int i = 0; i < C::KS; ++i) {
        if (h0 < G) {
          rec[h0 * D + 16 * i + dr] = acc[4 * i + 0];
          rec[h0 * D + 16 * i + dr + 8] = acc[4 * i + 2];
        }
        if (h0 + 1 < G) {
          rec[(h0 + 1) * D + 16 * i + dr] = acc[4 * i + 1];
          rec[(h0 + 1) * D + 16 * i + dr + 8] = acc[4 * i + 3];
        }
      }
      if (lane < 4) {
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (h0 + u < G) {
            rec[G * D + h0 + u] = mrun[u];
            rec[G * D + G + h0 + u] = lt[u];
          }
      }
    } else {
      const int vc = lane % C::CPR;
      // the row groups of p.v hold disjoint rows with the same (warp-uniform) max
#pragma unroll
      for (int mask = C::CPR; mask < 32; mask <<= 1)
#pragma unroll
        for (int e = 0; e < ACC; ++e) acc[e] += __shfl_xor_sync(FULL_MASK, acc[e], mask);
      if (lane < C::CPR) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float* dst = rec + g * D + vc * C::CH;
#pragma unroll
          for (int e = 0; e < C::CH; e += 4)
            *reinterpret_cast<float4*>(dst + e) =
                make_float4(acc[g * C::CH + e], acc[g * C::CH + e + 1], acc[g * C::CH + e + 2], acc[g * C::CH + e + 3]);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float lt = warp_sum(lrun[g]);
        if (lane == 0) {
          rec[G * D + g] = mrun[g];
          rec[G * D + G + g] = lt;
        }
      }
    }
    if (local) {
      __syncwarp();
      if (lane == 0) mbar_arrive(ready + warp);
    } else {
      __threadfence();
      __syncwarp();
      arrive_bh<D, G>(p, bh, lane);
    }
  };

  ChunkIter it;
  it.init(t0, t1, P);
  int cur_bh = -1;
  bool timed_out = false;
  bool next_loaded = false;
  int i = 0;       // chunks consumed
  int issued = 0;  // chunks whose copies were issued
  reset_state();
  // The first pass of the loop below runs the consumer over slot 0 holding
  // zeros with every row masked (it changes no state) before any global memory
  // is touched -- while the previous kernel in the stream may still run: the
  // consumer's instructions are then fetched before the copies load the memory
  // system, where each instruction-cache miss would wait behind them.
  {
    unsigned char* s0 = wb;
    if constexpr (MMA)
      for (int e = lane; e < C::SL_BIAS / 16; e += 32) reinterpret_cast<uint4*>(s0)[e] = make_uint4(0, 0, 0, 0);
    if (lane < C::TPW) reinterpret_cast<float*>(s0 + C::SL_BIAS)[lane] = -INFINITY;
    if (lane == 0) *reinterpret_cast<int*>(s0 + C::SL_HDR) = C::TPW;
    __syncwarp();
  }
  bool warm = true;
#pragma unroll 1
  while (true) {
    // keep the ring full: the only copy-issue site (the first S rounds only issue)
    if (!warm && issued - i < C::S && __shfl_sync(FULL_MASK, bcur.has, issued & 31)) {
      issue(issued, issued % C::S);
      issued_one(issued);
      ++issued;
      continue;
    }
    if (!warm && !next_loaded) {
      // the ring is full: fetch the next batch of chunk metadata
      next_loaded = true;
      load_batch(bnext);
    }
    int s = 0;
    bool first = true;
    if (!warm) {
      int bh, j0, rows;
      const bool more = it.next(P, p.L, C::TR, p.mode, bh, j0, rows);
      first = more && bh != cur_bh;
      if ((first || !more) && cur_bh >= 0) flush(cur_bh);  // the only flush site
      if (!more) break;
      s = i % C::S;
      const uint32_t phase = static_cast<uint32_t>(i / C::S) & 1u;
      if (first) {
        cur_bh = bh;
        reset_state();
      }
      if (!timed_out && !mbar_wait(bars + s, phase, p.status)) timed_out = true;
    }
    const unsigned char* sl = wb + s * C::SLOT;
    const int nvalid = *reinterpret_cast<const int*>(sl + C::SL_HDR);
    const float* bias = reinterpret_cast<const float*>(sl + C::SL_BIAS);
    if constexpr (MMA) {
      // ====================================================== tensor cores
      if (first) {
        // q^T as the B operand of q.k: b0 = q[h][16k + 2(l&3) .. +1], b1 = +8
        const int hq = lane >> 2;
        const unsigned char* qrow = sl + C::SL_Q + hq * C::RB;
#pragma unroll
        for (int k = 0; k < C::KS; ++k) {
          const int d0 = 16 * k + 2 * (lane & 3);
          qb[2 * k] = hq < G ? *reinterpret_cast<const uint32_t*>(qrow + d0 * 2) : 0u;
          qb[2 * k + 1] = hq < G ? *reinterpret_cast<const uint32_t*>(qrow + (d0 + 8) * 2) : 0u;
        }
      }
      if (p.mode != ATTN_WEIGHTED && nvalid > 0 && nvalid < C::TPW) {
        // The box brought rows past the valid ones (the next block, or cache
        // rows past the sequence); their logits are masked below, and their V
        // rows are zeroed so that a non-finite pattern there cannot reach p.v
        // as 0 * inf.
        unsigned char* vz = wb + s * C::SLOT + C::SL_V;
        const int per_box = (C::TPW - nvalid) * 8;  // 16-byte chunks past the valid rows
        for (int e = lane; e < per_box * C::KH; e += 32) {
          const int hx = e / per_box, r = e - hx * per_box;
          *reinterpret_cast<uint4*>(vz + hx * C::BOX + nvalid * 128 + r * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();  // the slot is refilled by the async proxy later
        __syncwarp();
      }
      if (nvalid > 0) {
        const uint32_t kbase = smem_u32(sl + C::SL_K);
        const uint32_t vbase = smem_u32(sl + C::SL_V);
        // ---- S^T = K q^T for two 16-token tiles: rows t = 16mt + l/4 (+8), heads h0, h0+1
        // (even and odd k-steps accumulate separately: two shorter mma chains)
        float sc4[2][4], sc4o[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) sc4[mt][e] = sc4o[mt][e] = 0.f;
          const int row = 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int k = 0; k < C::KS; ++k) {
            uint32_t a[4];
            ldsm_x4(kbase + C::swz(row, 2 * k + (lane >> 4)), a);
            if (k & 1)
              mma_bf16(sc4o[mt][0], sc4o[mt][1], sc4o[mt][2], sc4o[mt][3], a, qb[2 * k], qb[2 * k + 1]);
            else
              mma_bf16(sc4[mt][0], sc4[mt][1], sc4[mt][2], sc4[mt][3], a, qb[2 * k], qb[2 * k + 1]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) sc4[mt][e] += sc4o[mt][e];
        }
        // ---- logits (log2 domain) and the chunk maximum of each head
        const int tr = lane >> 2;
        float x[2][4];
        float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          // masked rows get -inf whatever their (possibly non-finite) dot
          const float ba = bias[16 * mt + tr], bb = bias[16 * mt + tr + 8];
          x[mt][0] = ba == -INFINITY ? -INFINITY : fmaf(sc4[mt][0], p.qscale, ba);
          x[mt][1] = ba == -INFINITY ? -INFINITY : fmaf(sc4[mt][1], p.qscale, ba);
          x[mt][2] = bb == -INFINITY ? -INFINITY : fmaf(sc4[mt][2], p.qscale, bb);
          x[mt][3] = bb == -INFINITY ? -INFINITY : fmaf(sc4[mt][3], p.qscale, bb);
          cm0 = fmaxf(cm0, fmaxf(x[mt][0], x[mt][2]));
          cm1 = fmaxf(cm1, fmaxf(x[mt][1], x[mt][3]));
        }
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
          cm0 = fmaxf(cm0, __shfl_xor_sync(FULL_MASK, cm0, m));
          cm1 = fmaxf(cm1, __shfl_xor_sync(FULL_MASK, cm1, m));
        }
        const float mn0 = fmaxf(mrun[0], cm0), mn1 = fmaxf(mrun[1], cm1);
        const float ms0 = safe_max_ref(mn0), ms1 = safe_max_ref(mn1);
        const float sc0 = fast_exp2(mrun[0] - ms0), sc1 = fast_exp2(mrun[1] - ms1);
        const bool same = __all_sync(FULL_MASK, mn0 == mrun[0] && mn1 == mrun[1]);
        mrun[0] = mn0;
        mrun[1] = mn1;
        if (!same) {
#pragma unroll
          for (int k = 0; k < C::KS; ++k) {
            acc[4 * k] *= sc0;
            acc[4 * k + 1] *= sc1;
            acc[4 * k + 2] *= sc0;
            acc[4 * k + 3] *= sc1;
          }
        }
        float ls0 = 0.f, ls1 = 0.f;
        // ---- P as the B operand of p.v (hi + lo bf16 parts), per token tile
        uint32_t bh_[2][2], bl_[2][2];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const float p0 = fast_exp2(x[mt][0] - ms0), p1 = fast_exp2(x[mt][1] - ms1);
          const float p2 = fast_exp2(x[mt][2] - ms0), p3 = fast_exp2(x[mt][3] - ms1);
          ls0 += p0 + p2;
          ls1 += p1 + p3;
          const uint32_t h01 = pack_bf16(p0, p1), h23 = pack_bf16(p2, p3);
          const uint32_t l01 = pack_bf16(p0 - bf16_lo(h01), p1 - bf16_hi(h01));
          const uint32_t l23 = pack_bf16(p2 - bf16_lo(h23), p3 - bf16_hi(h23));
          bh_[mt][0] = movm_trans(h01);
          bh_[mt][1] = movm_trans(h23);
          bl_[mt][0] = movm_trans(l01);
          bl_[mt][1] = movm_trans(l23);
        }
        lrun[0] = lrun[0] * sc0 + ls0;
        lrun[1] = lrun[1] * sc1 + ls1;
        // ---- O^T += V^T P over the two token tiles
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int row = 16 * mt + (lane & 7) + (lane >> 4) * 8;
#pragma unroll
          for (int k = 0; k < C::KS; ++k) {
            uint32_t a[4];
            ldsm_x4_trans(vbase + C::swz(row, 2 * k + ((lane >> 3) & 1)), a);
            mma_bf16(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3], a, bh_[mt][0], bh_[mt][1]);
            mma_bf16(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3], a, bl_[mt][0], bl_[mt][1]);
          }
        }
      }
    } else {
      // ====================================================== CUDA cores
      const int ts = lane >> 2;  // token group: rows ts + 8j, j < TPL
      const int pq = lane & 3;   // quarter of each row; lanes pq < TPL own row ts + 8 pq
      const bool owner = pq < C::TPL;
      const int vr = lane / C::CPR, vc = lane % C::CPR;
      if (first) {
        // q of the new group: input type -> fp32 * scale * log2(e), two planes
        constexpr int NQC = G * C::CPR;
        constexpr int PER = (NQC + 31) / 32;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const int qc = lane + 32 * k;
          if (qc < NQC) {
            const int g = qc / C::CPR, c = qc - g * C::CPR;
            float2 f[C::CH2];
            Chunk<T>::unpack(lds128(sl + C::SL_Q + qc * 16), f);
#pragma unroll
            for (int pl = 0; pl < C::QPL; ++pl)
              *reinterpret_cast<float4*>(q32 + (g * C::QHEAD + pl * C::QPLANE + c * 16) / 4) =
                  make_float4(f[2 * pl].x * p.qscale, f[2 * pl].y * p.qscale, f[2 * pl + 1].x * p.qscale,
                              f[2 * pl + 1].y * p.qscale);
          }
        }
        __syncwarp();
      }
      if (nvalid > 0) {
        float2 d[C::TPL][G];
#pragma unroll
        for (int j = 0; j < C::TPL; ++j)
#pragma unroll
          for (int g = 0; g < G; ++g) d[j][g] = make_float2(0.f, 0.f);
        const unsigned char* krow = sl + C::SL_K + ts * C::RB;
#pragma unroll
        for (int st = 0; st < C::CPL; ++st) {
          const int c = C::chunk_at(st, ts, pq);
          float2 kf[C::TPL][C::CH2];
#pragma unroll
          for (int j = 0; j < C::TPL; ++j) Chunk<T>::unpack(lds128(krow + j * 8 * C::RB + c * 16), kf[j]);
          const float* qc = q32 + c * 4;
#pragma unroll
          for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int pl = 0; pl < C::QPL; ++pl) {
              const float4 qv = *reinterpret_cast<const float4*>(qc + (g * C::QHEAD + pl * C::QPLANE) / 4);
              const float2 q0 = make_float2(qv.x, qv.y), q1 = make_float2(qv.z, qv.w);
#pragma unroll
              for (int j = 0; j < C::TPL; ++j) {
                d[j][g] = ffma2(q0, kf[j][2 * pl], d[j][g]);
                d[j][g] = ffma2(q1, kf[j][2 * pl + 1], d[j][g]);
              }
            }
          }
        }
        float sv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float v[C::TPL];
#pragma unroll
          for (int j = 0; j < C::TPL; ++j) {
            v[j] = d[j][g].x + d[j][g].y;
            v[j] += __shfl_xor_sync(FULL_MASK, v[j], 1);
            v[j] += __shfl_xor_sync(FULL_MASK, v[j], 2);
          }
          float mine = v[0];
#pragma unroll
          for (int j = 1; j < C::TPL; ++j)
            if (pq == j) mine = v[j];
          sv[g] = mine;
        }
        const int myrow = ts + 8 * pq;
        const float bz = owner ? bias[myrow] : -INFINITY;
        float sc[G];
        bool all_one = true;
        float pv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float xg = sv[g] + bz;
          const float cm = warp_max(xg);
          const float mn = fmaxf(mrun[g], cm);
          const float ms = safe_max_ref(mn);
          sc[g] = fast_exp2(mrun[g] - ms);
          all_one = all_one && (mn == mrun[g]);
          mrun[g] = mn;
          pv[g] = fast_exp2(xg - ms);
          lrun[g] = lrun[g] * sc[g] + pv[g];
        }
        if (owner) {
          float* prow = pbuf + myrow * C::PSTR;
#pragma unroll
          for (int g4 = 0; g4 < G; g4 += 4) {
            float a4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) a4[u] = g4 + u < G ? pv[g4 + u] : 0.f;
            *reinterpret_cast<float4*>(prow + g4) = make_float4(a4[0], a4[1], a4[2], a4[3]);
          }
        }
        if (!all_one) {
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < C::CH; ++e) acc[g * C::CH + e] *= sc[g];
        }
        __syncwarp();
#pragma unroll 4
        for (int r = vr; r < C::TPW; r += C::VR) {
          float2 vf[C::CH2];
          Chunk<T>::unpack(lds128(sl + C::SL_V + r * C::RB + vc * 16), vf);
          float pr[C::PSTR];
#pragma unroll
          for (int g4 = 0; g4 < C::PSTR; g4 += 4) {
            const float4 xx = *reinterpret_cast<const float4*>(pbuf + r * C::PSTR + g4);
            pr[g4] = xx.x;
            pr[g4 + 1] = xx.y;
            pr[g4 + 2] = xx.z;
            pr[g4 + 3] = xx.w;
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float2 pp = make_float2(pr[g], pr[g]);
#pragma unroll
            for (int e = 0; e < C::CH2; ++e) {
              float2 a2 = make_float2(acc[g * C::CH + 2 * e], acc[g * C::CH + 2 * e + 1]);
              a2 = ffma2(pp, vf[e], a2);
              acc[g * C::CH + 2 * e] = a2.x;
              acc[g * C::CH + 2 * e + 1] = a2.y;
            }
          }
        }
      }
    }
    // the slot is free again: order these reads before the next copy into it
    __syncwarp();
    fence_proxy_async_smem();
    if (warm) {
      warm = false;
      reset_state();
      // global memory from here on: the inputs may come from the kernel before
      grid_dep_wait();
      if constexpr (FUSED) fused_select<T, D, G, C>(p, smem, static_cast<int>(bh_of(wa[0])), warp, lane, pol);
      load_batch(bcur);
      if (p.mode == ATTN_WEIGHTED) {
        load_rows(__shfl_sync(FULL_MASK, bcur.bh, 0), __shfl_sync(FULL_MASK, bcur.j0, 0),
                  __shfl_sync(FULL_MASK, bcur.rows, 0), widx, ww);
        load_rows(__shfl_sync(FULL_MASK, bcur.bh, 1), __shfl_sync(FULL_MASK, bcur.j0, 1),
                  __shfl_sync(FULL_MASK, bcur.rows, 1), widx_n, ww_n);
      }
    } else {
      ++i;
    }
  }
  if (timed_out) {
    // give copies that may still be in flight a last bounded chance to land
    // before this CTA's shared memory is released
    for (int k = max(0, i - C::S); k < issued; ++k)
      mbar_wait(bars + (k % C::S), static_cast<uint32_t>(k / C::S) & 1u, nullptr);
  }
}

}  // namespace kvs
