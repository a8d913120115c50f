// Block-mode sparse decode attention, warp-specialised: exact softmax attention
// over the kept blocks' tokens plus the count-aware tail proxy, for bf16 caches
// with block size >= 32.
//
// Method: "OpenAttention reads 1% of the KV cache -- Count-aware tail proxy",
// section "Skipping reviews without losing the verdict" (the unread tail enters
// the softmax as one token: value = mean unread value, logit = mean unread logit
// + ln count), over the blocks chosen per KV head by the Equation 5 group score
// of "COBS: Cumulant Order Block Sparse Attention".
//
// Design (sm_100a, one CTA per SM).
//  * Work: every (sequence, KV head) pair ("bh") owns kmax * L / ROWS chunk
//    slots of ROWS = min(L, 64) rows on one axis (kept-block slot j, part of the
//    block); the axis is cut into one contiguous range per CTA -- whole pairs when
//    there are at least as many pairs as CTAs, else an even cut that shares pairs
//    between CTAs (a CTA then takes its shared pairs first, so that their
//    cross-CTA merges finish while its own pairs still stream).
//  * Producer warp: loads the chunk metadata (kept count, block index, sequence
//    length) 32 chunks per memory round trip, skips empty chunks, and keeps a
//    ring of NS slots full: per chunk one tensor copy of the ROWS x D key tile and
//    one of the value tile (128-byte swizzle; for D = 128 a three-dimensional
//    box takes both 128-byte column halves at once) and one bulk copy of the
//    pair's q, all counted in bytes on the slot's "full" mbarrier, keys and
//    values L2 evict-first. A single thread issues every copy, and each copy
//    instruction costs it tens of nanoseconds, so the copies are as few and as
//    large as the shared memory allows. It publishes the CTA's chunk count as
//    soon as its last metadata batch is read, which tells each consumer where
//    its work ends.
//  * Consumer warps (NC = 3): issue index i goes to consumer i % NC. A consumer keeps
//    the online-softmax state of its current pair on the tensor cores (q.k:
//    mma.sync m16n8k16 with the 16 tokens of a tile as M and the G query heads
//    as N; p.v: P split into a bf16 high part and remainder), and writes one
//    partial record (acc, max, sum) per pair into its record buffer.
//  * Merge warp: replays the chunk assignment from the same metadata, computes
//    the tail proxy of every pair whose first chunk slot lies in this CTA, folds
//    each pair's partial records (and the proxy) with the log-sum-exp merge, and
//    writes out / lse; a pair shared with other CTAs leaves one record in the
//    workspace and the last arriving CTA merges them.
//  * Proxy warp: computes the tail proxies of the CTA's pairs ahead of the merge
//    warp (their dependent memory round trips stay off every other warp's path).
// Progress: the producer waits only for ring slots, a consumer only for its next
// chunk and for its record buffers; with NS >= NC the chunk that lets any
// consumer flush the pair the merge warp waits for is always already issued.
// Every wait is bounded (1 s of %globaltimer, then KV_DEV_WAIT_TIMEOUT).
#pragma once

#include "attention.cuh"

namespace kvs {

// Warp roles. Warp w runs on scheduler partition w % 4; the consumers' tensor-core
// work slows every warp that shares their partition, so the producer and the
// merge warp get partition 3 to themselves (warps 3 and 7), the consumers are
// warps 0..2 and the proxy warp (memory round trips, few instructions) shares
// partition 2. Warps 4 and 5 have no role.
constexpr int GA_NC = 3;                        // consumer warps (warps 0 .. GA_NC - 1)
constexpr int GA_PRODUCER = 3;
constexpr int GA_PROXY = 6;
constexpr int GA_MERGER = 7;
constexpr int GA_THREADS = 8 * 32;
constexpr int GA_MAX_SLOTS = 32;
constexpr int GA_RB = 2;                        // record buffers per consumer
constexpr int GA_PR = 4;                        // proxy ring entries

template <int D, int G, int ROWS>
struct GaCfg {
  static constexpr int RB = D * 2;              // bytes per bf16 row
  static constexpr int KH = RB / 128;           // 128-byte column halves per row
  static constexpr int BOX = ROWS * 128;        // one swizzled column half of a tile
  static constexpr int KS = D / 16;             // k-steps of q.k, d-tiles of p.v
  static constexpr int QB = G * RB;             // q of one group
  static constexpr int SL_K = 0;
  static constexpr int SL_V = KH * BOX;
  static constexpr int SL_Q = 2 * KH * BOX;
  static constexpr int SLOT = (SL_Q + QB + 1023) & ~1023;  // 1024-aligned swizzled tiles
  static constexpr int SLOT_TX = 2 * KH * BOX + QB;        // bytes a data slot receives
  static constexpr int RECF = (G * D + 2 * G + 3) & ~3;    // record: acc[G][D], m[G], l[G]
  static constexpr int REC_BYTES = RECF * 4;
  static constexpr int PXF = (D + G + 3) & ~3;              // proxy entry: value[D], logit[G]
  static constexpr int PX_BYTES = PXF * 4;
  static constexpr int HDR_BYTES = GA_MAX_SLOTS * 16;      // per slot: bh, nvalid, tag
  static constexpr int BAR_BYTES = (2 * GA_MAX_SLOTS + 2 * GA_NC * GA_RB + 2 * GA_PR) * 8;
  static constexpr int FIXED = GA_NC * GA_RB * REC_BYTES + GA_PR * PX_BYTES + HDR_BYTES + BAR_BYTES;
  // the opt-in per-block limit (227 KB) minus the base-alignment slack, 1 KB of
  // margin and the static variables
  static constexpr int BUDGET = 227 * 1024 - 2 * 1024 - 64;
  static constexpr int NS0 = (BUDGET - FIXED) / SLOT;
  static constexpr int NS = NS0 > GA_MAX_SLOTS ? GA_MAX_SLOTS : NS0;
  static constexpr int SMEM = NS * SLOT + FIXED + 1024;
  // offsets from the 1024-aligned base
  static constexpr int O_REC = NS * SLOT;
  static constexpr int O_PX = O_REC + GA_NC * GA_RB * REC_BYTES;
  static constexpr int O_HDR = O_PX + GA_PR * PX_BYTES;
  static constexpr int O_BAR = O_HDR + HDR_BYTES;
  static_assert(NS >= GA_NC, "progress needs at least as many ring slots as consumers");
  static_assert(G <= 8 && RB % 128 == 0, "tensor-core consumer: G <= 8, rows of 128-byte boxes");
  static_assert(ROWS == 32 || ROWS == 64, "chunk rows");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  // byte offset of 16-byte chunk c of row r in a slot's K or V tiles
  // (128-byte swizzle: chunk c of a 128-byte line sits at c ^ (r mod 8))
  __device__ __forceinline__ static int swz(int r, int c) {
    return (c >> 3) * BOX + r * 128 + (((c & 7) ^ (r & 7)) << 4);
  }
};

// Slot header written by the producer (generic stores, published by the slot's
// full-barrier arrival).
struct GaHdr {
  int bh;      // pair of the chunk
  int nvalid;  // rows that take part (a prefix of the chunk's rows)
  int idx;     // issue index of the chunk now in the slot (-1: none yet)
  int pad;
};

// The CTA's chunk range [x0, x1) of the pair-major chunk axis (PC chunks a pair),
// in processing order: the pair it shares with the CTA before (segment A), the
// pair it shares with the CTA after (segment B), then the pairs in between. With
// at least as many pairs as CTAs the ranges hold whole pairs (pair c * NBH / N
// up to pair (c + 1) * NBH / N): no pair is shared, so every merge stays in
// shared memory, and an SM holding one pair more than another still finishes in
// time because HBM, not the SM, bounds the stream. With fewer pairs the chunk
// axis is cut evenly and pairs are shared.
__device__ __forceinline__ int64_t ga_x0(int64_t T, int c, int ncta, int PC, int NBH) {
  return NBH >= ncta ? static_cast<int64_t>(PC) * (static_cast<int64_t>(NBH) * c / ncta) : T * c / ncta;
}
struct GaRange {
  int64_t x0, x1, endA, startB;
  int64_t lenA, lenB;
  __device__ __forceinline__ void init(int64_t T, int cta, int ncta, int PC, int NBH) {
    x0 = ga_x0(T, cta, ncta, PC, NBH);
    x1 = ga_x0(T, cta + 1, ncta, PC, NBH);
    const int64_t pA = x0 / PC, pB = (x1 - 1) / PC;
    endA = min(x1, (pA + 1) * PC);
    if (pB != pA) {
      startB = pB * PC;
      lenB = x1 - startB;
    } else {
      startB = x1;
      lenB = 0;
    }
    lenA = endA - x0;
  }
  __device__ __forceinline__ int64_t len() const { return x1 - x0; }
  __device__ __forceinline__ int64_t x_at(int64_t k) const {
    if (k < lenA) return x0 + k;
    if (k < lenA + lenB) return startB + (k - lenA);
    return endA + (k - lenA - lenB);
  }
};

// CTA whose range holds chunk x (even cut: the largest c with floor(T c / N) <= x;
// only used when pairs are shared, i.e. with fewer pairs than CTAs).
__device__ __forceinline__ int ga_cta_of(int64_t x, int64_t T, int ncta) {
  return static_cast<int>((static_cast<int64_t>(ncta) * (x + 1) + T - 1) / T) - 1;
}

// One chunk's metadata: its pair, first cache row and rows that take part (0 for
// an empty chunk: slot past n_kept, or rows past the sequence). Device-resident
// values are checked here; a bad one sets a status bit and the chunk is skipped
// (report != 0: this lane may report).
struct GaChunk {
  int bh, nvalid;
  int64_t row;  // bh * Ncap + first token
};
__device__ __forceinline__ GaChunk ga_chunk(const AttnParams& p, int64_t x, int PC, int CPB, int ROWS, bool in,
                                            bool report) {
  GaChunk c;
  c.bh = in ? static_cast<int>(x / PC) : -1;
  c.nvalid = 0;
  c.row = 0;
  if (!in) return c;
  const int rem = static_cast<int>(x - static_cast<int64_t>(c.bh) * PC);
  const int j = rem / CPB, half = rem - j * CPB;
  const int b = c.bh / p.Hkv;
  // three independent loads (one memory round trip); j < max(kmax, 1)
  int n = p.seq_lens[b];
  int nk = p.n_kept[c.bh];
  const int blk = p.kmax > 0 ? p.block_idx[static_cast<size_t>(c.bh) * p.kmax + j] : -1;
  if (n < 0 || n > p.Ncap) {
    if (report) atomicOr(p.status, KV_DEV_BAD_SEQ_LEN);
    n = max(0, min(n, p.Ncap));
  }
  if (nk < 0 || nk > p.kmax) {
    if (report) atomicOr(p.status, KV_DEV_BAD_N_KEPT);
    nk = max(0, min(nk, p.kmax));
  }
  if (j >= nk) return c;
  const int nbv = (n + p.L - 1) >> p.log2L;
  if (blk < 0 || blk >= nbv) {
    if (report) atomicOr(p.status, KV_DEV_BAD_BLOCK_INDEX);
    return c;
  }
  const int tok0 = (blk << p.log2L) + half * ROWS;
  c.nvalid = max(0, min(ROWS, n - tok0));
  c.row = static_cast<int64_t>(c.bh) * p.Ncap + tok0;
  return c;
}

// ---------------------------------------------------------------- consumer math
// Online-softmax state of one consumer warp for one pair (tensor-core layout):
// lane holds heads h0 = 2 (lane & 3) and h0 + 1; acc[4 k + e] is the fragment of
// O^T rows 16 k + lane / 4 (+ 8) for those heads.
template <int D, int G, int ROWS>
struct GaState {
  using C = GaCfg<D, G, ROWS>;
  float m[2], l[2];
  float acc[C::KS * 4];
  uint32_t qb[C::KS * 2];  // q^T fragments (B operand of q.k)
  __device__ __forceinline__ void reset() {
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
#pragma unroll
    for (int e = 0; e < C::KS * 4; ++e) acc[e] = 0.f;
  }
  // q^T fragments from the slot's raw q rows: b0 = q[h][16k + 2(l&3) .. +1], b1 = +8
  __device__ __forceinline__ void load_q(const unsigned char* qrow0, int lane) {
    const int hq = lane >> 2;
    const unsigned char* qrow = qrow0 + hq * C::RB;
#pragma unroll
    for (int k = 0; k < C::KS; ++k) {
      const int d0 = 16 * k + 2 * (lane & 3);
      qb[2 * k] = hq < G ? *reinterpret_cast<const uint32_t*>(qrow + d0 * 2) : 0u;
      qb[2 * k + 1] = hq < G ? *reinterpret_cast<const uint32_t*>(qrow + (d0 + 8) * 2) : 0u;
    }
  }
  // Rows rb .. rb + 16 MT - 1 of the chunk in slot sl, of which the first nvalid
  // take part: logits in the log2 domain (qscale = softmax scale * log2 e), rows
  // >= nvalid masked. The MT tiles of 16 rows go through the tensor cores
  // together (independent accumulation chains) and share one softmax update. The
  // V rows past nvalid (the next block, or cache rows past the sequence) must
  // have been zeroed: their p is 0, and 0 times a non-finite pattern would reach
  // acc.
  template <int MT>
  __device__ __forceinline__ void consume(const unsigned char* sl, int rb, int nvalid, float qscale, int lane) {
    const uint32_t kbase = smem_u32(sl + C::SL_K);
    const uint32_t vbase = smem_u32(sl + C::SL_V);
    // S^T = K q^T: rows t = 16 mt + lane / 4 (+ 8), heads h0, h0 + 1; even and
    // odd k-steps accumulate separately (shorter dependency chains)
    float sc4[MT][4], sc4o[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc4[mt][e] = sc4o[mt][e] = 0.f;
#pragma unroll
    for (int k = 0; k < C::KS; ++k) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int row = rb + 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
        uint32_t a[4];
        ldsm_x4(kbase + C::swz(row, 2 * k + (lane >> 4)), a);
        if (k & 1)
          mma_bf16(sc4o[mt][0], sc4o[mt][1], sc4o[mt][2], sc4o[mt][3], a, qb[2 * k], qb[2 * k + 1]);
        else
          mma_bf16(sc4[mt][0], sc4[mt][1], sc4[mt][2], sc4[mt][3], a, qb[2 * k], qb[2 * k + 1]);
      }
    }
    const int tr = lane >> 2;
    float x[MT][4];
    float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const bool va = 16 * mt + tr < nvalid, vb = 16 * mt + tr + 8 < nvalid;
      x[mt][0] = va ? (sc4[mt][0] + sc4o[mt][0]) * qscale : -INFINITY;
      x[mt][1] = va ? (sc4[mt][1] + sc4o[mt][1]) * qscale : -INFINITY;
      x[mt][2] = vb ? (sc4[mt][2] + sc4o[mt][2]) * qscale : -INFINITY;
      x[mt][3] = vb ? (sc4[mt][3] + sc4o[mt][3]) * qscale : -INFINITY;
      cm0 = fmaxf(cm0, fmaxf(x[mt][0], x[mt][2]));
      cm1 = fmaxf(cm1, fmaxf(x[mt][1], x[mt][3]));
    }
#pragma unroll
    for (int s = 4; s < 32; s <<= 1) {
      cm0 = fmaxf(cm0, __shfl_xor_sync(FULL_MASK, cm0, s));
      cm1 = fmaxf(cm1, __shfl_xor_sync(FULL_MASK, cm1, s));
    }
    const float mn0 = fmaxf(m[0], cm0), mn1 = fmaxf(m[1], cm1);
    const float ms0 = safe_max_ref(mn0), ms1 = safe_max_ref(mn1);
    const float r0 = fast_exp2(m[0] - ms0), r1 = fast_exp2(m[1] - ms1);
    const bool same = __all_sync(FULL_MASK, mn0 == m[0] && mn1 == m[1]);
    m[0] = mn0;
    m[1] = mn1;
    if (!same) {
#pragma unroll
      for (int k = 0; k < C::KS; ++k) {
        acc[4 * k] *= r0;
        acc[4 * k + 1] *= r1;
        acc[4 * k + 2] *= r0;
        acc[4 * k + 3] *= r1;
      }
    }
    // P as the B operand of p.v: a bf16 high part and the bf16 remainder
    float ls0 = 0.f, ls1 = 0.f;
    uint32_t bh_[MT][2], bl_[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
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
    l[0] = l[0] * r0 + ls0;
    l[1] = l[1] * r1 + ls1;
    // O^T += V^T P over the MT token tiles
#pragma unroll
    for (int k = 0; k < C::KS; ++k) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int row = rb + 16 * mt + (lane & 7) + (lane >> 4) * 8;
        uint32_t a[4];
        ldsm_x4_trans(vbase + C::swz(row, 2 * k + ((lane >> 3) & 1)), a);
        mma_bf16(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3], a, bh_[mt][0], bh_[mt][1]);
        mma_bf16(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3], a, bl_[mt][0], bl_[mt][1]);
      }
    }
  }
  // The record (acc[G][D], m[G], l[G]) of this warp's state.
  __device__ __forceinline__ void write(float* rec, int lane) const {
    const int h0 = 2 * (lane & 3);
    float lt[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float v = l[u];
      v += __shfl_xor_sync(FULL_MASK, v, 4);
      v += __shfl_xor_sync(FULL_MASK, v, 8);
      v += __shfl_xor_sync(FULL_MASK, v, 16);
      lt[u] = v;
    }
    const int dr = lane >> 2;
#pragma unroll
    for (int k = 0; k < C::KS; ++k) {
      if (h0 < G) {
        rec[h0 * D + 16 * k + dr] = acc[4 * k + 0];
        rec[h0 * D + 16 * k + dr + 8] = acc[4 * k + 2];
      }
      if (h0 + 1 < G) {
        rec[(h0 + 1) * D + 16 * k + dr] = acc[4 * k + 1];
        rec[(h0 + 1) * D + 16 * k + dr + 8] = acc[4 * k + 3];
      }
    }
    if (lane < 4) {
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (h0 + u < G) {
          rec[G * D + h0 + u] = m[u];
          rec[G * D + G + h0 + u] = lt[u];
        }
    }
  }
};


// Zeroes the V rows nvalid..ROWS-1 of a slot (both column halves); the caller
// fences the generic writes against the tensor copies that later refill the slot.
template <int D, int G, int ROWS>
__device__ __forceinline__ void ga_zero_tail_rows(unsigned char* sl, int nvalid, int lane) {
  using C = GaCfg<D, G, ROWS>;
  unsigned char* vz = sl + C::SL_V;
  const int per_box = (ROWS - nvalid) * 8;  // 16-byte pieces past the valid rows
  for (int e = lane; e < per_box * C::KH; e += 32) {
    const int hx = e / per_box, r = e - hx * per_box;
    *reinterpret_cast<uint4*>(vz + hx * C::BOX + nvalid * 128 + r * 16) = make_uint4(0, 0, 0, 0);
  }
}

// The tail proxy of pair bh ("OpenAttention reads 1% of the KV cache", section
// "Skipping reviews without losing the verdict"): the unread tokens' mean value
// (this lane's VEC channels) and, per head, the log2-domain logit
// scale * log2(e) * q . (mean unread key) + log2(unread count); -inf when every
// token is kept. The unread sums are the totals minus the kept blocks' sums.
// Kept indices are checked (in [0, nbv), ascending); a bad one is left out and
// flags KV_DEV_BAD_BLOCK_INDEX. Two dependent memory round trips (up to 32 kept
// blocks): the indices with the totals and q, then the kept blocks' counts and
// sums, eight rows in flight; under a saturated HBM each round trip costs
// microseconds, and the merge of the CTA's last pair waits for this value.
template <int D, int G>
__device__ void ga_proxy(const AttnParams& p, int bh, int lane, float (&vb)[D / 32], float (&pm)[G]) {
  constexpr int VEC = D / 32;
  constexpr int UNR = 8;  // kept rows of sums in flight together
  const int b = bh / p.Hkv;
  const int32_t* idx = p.block_idx + static_cast<size_t>(bh) * p.kmax;
  // first round trip: everything that does not depend on the kept indices
  const int n = max(0, min(p.seq_lens[b], p.Ncap));
  const int nk = max(0, min(p.n_kept[bh], p.kmax));
  const int first32 = lane < p.kmax ? idx[lane] : INT_MAX;
  float kt[VEC], vt[VEC], qv[G][VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    kt[v] = p.k_tot[static_cast<size_t>(bh) * D + lane * VEC + v];
    vt[v] = p.v_tot[static_cast<size_t>(bh) * D + lane * VEC + v];
  }
  const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + (static_cast<size_t>(b) * p.Hq +
                                                                          (bh - b * p.Hkv) * G) * D + lane * VEC;
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int v = 0; v < VEC; ++v) qv[g][v] = __bfloat162float(qrow[g * D + v]);
  const int nbv = (n + p.L - 1) >> p.log2L;
  float ks[VEC], vs[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) ks[v] = vs[v] = 0.f;
  int cnt = 0;
  int prev = -1;
  // second round trip (per 32 kept blocks): their counts and sums together
  for (int s0 = 0; s0 < nk; s0 += 32) {
    const bool in_list = s0 + lane < nk;
    const int mine = in_list ? (s0 == 0 ? first32 : idx[s0 + lane]) : INT_MAX;
    int before = __shfl_up_sync(FULL_MASK, mine, 1);
    if (lane == 0) before = prev;
    const bool ok = in_list && mine >= 0 && mine < nbv && mine > before;
    if (__any_sync(FULL_MASK, in_list && !ok) && lane == 0) atomicOr(p.status, KV_DEV_BAD_BLOCK_INDEX);
    const unsigned okmask = __ballot_sync(FULL_MASK, ok);
    prev = __shfl_sync(FULL_MASK, mine, 31);
    const int c = ok ? p.counts[static_cast<size_t>(b) * p.NBcap + mine] : 0;
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
    cnt += __reduce_add_sync(FULL_MASK, c);
  }
  const int nT = n - cnt;
  if (nT <= 0) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) vb[v] = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) pm[g] = -INFINITY;
    return;
  }
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
    pm[g] = warp_sum(d) * p.qscale + lc;
  }
}

// Folds one record (m, l, acc for this lane's VEC channels of each head) into a
// running merge state.
template <int D, int G>
struct GaMerge {
  static constexpr int VEC = D / 32;
  float M[G], Ls[G], acc[G][VEC];
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      M[g] = -INFINITY;
      Ls[g] = 0.f;
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[g][v] = 0.f;
    }
  }
  // m, l of head g and its VEC values x
  __device__ __forceinline__ void fold(int g, float m, float l, const float (&x)[VEC]) {
    if (m == -INFINITY) return;
    const float Mn = fmaxf(M[g], m);
    const float a = fast_exp2(M[g] - Mn), b = fast_exp2(m - Mn);
    Ls[g] = Ls[g] * a + l * b;
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[g][v] = acc[g][v] * a + x[v] * b;
    M[g] = Mn;
  }
  __device__ __forceinline__ void fold_record(const float* rec, int lane, bool cached) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float x[VEC];
      const float* r = rec + g * D + lane * VEC;
      float m, l;
      if (cached) {
#pragma unroll
        for (int v = 0; v < VEC; ++v) x[v] = __ldcg(r + v);
        m = __ldcg(rec + G * D + g);
        l = __ldcg(rec + G * D + G + g);
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) x[v] = r[v];
        m = rec[G * D + g];
        l = rec[G * D + G + g];
      }
      fold(g, m, l, x);
    }
  }
  // Folds records of other CTAs (global memory, read through L2), NB at a time: every
  // record's loads of a batch are issued before the first fold, so their latencies
  // overlap.
  template <int NB>
  __device__ __forceinline__ void fold_records_global(const float* const (&rec)[NB], int n, int lane) {
    float x[NB][G][VEC], m[NB][G], l[NB][G];
#pragma unroll
    for (int t = 0; t < NB; ++t) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (t < n) {
#pragma unroll
          for (int v = 0; v < VEC; ++v) x[t][g][v] = __ldcg(rec[t] + g * D + lane * VEC + v);
          m[t][g] = __ldcg(rec[t] + G * D + g);
          l[t][g] = __ldcg(rec[t] + G * D + G + g);
        } else {
          m[t][g] = -INFINITY;
          l[t][g] = 0.f;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < NB; ++t)
#pragma unroll
      for (int g = 0; g < G; ++g)
        if (t < n) fold(g, m[t][g], l[t][g], x[t][g]);
  }
  // Folds up to N records of shared memory at once (rec[t] for t < n): the
  // maxima and sums first, then each lane's channels with 16-byte loads.
  template <int N>
  __device__ __forceinline__ void fold_records(const float* const (&rec)[N], int n, int lane) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mt[N], lt[N];
      float Mn = M[g];
#pragma unroll
      for (int t = 0; t < N; ++t) {
        mt[t] = t < n ? rec[t][G * D + g] : -INFINITY;
        lt[t] = t < n ? rec[t][G * D + G + g] : 0.f;
        Mn = fmaxf(Mn, mt[t]);
      }
      if (Mn == -INFINITY) continue;
      const float a = fast_exp2(M[g] - Mn);
      float wt[N];
      float Lsum = Ls[g] * a;
#pragma unroll
      for (int t = 0; t < N; ++t) {
        wt[t] = mt[t] == -INFINITY ? 0.f : fast_exp2(mt[t] - Mn);
        Lsum = fmaf(wt[t], lt[t], Lsum);
      }
      float x[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) x[v] = acc[g][v] * a;
#pragma unroll
      for (int t = 0; t < N; ++t) {
        if (t < n) {
          const float* r = rec[t] + g * D + lane * VEC;
          if constexpr (VEC == 4) {
            const float4 f = *reinterpret_cast<const float4*>(r);
            x[0] = fmaf(wt[t], f.x, x[0]);
            x[1] = fmaf(wt[t], f.y, x[1]);
            x[2] = fmaf(wt[t], f.z, x[2]);
            x[3] = fmaf(wt[t], f.w, x[3]);
          } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) x[v] = fmaf(wt[t], r[v], x[v]);
          }
        }
      }
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[g][v] = x[v];
      Ls[g] = Lsum;
      M[g] = Mn;
    }
  }
  __device__ __forceinline__ void write_record(float* rec, int lane) const {
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int v = 0; v < VEC; ++v) rec[g * D + lane * VEC + v] = acc[g][v];
      if (lane == 0) {
        rec[G * D + g] = M[g];
        rec[G * D + G + g] = Ls[g];
      }
    }
  }
  __device__ __forceinline__ void write_out(const AttnParams& p, int bh, int lane) const {
    const int b = bh / p.Hkv, h = bh - b * p.Hkv;
    float* o = p.out + (static_cast<size_t>(b) * p.Hq + h * G) * D + lane * VEC;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float inv = Ls[g] > 0.f ? 1.f / Ls[g] : 0.f;
      if constexpr (VEC == 4) {
        *reinterpret_cast<float4*>(o + g * D) =
            make_float4(acc[g][0] * inv, acc[g][1] * inv, acc[g][2] * inv, acc[g][3] * inv);
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) o[g * D + v] = acc[g][v] * inv;
      }
      if (p.lse && lane == 0)
        p.lse[static_cast<size_t>(b) * p.Hq + h * G + g] = Ls[g] > 0.f ? (M[g] + log2f(Ls[g])) * LN2 : -INFINITY;
    }
  }
};

// Waits until the chunk with issue index i has landed in its slot: 1, or 0 once
// *total shows that index i will never be issued, or -1 (and the timeout bit)
// after WAIT_LIMIT_NS. A parity wait is exact only while the barrier has at most
// one phase to go before the awaited one; consumers take the slots in turns, so
// a consumer can arrive at a slot while its previous use (another consumer's
// chunk) is still in flight. The slot header's issue index closes that gap: once
// it reads i, the producer has issued this use, which it does only after the
// previous use was consumed, and the parity wait is then exact.
__device__ __forceinline__ int ga_wait_chunk(uint64_t* bar, uint32_t parity, const volatile int* total,
                                             const volatile int* slot_idx, int i, uint32_t* status) {
  const uint64_t t0 = global_ns();
  while (true) {
    if (*slot_idx == i) {
      uint32_t ok;
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(ok)
          : "r"(smem_u32(bar)), "r"(parity), "r"(2000u)
          : "memory");
      if (ok) return 1;  // the chunk landed
    } else if (i >= *total) {
      return 0;  // no such chunk: this consumer's work is done
    } else {
      __nanosleep(64);
    }
    if (global_ns() - t0 > WAIT_LIMIT_NS) {
      atomicOr(status, KV_DEV_WAIT_TIMEOUT);
      return -1;
    }
  }
}

// One tile (ROWS rows x D) of K or V into its 128-byte-swizzled slot region:
// D = 128 takes both column halves with one three-dimensional box, D = 64 is one
// two-dimensional box.
template <int D>
__device__ __forceinline__ void ga_load_tile(void* dst, const CUtensorMap* m, int row, uint64_t* bar, uint64_t pol) {
  if constexpr (D == 128) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(0), "r"(row), "r"(0), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
  } else {
    tma_load_2d(dst, m, 0, row, bar, pol);
  }
}

template <int D, int G, int ROWS>
__global__ void __launch_bounds__(GA_THREADS, 1)
    gather_attn_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV) {
  using C = GaCfg<D, G, ROWS>;
  constexpr int VEC = D / 32;
  extern __shared__ __align__(1024) unsigned char ga_smem_raw[];
  unsigned char* smem = ga_smem_raw + ((1024u - (smem_u32(ga_smem_raw) & 1023u)) & 1023u);
  GaHdr* hdr = reinterpret_cast<GaHdr*>(smem + C::O_HDR);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::O_BAR);
  uint64_t* empty = full + GA_MAX_SLOTS;
  uint64_t* rec_full = empty + GA_MAX_SLOTS;   // [consumer][buffer]
  uint64_t* rec_empty = rec_full + GA_NC * GA_RB;
  uint64_t* px_full = rec_empty + GA_NC * GA_RB;
  uint64_t* px_empty = px_full + GA_PR;
  auto rec_buf = [&](int w, int k) -> float* {
    return reinterpret_cast<float*>(smem + C::O_REC + (w * GA_RB + k) * C::REC_BYTES);
  };
  auto px_buf = [&](int e) -> float* { return reinterpret_cast<float*>(smem + C::O_PX + e * C::PX_BYTES); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CPB = p.L / ROWS;                        // chunks per kept block
  const int PC = (p.kmax > 0 ? p.kmax : 1) * CPB;    // chunks per pair
  const int NBH = p.B * p.Hkv;
  const int64_t T = static_cast<int64_t>(NBH) * PC;
  const int cta = blockIdx.x, ncta = gridDim.x;
  GaRange rg;
  rg.init(T, cta, ncta, PC, NBH);
  // the CTA's pairs in processing order: pA, then pB (if another pair), then the
  // pairs between them
  const int64_t pA = rg.x0 / PC, pB = (rg.x1 - 1) / PC;
  const int64_t npairs = pB - pA + 1;
  auto pair_at = [&](int64_t k) -> int64_t { return k == 0 ? pA : (k == 1 ? pB : pA + k - 1); };
  auto owns = [&](int64_t bh) { const int64_t ps = bh * PC; return ps >= rg.x0 && ps < rg.x1; };
  const bool proxy_on = p.use_proxy != 0;
  __shared__ int prod_issued;       // ring uses the producer armed (for the drain at the end)
  __shared__ volatile int total;    // chunks this CTA issues, once the producer knows it

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int w = 0; w < GA_NC * GA_RB; ++w) {
      mbar_init(rec_full + w, 1);
      mbar_init(rec_empty + w, 1);
    }
    for (int e = 0; e < GA_PR; ++e) {
      mbar_init(px_full + e, 1);
      mbar_init(px_empty + e, 1);
    }
    fence_mbar_init();
    for (int s = 0; s < GA_MAX_SLOTS; ++s) hdr[s].idx = -1;
    prod_issued = 0;
    total = INT_MAX;
  }
  __syncthreads();

  if (warp == GA_PRODUCER) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tensor_map(&tmK);
      prefetch_tensor_map(&tmV);
    }
    const uint64_t pol = l2_evict_first_policy();   // K, V: read once
    const uint64_t qpol = l2_evict_last_policy();   // q: read by every chunk of its pair
    const unsigned char* Qg = static_cast<const unsigned char*>(p.q);
    grid_dep_wait();  // metadata and q come from the kernels before this one
    int issued = 0;
    bool ok = true;
    auto take_slot = [&](int i) -> int {  // wait until slot i % NS is free (bounded)
      const int s = i % C::NS;
      if (i >= C::NS && ok && !mbar_wait(empty + s, static_cast<uint32_t>(i / C::NS - 1) & 1u, p.status)) ok = false;
      return s;
    };
    const int64_t len = rg.len();
    for (int64_t k0 = 0; k0 < len && ok; k0 += 32) {
      const bool in = k0 + lane < len;
      const GaChunk ch = ga_chunk(p, in ? rg.x_at(k0 + lane) : 0, PC, CPB, ROWS, in, true);
      const int cnt = static_cast<int>(min(static_cast<int64_t>(32), len - k0));
      if (k0 + 32 >= len) {
        // the last batch: publish how many chunks this CTA issues in all, before
        // any of them is issued (no consumer has reached its end yet)
        const int nval = __popc(__ballot_sync(FULL_MASK, ch.nvalid > 0));
        if (lane == 0) total = issued + nval;
        __syncwarp();
      }
      for (int t = 0; t < cnt; ++t) {
        const int nv = __shfl_sync(FULL_MASK, ch.nvalid, t);
        if (nv <= 0) continue;
        const int cbh = __shfl_sync(FULL_MASK, ch.bh, t);
        const int64_t row = __shfl_sync(FULL_MASK, ch.row, t);
        const int s = take_slot(issued);
        if (!ok) break;
        if (lane == 0) {
          hdr[s].bh = cbh;
          hdr[s].nvalid = nv;
          *reinterpret_cast<volatile int*>(&hdr[s].idx) = issued;
          unsigned char* sl = smem + s * C::SLOT;
          mbar_arrive_expect_tx(full + s, C::SLOT_TX);
          const int y = static_cast<int>(row);
          ga_load_tile<D>(sl + C::SL_K, &tmK, y, full + s, pol);
          ga_load_tile<D>(sl + C::SL_V, &tmV, y, full + s, pol);
          const int b = cbh / p.Hkv, h = cbh - b * p.Hkv;
          bulk_g2s(sl + C::SL_Q, Qg + (static_cast<size_t>(b) * p.Hq + h * G) * C::RB, C::QB, full + s, qpol);
        }
        __syncwarp();
        ++issued;
      }
    }
    if (lane == 0) {
      prod_issued = issued;
      total = issued;  // after a timed-out wait: what was issued
    }
  } else if (warp < GA_NC) {
    // ================================================================ consumer
    GaState<D, G, ROWS> st;
    st.reset();
    int cur = -1;
    int flushes = 0;
    bool ok = true;
    auto flush = [&]() {
      const int k = flushes % GA_RB;
      if (flushes >= GA_RB && ok &&
          !mbar_wait(rec_empty + warp * GA_RB + k, static_cast<uint32_t>(flushes / GA_RB - 1) & 1u, p.status))
        ok = false;
      st.write(rec_buf(warp, k), lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(rec_full + warp * GA_RB + k);
      ++flushes;
    };
    for (int i = warp;; i += GA_NC) {
      const int s = i % C::NS;
      int got = 0;
      if (ok) {
        got = ga_wait_chunk(full + s, static_cast<uint32_t>(i / C::NS) & 1u, &total,
                            reinterpret_cast<volatile int*>(&hdr[s].idx), i, p.status);
        if (got < 0) ok = false;
      }
      const int bh = got > 0 ? hdr[s].bh : -1;
      const int nv = hdr[s].nvalid;
      unsigned char* sl = smem + s * C::SLOT;
      if (bh != cur) {
        if (cur >= 0) flush();
        cur = bh;
        if (bh >= 0) {
          st.reset();
          st.load_q(sl + C::SL_Q, lane);
        }
      }
      if (bh < 0) break;  // past this consumer's last chunk (or a timed-out wait)
      if (nv < ROWS) {
        ga_zero_tail_rows<D, G, ROWS>(sl, nv, lane);
        __syncwarp();
      }
      if (ROWS == 64 && nv > 32)
        st.template consume<ROWS / 16>(sl, 0, nv, p.qscale, lane);
      else
        st.template consume<2>(sl, 0, nv, p.qscale, lane);
      // the slot is free: order these reads before the copies that refill it
      __syncwarp();
      fence_proxy_async_smem();
      if (lane == 0) mbar_arrive(empty + s);
    }
  } else if (warp == GA_PROXY) {
    // ============================================================ proxy warp
    // the tail proxies of the pairs whose first chunk slot is here, in processing
    // order, into a ring the merge warp reads
    if (proxy_on) {
      grid_dep_wait();
      int e = 0;
      bool ok = true;
      for (int64_t k = 0; k < npairs; ++k) {
        const int64_t bh = pair_at(k);
        if (!owns(bh)) continue;
        const int slot = e % GA_PR;
        if (e >= GA_PR && ok && !mbar_wait(px_empty + slot, static_cast<uint32_t>(e / GA_PR - 1) & 1u, p.status))
          ok = false;
        float vb[VEC], pm[G];
        ga_proxy<D, G>(p, static_cast<int>(bh), lane, vb, pm);
        float* px = px_buf(slot);
#pragma unroll
        for (int v = 0; v < VEC; ++v) px[lane * VEC + v] = vb[v];
        if (lane == 0)
#pragma unroll
          for (int g = 0; g < G; ++g) px[D + g] = pm[g];
        __syncwarp();
        if (lane == 0) mbar_arrive(px_full + slot);
        ++e;
      }
    }
  } else if (warp == GA_MERGER) {
    // ================================================================ merge warp
    grid_dep_wait();
    uint32_t taken = 0;  // records taken per consumer (bits 4w..4w+3, modulo 16)
    int pxe = 0;         // proxy entries taken
    int issued = 0;      // issue index of the next valid chunk (replayed)
    bool ok = true;
    const int64_t len = rg.len();
    int cur = -1, cur_first = 0, cur_cnt = 0;
    auto finish_pair = [&](int bh, int first, int cnt) {
      const int64_t ps = static_cast<int64_t>(bh) * PC, pe = ps + PC;
      const bool shared = ps < rg.x0 || pe > rg.x1;
      GaMerge<D, G> mg;
      mg.reset();
      // the proxy (computed ahead by the proxy warp), then every record of the
      // pair; all of them are folded in one pass once they are there
      if (proxy_on && owns(bh)) {
        const int slot = pxe % GA_PR;
        if (ok && !mbar_wait(px_full + slot, static_cast<uint32_t>(pxe / GA_PR) & 1u, p.status)) ok = false;
        const float* px = px_buf(slot);
        float vb[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) vb[v] = px[lane * VEC + v];
#pragma unroll
        for (int g = 0; g < G; ++g) mg.fold(g, px[D + g], 1.f, vb);
        __syncwarp();
        if (lane == 0) mbar_arrive(px_empty + slot);
        ++pxe;
      }
      const int nrec = min(GA_NC, cnt);
      const float* recp[GA_NC];
#pragma unroll
      for (int t = 0; t < GA_NC; ++t) {
        recp[t] = nullptr;
        if (t < nrec) {
          const int w = (first + t) % GA_NC;
          const int tk = static_cast<int>((taken >> (4 * w)) & 15u);
          const int k = tk % GA_RB;
          if (ok && !mbar_wait(rec_full + w * GA_RB + k, static_cast<uint32_t>(tk / GA_RB) & 1u, p.status))
            ok = false;
          recp[t] = rec_buf(w, k);
        }
      }
      mg.template fold_records<GA_NC>(recp, nrec, lane);
      __syncwarp();
#pragma unroll
      for (int t = 0; t < GA_NC; ++t) {
        if (t < nrec) {
          const int w = (first + t) % GA_NC;
          const int tk = static_cast<int>((taken >> (4 * w)) & 15u);
          if (lane == 0) mbar_arrive(rec_empty + w * GA_RB + tk % GA_RB);
          taken = (taken & ~(15u << (4 * w))) | (static_cast<uint32_t>((tk + 1) & 15) << (4 * w));
        }
      }
      if (!shared) {
        mg.write_out(p, bh, lane);
        return;
      }
      // shared with other CTAs: leave this CTA's record, the last arriver merges
      const int side = (static_cast<int64_t>(bh) == pA) ? 0 : 1;
      float* wrec = p.recs + static_cast<size_t>(2 * cta + side) * C::RECF;
      mg.write_record(wrec, lane);
      __threadfence();
      __syncwarp();
      const int cf = ga_cta_of(ps, T, ncta), cl = ga_cta_of(pe - 1, T, ncta);
      int last = 0;
      if (lane == 0) {
        const uint32_t old = atomicAdd(p.counters + bh, 1u);
        last = old + 1 == static_cast<uint32_t>(cl - cf + 1);
        if (last) p.counters[bh] = 0u;  // ready for the next launch
      }
      last = __shfl_sync(FULL_MASK, last, 0);
      if (!last) return;
      __threadfence();
      mg.reset();
      constexpr int NBR = G <= 4 ? 4 : 2;  // records whose loads are in flight together
      for (int c0 = cf; c0 <= cl; c0 += NBR) {
        const float* recs[NBR];
#pragma unroll
        for (int t = 0; t < NBR; ++t) {
          const int c = min(c0 + t, cl);
          const int64_t cx0 = ga_x0(T, c, ncta, PC, NBH);
          const int cside = (static_cast<int64_t>(bh) == cx0 / PC) ? 0 : 1;
          recs[t] = p.recs + static_cast<size_t>(2 * c + cside) * C::RECF;
        }
        mg.template fold_records_global<NBR>(recs, min(NBR, cl - c0 + 1), lane);
      }
      mg.write_out(p, bh, lane);
    };
    for (int64_t k0 = 0; k0 < len; k0 += 32) {
      const bool in = k0 + lane < len;
      const GaChunk ch = ga_chunk(p, in ? rg.x_at(k0 + lane) : 0, PC, CPB, ROWS, in, false);
      const int cnt = static_cast<int>(min(static_cast<int64_t>(32), len - k0));
      for (int t = 0; t < cnt; ++t) {
        const int cbh = __shfl_sync(FULL_MASK, ch.bh, t);
        const int nv = __shfl_sync(FULL_MASK, ch.nvalid, t);
        if (cbh != cur) {
          if (cur >= 0) finish_pair(cur, cur_first, cur_cnt);
          cur = cbh;
          cur_first = issued;
          cur_cnt = 0;
        }
        if (nv > 0) {
          ++issued;
          ++cur_cnt;
        }
      }
    }
    if (cur >= 0) finish_pair(cur, cur_first, cur_cnt);
  }
  // No copy may still be in flight into this CTA's shared memory when it exits.
  // The producer waits for the last armed phase of every slot, under one overall
  // bound; normally the consumers saw them all complete and this returns at once.
  __syncthreads();
  if (warp == GA_PRODUCER && lane == 0) {
    const uint64_t t0 = global_ns();
    const int n_iss = prod_issued;
    for (int i = max(0, n_iss - C::NS); i < n_iss; ++i) {
      const int s = i % C::NS;
      const uint32_t par = static_cast<uint32_t>(i / C::NS) & 1u;
      while (!mbar_try_wait(full + s, par)) {
        if (global_ns() - t0 > WAIT_LIMIT_NS) {
          atomicOr(p.status, KV_DEV_WAIT_TIMEOUT);
          break;
        }
      }
    }
  }
}

}  // namespace kvs
