// Work partition and workspace layout of the split-K attention kernels. Shared
// by host code (sizes, grid) and device code (which warp covers which tokens, where
// partial results live), so both sides derive them from the same functions.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "kvsparse.h"

#if defined(__CUDACC__)
#define KVS_HD __host__ __device__ __forceinline__
#else
#define KVS_HD inline
#endif

namespace kvs {

constexpr int ATTN_NW = 3;                 // worker warps per attention CTA
constexpr int MAX_WORKERS = 2048;          // upper bound on attention warps per launch
constexpr int MIN_TOKENS_PER_WORKER = 64;  // below this a warp is not worth starting
constexpr int RANGE_ALIGN = 32;            // worker ranges start on multiples of 32 (one copy box)
constexpr int64_t ALIGN_MAX_TOKENS = 4096; // bh-aligned ranges only up to this many tokens a worker

// Every (sequence, KV head) pair "bh" owns P consecutive slots of a global token
// axis of length TT = NBH * P: the kept blocks' tokens (P = kmax * L), the coreset
// rows (P = m) or the whole cache (P = Ncap). The axis is cut into C contiguous
// ranges, one per worker (a warp: worker u is warp u % ATTN_NW of CTA
// u / ATTN_NW); worker u processes [t0(u), t0(u + 1)). A worker index at or past
// C has an empty range.
struct Partition {
  int64_t TT;
  int P;
  int NBH;
  int C;
  int64_t tq;  // TT / C
  int tr;      // TT % C
};

// floor(u TT / C) rounded down to RANGE_ALIGN, as u tq + floor(u tr / C): one
// 32-bit division (u, tr < C <= MAX_WORKERS).
KVS_HD int64_t part_t0(const Partition& p, int u) {
  if (u >= p.C) return p.TT;
  const int64_t t = static_cast<int64_t>(u) * p.tq + static_cast<int64_t>(static_cast<unsigned>(u * p.tr) / static_cast<unsigned>(p.C));
  return t & ~static_cast<int64_t>(RANGE_ALIGN - 1);
}

// Worker whose range contains token x (0 <= x < TT): a floating-point estimate,
// corrected against the exact range starts. Ranges are never empty below C:
// make_partition keeps consecutive starts at least RANGE_ALIGN apart before they
// are rounded down to a multiple of RANGE_ALIGN.
KVS_HD int part_worker_of(const Partition& p, int64_t x) {
  int u = static_cast<int>(static_cast<double>(x) * p.C / static_cast<double>(p.TT > 0 ? p.TT : 1));
  if (u >= p.C) u = p.C - 1;
  if (u < 0) u = 0;
  while (u + 1 < p.C && part_t0(p, u + 1) <= x) ++u;
  while (u > 0 && part_t0(p, u) > x) --u;
  return u;
}

// max_workers: resident warps the device can hold for this kernel. For short
// ranges (up to ALIGN_MAX_TOKENS a worker) worker boundaries fall on bh
// boundaries where the counts allow it -- each bh split into ATTN_NW ranges (one
// CTA a bh) or one range a bh, or each worker holding whole bhs -- so that a
// worker finishes only once, at the end of its range, and a CTA holds whole bhs
// (its partial results merge in shared memory). With few bhs (one CTA each would
// fill less than a quarter of the resident warps) each bh is cut into as many
// ranges as fit instead, merged through the workspace. Long ranges use every resident
// warp with equal ranges: there the balance across SMs matters more than a
// round trip or two.
KVS_HD Partition make_partition(int NBH, int P, int64_t max_workers) {
  Partition p;
  p.NBH = NBH;
  p.P = P > 0 ? P : 1;
  p.TT = static_cast<int64_t>(NBH) * p.P;
  int64_t cap = max_workers;
  if (cap > MAX_WORKERS) cap = MAX_WORKERS;
  if (cap < 1) cap = 1;
  int64_t lim = (p.TT + MIN_TOKENS_PER_WORKER - 1) / MIN_TOKENS_PER_WORKER;  // >= 64 tokens a worker
  if (lim < 1) lim = 1;
  int64_t want;
  if (NBH <= cap && NBH <= lim) {
    int64_t smax = cap / NBH;
    if (smax > lim / NBH) smax = lim / NBH;
    const bool fills = static_cast<int64_t>(NBH) * ATTN_NW * 4 >= cap;  // a CTA per bh fills >= 1/4
    if (smax > ATTN_NW && !fills) {
      // few bhs: many ranges per bh fill the GPU; their partial results merge
      // through the workspace
      want = static_cast<int64_t>(NBH) * smax;
    } else {
      // ATTN_NW ranges a bh (one CTA per bh, each range at least one 32-token
      // box) or one range a bh (ATTN_NW bhs a CTA): every CTA then holds whole
      // bhs and merges them in shared memory
      const bool per_cta = static_cast<int64_t>(NBH) * ATTN_NW <= cap && p.P >= ATTN_NW * RANGE_ALIGN;
      want = static_cast<int64_t>(NBH) * (per_cta ? ATTN_NW : 1);
      if (per_cta) lim = want;  // ranges of >= 32 tokens are fine here
    }
  } else if (NBH > cap) {
    const int64_t per = (NBH + cap - 1) / cap;  // whole bhs per worker
    want = (NBH + per - 1) / per;
  } else {
    want = lim;
  }
  if (want > cap) want = cap;
  if (want > lim) want = lim;
  if (want < 1) want = 1;
  if (p.TT / want > ALIGN_MAX_TOKENS) want = cap < lim ? cap : lim;
  p.C = static_cast<int>(want);
  p.tq = p.TT / p.C;
  p.tr = static_cast<int>(p.TT % p.C);
  return p;
}

KVS_HD int part_grid(const Partition& p) { return (p.C + ATTN_NW - 1) / ATTN_NW; }

// ------------------------------------------------------- workspace layout
// [status word | counters[NBH] | records[MAX_WORKERS + NBH] | proxy records[NBH]]
// A record holds acc[G][D], m[G] (log2 domain), l[G] as fp32, padded to 16 bytes.
// Worker u writes its record for pair bh at index u + bh: the workers of one bh
// are consecutive, and a worker whose range reaches into bh + 1 is the first
// worker of bh + 1, so no two (worker, bh) pairs share an index.
KVS_HD int record_floats(int G, int D) { return ((G * D + 2 * G) + 3) & ~3; }
KVS_HD size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
KVS_HD size_t ws_counters_off() { return 256; }
KVS_HD size_t ws_records_off(int NBH) { return ws_counters_off() + align256(sizeof(uint32_t) * NBH); }
KVS_HD size_t ws_proxy_off(int NBH, int G, int D) {
  return ws_records_off(NBH) +
         align256(sizeof(float) * static_cast<size_t>(record_floats(G, D)) * (MAX_WORKERS + NBH));
}
KVS_HD size_t ws_total(int NBH, int G, int D) {
  return ws_proxy_off(NBH, G, D) +
         align256(sizeof(float) * static_cast<size_t>(record_floats(G, D)) * NBH);
}

}  // namespace kvs
