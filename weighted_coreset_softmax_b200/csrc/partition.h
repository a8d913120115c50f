// Work partition and workspace layout of the split-K attention kernels. Shared
// by host code (sizes, grid) and device code (which CTA covers which tokens, where
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

constexpr int MAX_CTAS = 1024;          // upper bound on attention CTAs per launch
constexpr int ATTN_NW = 2;              // warps per attention CTA (one partial record each)
constexpr int MIN_TOKENS_PER_CTA = 64;  // below this a CTA is not worth launching
constexpr int RANGE_ALIGN = 8;          // CTA token ranges start on multiples of 8

// Every (sequence, KV head) pair "bh" owns P consecutive slots of a global token
// axis of length TT = NBH * P: the kept blocks' tokens (P = kmax * L), the coreset
// rows (P = m) or the whole cache (P = Ncap). CTA c processes [t0(c), t0(c+1)).
struct Partition {
  int64_t TT;
  int P;
  int NBH;
  int C;
};

KVS_HD int64_t part_t0(const Partition& p, int c) {
  if (c >= p.C) return p.TT;
  const int64_t t = (static_cast<int64_t>(c) * p.TT) / p.C;
  return t - (t % RANGE_ALIGN);
}

// CTA whose range contains token x (0 <= x < TT).
KVS_HD int part_cta_of(const Partition& p, int64_t x) {
  int c = static_cast<int>((x * p.C) / (p.TT > 0 ? p.TT : 1));
  if (c >= p.C) c = p.C - 1;
  while (c + 1 < p.C && part_t0(p, c + 1) <= x) ++c;
  while (c > 0 && part_t0(p, c) > x) --c;
  return c;
}

KVS_HD Partition make_partition(int NBH, int P, int num_sms, int ctas_per_sm) {
  Partition p;
  p.NBH = NBH;
  p.P = P > 0 ? P : 1;
  p.TT = static_cast<int64_t>(NBH) * p.P;
  int64_t want = (p.TT + MIN_TOKENS_PER_CTA - 1) / MIN_TOKENS_PER_CTA;
  int64_t cap = static_cast<int64_t>(num_sms) * ctas_per_sm;
  if (cap > MAX_CTAS) cap = MAX_CTAS;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  p.C = static_cast<int>(want);
  return p;
}

// ------------------------------------------------------- workspace layout
// [status word | counters[NBH] | records[(MAX_CTAS + NBH) * ATTN_NW] | proxy records[NBH]]
// A record holds acc[G][D], m[G] (log2 domain), l[G] as fp32, padded to 16 bytes;
// warp w of CTA c writes its record for pair bh at index (c + bh) * ATTN_NW + w.
KVS_HD int record_floats(int G, int D) { return ((G * D + 2 * G) + 3) & ~3; }
KVS_HD size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
KVS_HD size_t ws_counters_off() { return 256; }
KVS_HD size_t ws_records_off(int NBH) { return ws_counters_off() + align256(sizeof(uint32_t) * NBH); }
KVS_HD size_t ws_proxy_off(int NBH, int G, int D) {
  return ws_records_off(NBH) +
         align256(sizeof(float) * static_cast<size_t>(record_floats(G, D)) * (MAX_CTAS + NBH) * ATTN_NW);
}
KVS_HD size_t ws_total(int NBH, int G, int D) {
  return ws_proxy_off(NBH, G, D) +
         align256(sizeof(float) * static_cast<size_t>(record_floats(G, D)) * NBH);
}

}  // namespace kvs
