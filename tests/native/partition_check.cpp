// Host-side check of the attention work partition: every worker range is
// non-empty and contiguous, the token -> worker map inverts the ranges, the
// record slots (worker + bh) never collide, and the arrival count a bh waits for
// equals the number of workers whose range meets it. Exits non-zero on the
// first violation.
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <set>

#include "partition.h"

using namespace kvs;

static int fail(const char* what, int NBH, int P, long long cap, long long a, long long b) {
  std::printf("FAIL %s NBH=%d P=%d cap=%lld (%lld, %lld)\n", what, NBH, P, cap, a, b);
  return 1;
}

static int check(int NBH, int P, long long cap) {
  const Partition pt = make_partition(NBH, P, cap);
  if (pt.C < 1 || pt.C > MAX_WORKERS) return fail("worker count", NBH, P, cap, pt.C, 0);
  if (part_t0(pt, 0) != 0 || part_t0(pt, pt.C) != pt.TT) return fail("ends", NBH, P, cap, 0, 0);
  for (int u = 0; u < pt.C; ++u) {
    const long long a = part_t0(pt, u), b = part_t0(pt, u + 1);
    if (!(a < b) && pt.TT > 0) return fail("empty range", NBH, P, cap, u, a);
    if (a % RANGE_ALIGN) return fail("alignment", NBH, P, cap, u, a);
    if (part_t0(pt, u + pt.C) != pt.TT) return fail("past C", NBH, P, cap, u, 0);
    for (long long x : {a, (a + b) / 2, b - 1})
      if (x >= a && x < b && part_worker_of(pt, x) != u) return fail("worker_of", NBH, P, cap, u, x);
  }
  std::set<long long> slots;
  for (int bh = 0; bh < NBH; ++bh) {
    const long long lo = static_cast<long long>(bh) * pt.P, hi = lo + pt.P;
    const int cf = part_worker_of(pt, lo), cl = part_worker_of(pt, hi - 1);
    int meet = 0;
    for (int u = 0; u < pt.C; ++u) {
      const long long a = part_t0(pt, u), b = part_t0(pt, u + 1);
      if (a < hi && b > lo) {
        ++meet;
        if (u < cf || u > cl) return fail("meets outside [cf, cl]", NBH, P, cap, u, bh);
        if (!slots.insert(static_cast<long long>(u) + bh).second) return fail("slot collision", NBH, P, cap, u, bh);
        if (u + bh >= MAX_WORKERS + NBH) return fail("slot range", NBH, P, cap, u, bh);
      }
    }
    if (meet != cl - cf + 1) return fail("arrival count", NBH, P, cap, meet, cl - cf + 1);
  }
  if (part_grid(pt) * ATTN_NW < pt.C) return fail("grid", NBH, P, cap, part_grid(pt), pt.C);
  // bh-aligned splits: with enough room, every bh boundary is a worker boundary
  // (P a multiple of the range alignment), so no worker straddles two bhs
  const long long cap1 = cap < MAX_WORKERS ? cap : MAX_WORKERS;
  const long long lim = (pt.TT + MIN_TOKENS_PER_WORKER - 1) / MIN_TOKENS_PER_WORKER;
  long long splits = 0;
  if (NBH <= cap1 && NBH <= lim) {
    const long long smax = std::min(cap1 / NBH, lim / NBH);
    if (smax > ATTN_NW && static_cast<long long>(NBH) * ATTN_NW * 4 < cap1)
      splits = smax;
    else
      splits = (static_cast<long long>(NBH) * ATTN_NW <= cap1 && P >= ATTN_NW * RANGE_ALIGN) ? ATTN_NW : 1;
  }
  if (splits > 0 && P % RANGE_ALIGN == 0 && pt.TT / (NBH * splits) <= ALIGN_MAX_TOKENS) {
    if (pt.C % NBH) return fail("splits", NBH, P, cap, pt.C, NBH);
    if (pt.C / NBH != splits) return fail("splits per bh", NBH, P, cap, pt.C, NBH);
    for (int bh = 1; bh < NBH; ++bh) {
      const int u = part_worker_of(pt, static_cast<long long>(bh) * pt.P);
      if (part_t0(pt, u) != static_cast<long long>(bh) * pt.P) return fail("bh boundary", NBH, P, cap, bh, u);
    }
  }
  return 0;
}

int main() {
  const int nbhs[] = {1, 2, 3, 7, 8, 64, 256, 1000, 4096};
  const int Ps[] = {1, 16, 31, 32, 64, 100, 320, 1024, 2088, 32768, 131072};
  const long long caps[] = {1, 2, 3, 296, 592, 888, 1184, 4096};
  long long n = 0;
  for (int nbh : nbhs)
    for (int P : Ps)
      for (long long cap : caps) {
        if (static_cast<long long>(nbh) * P > (1ll << 31)) continue;
        if (check(nbh, P, cap)) return 1;
        ++n;
      }
  std::printf("OK %lld cases\n", n);
  return 0;
}
