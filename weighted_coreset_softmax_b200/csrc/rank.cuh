// Block ranking of one (sequence, KV head) by a whole CTA of NT threads, from
// the block logits in shared memory: the Eq. 5 group scores, the forced blocks,
// the k-th largest key and the ascending kept list. Used by the fused decode
// step (selection and attention in one CTA).
//
// Source: "COBS: Cumulant Order Block Sparse Attention" -- Equation (5): a KV
// head's block ranking is by the sum over its G query heads of per-head block
// softmax probabilities m_b / Z^(g,h).
//
// Keys are 64-bit: the score's bits above the inverted block index, so larger
// keys win and ties go to the lower index; forced blocks get key 0 and are kept
// outside the competition. For k <= 32 each warp extracts its k largest keys (k
// rounds of "largest key below the previous one", two 32-bit warp reductions
// each) and one warp takes the k-th largest of those; larger k use a
// most-significant-digit-first radix select over 8-bit digits.
#pragma once

#include "common.cuh"

namespace kvs {

template <int NT>
struct RankMisc {
  static constexpr int NWR = NT / 32;
  float pm[NWR][8], ps[NWR][8];           // per-warp (max, sum) of the normalisers
  unsigned hist[256];
  unsigned long long wtop[NWR * 32];      // per-warp k largest keys (k <= 32)
  unsigned long long prefix, mask;
  int krem, digit, above, bucket;
  int wsum[NWR];
};

// Sum of one int per thread over the CTA; every thread gets the result.
template <int NT>
__device__ __forceinline__ int cta_sum(int v, int* wsum) {
  v = __reduce_add_sync(FULL_MASK, v);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) s += wsum[w];
  __syncthreads();
  return s;
}

// 64-bit maximum over the warp (two 32-bit hardware reductions)
__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long x) {
  const unsigned hi = static_cast<unsigned>(x >> 32), lo = static_cast<unsigned>(x);
  const unsigned mh = __reduce_max_sync(FULL_MASK, hi);
  const unsigned ml = __reduce_max_sync(FULL_MASK, hi == mh ? lo : 0u);
  return (static_cast<unsigned long long>(mh) << 32) | ml;
}

// lg[g * nbp + i]: log2-domain block logits of the G heads for blocks i < nbv.
// Writes scores (optional, [NBcap] per bh), block_idx ([kmax] per bh, ascending)
// and n_kept. Every thread of the CTA calls it.
template <int G, int NT>
__device__ void rank_in_cta(const float* lg, int nbp, int nbv, int NBcap, int k_top, bool force_first,
                            bool force_last, int kmax, float* scores, int32_t* block_idx, int32_t* n_kept,
                            unsigned long long* key, RankMisc<NT>& ms) {
  constexpr int NWR = NT / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto forced_at = [&](int i) { return (force_first && i == 0) || (force_last && i == nbv - 1); };

  // normalisers log2 sum_b 2^lg (Equation 5's Z, log2 domain): (max, sum) pairs
  float lse[G];
  {
    float m[G], sm[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      sm[g] = 0.f;
    }
    for (int i = tid; i < nbv; i += NT)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float x = lg[g * nbp + i];
        if (x == -INFINITY) continue;
        if (x > m[g]) {
          sm[g] = sm[g] * exp2f(m[g] - x) + 1.f;
          m[g] = x;
        } else {
          sm[g] += exp2f(x - m[g]);
        }
      }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float m2 = __shfl_xor_sync(FULL_MASK, m[g], o), s2 = __shfl_xor_sync(FULL_MASK, sm[g], o);
        const float M = fmaxf(m[g], m2);
        sm[g] = (m[g] == -INFINITY ? 0.f : sm[g] * exp2f(m[g] - M)) + (m2 == -INFINITY ? 0.f : s2 * exp2f(m2 - M));
        m[g] = M;
      }
    if (lane == 0)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        ms.pm[warp][g] = m[g];
        ms.ps[warp][g] = sm[g];
      }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NWR; ++w) M = fmaxf(M, ms.pm[w][g]);
      float S = 0.f;
      if (M != -INFINITY)
#pragma unroll
        for (int w = 0; w < NWR; ++w)
          if (ms.pm[w][g] != -INFINITY) S += ms.ps[w][g] * exp2f(ms.pm[w][g] - M);
      lse[g] = (M == -INFINITY || S <= 0.f) ? -INFINITY : M + log2f(S);
    }
  }

  // group scores and keys
  int ncand = 0;
  for (int i = tid; i < nbv; i += NT) {
    float Sg = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (lse[g] != -INFINITY) Sg += exp2f(lg[g * nbp + i] - lse[g]);
    if (scores) scores[i] = Sg;
    const bool forced = forced_at(i);
    key[i] = forced ? 0ull
                    : ((static_cast<unsigned long long>(__float_as_uint(Sg)) << 32) |
                       static_cast<unsigned long long>(0xffffffffu - static_cast<uint32_t>(i)));
    ncand += !forced;
  }
  if (scores)
    for (int i = nbv + tid; i < NBcap; i += NT) scores[i] = 0.f;
  ncand = cta_sum<NT>(ncand, ms.wsum);  // also orders the key writes

  // threshold: keep keys with (key & mask) >= prefix
  unsigned long long prefix = 1ull, mask = ~0ull;  // default: every candidate
  if (k_top <= 0) {
    prefix = ~0ull;  // nothing competes successfully
  } else if (k_top < ncand && k_top <= 32) {
    const int per = (nbv + NWR - 1) / NWR;
    const int lo = warp * per, hi = min(nbv, lo + per);
    unsigned long long prev = ~0ull;
    for (int r = 0; r < k_top; ++r) {
      unsigned long long best = 0ull;
      for (int i = lo + lane; i < hi; i += 32) {
        const unsigned long long x = key[i];
        if (x < prev && x > best) best = x;
      }
      best = warp_max_key(best);
      if (lane == 0) ms.wtop[warp * 32 + r] = best;  // 0: this warp has no more candidates
      prev = best;
    }
    __syncthreads();
    if (warp == 0) {
      prev = ~0ull;
      for (int r = 0; r < k_top; ++r) {
        unsigned long long best = 0ull;
#pragma unroll
        for (int w = 0; w < NWR; ++w) {
          const unsigned long long x = lane < k_top ? ms.wtop[w * 32 + lane] : 0ull;
          if (x < prev && x > best) best = x;
        }
        prev = warp_max_key(best);
      }
      if (lane == 0) ms.prefix = prev;  // the k-th largest key
    }
    __syncthreads();
    prefix = ms.prefix;
  } else if (k_top < ncand) {
    if (tid == 0) {
      ms.prefix = 0ull;
      ms.mask = 0ull;
      ms.krem = k_top;
    }
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int d = tid; d < 256; d += NT) ms.hist[d] = 0u;
      __syncthreads();
      const unsigned long long pf = ms.prefix, mk = ms.mask;
      for (int i0 = 0; i0 < nbv; i0 += NT) {
        const int i = i0 + tid;
        int d = -1;
        if (i < nbv) {
          const unsigned long long x = key[i];
          if (x != 0ull && (x & mk) == pf) d = static_cast<int>((x >> shift) & 0xffull);
        }
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
        const unsigned before = incl - tot;
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
      if (ms.bucket == ms.krem) break;  // the whole bucket is taken (uniform)
    }
    prefix = ms.prefix;
    mask = ms.mask;
  }

  // ascending compaction of the kept blocks (forced ones included)
  const int per = (nbv + NT - 1) / NT;
  const int a0 = min(nbv, tid * per), a1 = min(nbv, a0 + per);
  int mine = 0;
  for (int i = a0; i < a1; ++i) {
    const unsigned long long x = key[i];
    mine += forced_at(i) || (x != 0ull && (x & mask) >= prefix);
  }
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
  for (int w = 0; w < NWR; ++w) {
    const int v = ms.wsum[w];
    if (w < warp) wbase += v;
    total += v;
  }
  int pos = wbase + incl - mine;
  for (int i = a0; i < a1; ++i) {
    const unsigned long long x = key[i];
    if (forced_at(i) || (x != 0ull && (x & mask) >= prefix)) {
      if (pos < kmax) block_idx[pos] = i;
      ++pos;
    }
  }
  if (tid == 0) *n_kept = min(total, kmax);
}

}  // namespace kvs
