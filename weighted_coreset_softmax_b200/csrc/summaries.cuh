// Block summaries built once after prefill: per-block key sum, value sum and
// token count, and per-(sequence, KV head) totals.
//
// Sources: "COBS: Cumulant Order Block Sparse Attention" -- the mean-pool block
// summary (affine score (18): phi_b = mean key, a_b = ln L) and the per-block
// stored mean key; "OpenAttention reads 1% of the KV cache -- Count-aware tail
// proxy" -- the unread tail's mean key and value, which the attention kernel
// forms as (total - sum over kept blocks) / count.
//
// One thread owns one 16-byte channel chunk of one block and walks the block's
// rows, so a warp reads whole 256-byte rows of two blocks per instruction and no
// cross-thread reduction is needed. The totals are summed from the block sums by a
// second kernel in a fixed order (bit-reproducible, no float atomics).
#pragma once

#include "common.cuh"

namespace kvs {

template <typename T, int D>
__global__ void __launch_bounds__(256) block_sums_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                         const int32_t* __restrict__ seq_lens,
                                                         float* __restrict__ k_sum, float* __restrict__ v_sum,
                                                         int32_t* __restrict__ counts, int NBH, int Hkv, int Ncap,
                                                         int L, int NBcap) {
  constexpr int CH = 16 / sizeof(T);
  constexpr int LPR = D / CH;
  constexpr int CH2 = CH / 2;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = 2LL * NBH * NBcap * LPR;
  if (gid >= total) return;
  const int c = static_cast<int>(gid % LPR);
  int64_t rest = gid / LPR;
  const int blk = static_cast<int>(rest % NBcap);
  rest /= NBcap;
  const int bh = static_cast<int>(rest % NBH);
  const int tensor = static_cast<int>(rest / NBH);
  const int b = bh / Hkv;
  const int n = max(0, min(seq_lens[b], Ncap));
  const int start = blk * L;
  const int cnt = max(0, min(L, n - start));
  const T* src = (tensor ? V : K) + (static_cast<int64_t>(bh) * Ncap + start) * D + c * CH;
  float2 acc[CH2];
#pragma unroll
  for (int e = 0; e < CH2; ++e) acc[e] = make_float2(0.f, 0.f);
  int r = 0;
  for (; r + 8 <= cnt; r += 8) {
    uint4 raw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) raw[u] = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r + u) * D));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float2 f[CH2];
      Chunk<T>::unpack(raw[u], f);
#pragma unroll
      for (int e = 0; e < CH2; ++e) {
        acc[e].x += f[e].x;
        acc[e].y += f[e].y;
      }
    }
  }
  for (; r < cnt; ++r) {
    const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r) * D));
    float2 f[CH2];
    Chunk<T>::unpack(raw, f);
#pragma unroll
    for (int e = 0; e < CH2; ++e) {
      acc[e].x += f[e].x;
      acc[e].y += f[e].y;
    }
  }
  float* dst = (tensor ? v_sum : k_sum) + (static_cast<int64_t>(bh) * NBcap + blk) * D + c * CH;
#pragma unroll
  for (int e = 0; e < CH2; e += 2) {
    if (e + 1 < CH2)
      *reinterpret_cast<float4*>(dst + 2 * e) = make_float4(acc[e].x, acc[e].y, acc[e + 1].x, acc[e + 1].y);
    else
      *reinterpret_cast<float2*>(dst + 2 * e) = acc[e];
  }
  if (tensor == 0 && (bh % Hkv) == 0 && c == 0) counts[static_cast<int64_t>(b) * NBcap + blk] = cnt;
}

// Per-block key bounds for the Quest scorer ("COBS: Cumulant Order Block Sparse
// Attention", the paragraph on escaping the first-order ceiling: per block the
// element-wise minimum and maximum of its keys). bf16 caches; output
// [B][Hkv][NBcap][D][2] bf16, (min, max) of each channel side by side, so a block
// is one 4D-byte row like the fp32 key sums; blocks past the sequence get zeros.
// One thread owns one 16-byte channel chunk of one block and walks its rows.
template <int D>
__global__ void __launch_bounds__(256) block_bounds_kernel(const __nv_bfloat16* __restrict__ K,
                                                           const int32_t* __restrict__ seq_lens,
                                                           __nv_bfloat16* __restrict__ bounds, int NBH, int Hkv,
                                                           int Ncap, int L, int NBcap) {
  constexpr int LPR = D / 8;  // 16-byte chunks (8 channels) per row
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(NBH) * NBcap * LPR;
  if (gid >= total) return;
  const int c = static_cast<int>(gid % LPR);
  const int64_t rest = gid / LPR;
  const int blk = static_cast<int>(rest % NBcap);
  const int bh = static_cast<int>(rest / NBcap);
  const int n = max(0, min(seq_lens[bh / Hkv], Ncap));
  const int start = blk * L;
  const int cnt = max(0, min(L, n - start));
  const __nv_bfloat16* src = K + (static_cast<int64_t>(bh) * Ncap + start) * D + c * 8;
  __nv_bfloat162 mn[4], mx[4];
  if (cnt > 0) {
    const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(src));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) mn[e] = mx[e] = h[e];
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) mn[e] = mx[e] = __floats2bfloat162_rn(0.f, 0.f);
  }
  for (int r = 1; r < cnt; ++r) {
    const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r) * D));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      mn[e] = __hmin2(mn[e], h[e]);
      mx[e] = __hmax2(mx[e], h[e]);
    }
  }
  // channels 8c .. 8c + 7 as (min, max) pairs: 32 bytes
  __nv_bfloat162 out[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    out[2 * e] = __halves2bfloat162(__low2bfloat16(mn[e]), __low2bfloat16(mx[e]));
    out[2 * e + 1] = __halves2bfloat162(__high2bfloat16(mn[e]), __high2bfloat16(mx[e]));
  }
  uint4* dst = reinterpret_cast<uint4*>(bounds + ((static_cast<int64_t>(bh) * NBcap + blk) * D + c * 8) * 2);
  dst[0] = *reinterpret_cast<const uint4*>(&out[0]);
  dst[1] = *reinterpret_cast<const uint4*>(&out[4]);
}

// tot[bh][d] = sum over blocks of sums[bh][blk][d], four interleaved partial sums
// combined in a fixed order.
__global__ void __launch_bounds__(256) block_totals_kernel(const float* __restrict__ k_sum,
                                                           const float* __restrict__ v_sum,
                                                           float* __restrict__ k_tot, float* __restrict__ v_tot,
                                                           int NBH, int NBcap, int D) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = 2LL * NBH * D;
  if (gid >= total) return;
  const int d = static_cast<int>(gid % D);
  const int64_t rest = gid / D;
  const int bh = static_cast<int>(rest % NBH);
  const int tensor = static_cast<int>(rest / NBH);
  const float* src = (tensor ? v_sum : k_sum) + static_cast<int64_t>(bh) * NBcap * D + d;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  int blk = 0;
  for (; blk + 4 <= NBcap; blk += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] += src[static_cast<int64_t>(blk + u) * D];
  }
  for (; blk < NBcap; ++blk) a[0] += src[static_cast<int64_t>(blk) * D];
  (tensor ? v_tot : k_tot)[static_cast<int64_t>(bh) * D + d] = (a[0] + a[1]) + (a[2] + a[3]);
}

}  // namespace kvs

namespace kvs {

// Block mean keys at bf16 precision, built once from the fp32 key sums and the
// counts ("COBS: Cumulant Order Block Sparse Attention", the quantisation
// paragraph: the block mean is kept at bf16). Each thread converts eight
// channels: the mean is the correctly rounded fp32 quotient k_sum / n_b, rounded
// to the nearest bf16 (ties to even); blocks with no token get zeros.
__global__ void __launch_bounds__(256) block_mean16_kernel(const float* __restrict__ k_sum,
                                                           const int32_t* __restrict__ counts,
                                                           __nv_bfloat16* __restrict__ k_mean, int64_t rows, int Hkv,
                                                           int NBcap, int D) {
  const int per_row = D / 8;
  const int64_t total = rows * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / per_row;  // (b, h, blk)
    const int c = static_cast<int>(i - row * per_row);
    const int blk = static_cast<int>(row % NBcap);
    const int64_t bh = row / NBcap;
    const int b = static_cast<int>(bh / Hkv);
    const int n = counts[static_cast<int64_t>(b) * NBcap + blk];
    const float4* src = reinterpret_cast<const float4*>(k_sum + row * D + c * 8);
    const float4 a = __ldcs(src), bq = __ldcs(src + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float lo = 0.f, hi = 0.f;
      if (n > 0) {
        lo = __fdiv_rn(v[2 * e], static_cast<float>(n));
        hi = __fdiv_rn(v[2 * e + 1], static_cast<float>(n));
      }
      const __nv_bfloat16 bl = __float2bfloat16_rn(lo), bhv = __float2bfloat16_rn(hi);
      w[e] = static_cast<uint32_t>(__bfloat16_as_ushort(bl)) | (static_cast<uint32_t>(__bfloat16_as_ushort(bhv)) << 16);
    }
    *reinterpret_cast<uint4*>(k_mean + row * D + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace kvs
