// Device helpers shared by the kvsparse kernels (sm_100a): mbarrier and bulk-copy
// wrappers, bf16 unpacking, packed fp32 FMA, and the cross-lane "transpose
// reduction" that finishes many short dot products at once.
#pragma once

#include <cuda.h>

#include <cuda_bf16.h>
#include <cstdint>

#include "partition.h"

namespace kvs {

constexpr unsigned FULL_MASK = 0xffffffffu;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
// Wall-clock bound of a wait on a copy before it gives up and flags
// KV_DEV_WAIT_TIMEOUT: far beyond any legitimate copy latency (microseconds).
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;

__host__ __device__ constexpr int pow2ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}
__host__ __device__ constexpr int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for the phase with the given parity. Returns false (and sets the
// timeout bit in *status) once limit_ns of wall time has passed.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint32_t* status, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) break;
  }
  if (status) atomicOr(status, KV_DEV_WAIT_TIMEOUT);
  return false;
}
// The kernels' wait on a copy: gives up after WAIT_LIMIT_NS.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  return mbar_wait_for(bar, parity, status, WAIT_LIMIT_NS);
}

// ------------------------------------------------ programmatic dependent launch
// A kernel launched with programmatic stream serialization may start while the
// kernel before it in the stream is still running. Everything it does before
// grid_dep_wait() must touch no global memory that a preceding kernel writes or
// reads; grid_dep_wait() returns once the preceding grids have completed and
// their writes are visible (at once when nothing precedes). grid_dep_launch()
// lets the next kernel in the stream be scheduled early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------- bulk copies
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// Global -> this CTA's shared memory, completion counted in bytes on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Four rows of a 2-D tensor at arbitrary row coordinates (the map's box is one
// row high) into four consecutive box rows at dst, in the map's swizzle.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* tmap, int x, int y0, int y1, int y2, int y3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(smem_u32(bar))
      : "memory");
}

// Brings a tensor map (a __grid_constant__ kernel parameter) into the
// descriptor cache ahead of its first tiled copy.
__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// Tiled tensor copy of one box (2-D tensor map) into this CTA's shared memory.
// The box shape, swizzle and fill come from the tensor map; x (innermost) must
// be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ------------------------------------------------------------ arithmetic
// Two fp32 FMAs in one packed instruction: (a.x*b.x + c.x, a.y*b.y + c.y).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// A 16-byte chunk of a row, converted to fp32 pairs: 8 bf16 -> 4 float2,
// 4 fp32 -> 2 float2.
template <typename T>
struct Chunk;
template <>
struct Chunk<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(const uint4& r, float2 (&f)[4]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
  }
};
template <>
struct Chunk<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void unpack(const uint4& r, float2 (&f)[2]) {
    f[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
    f[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
  }
};

__device__ __forceinline__ uint4 lds128(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// ------------------------------------------------- transpose reduction
// Every lane of a group of LPR lanes holds N partial sums (value index 0..N-1).
// After the call the group's full sums are spread over its lanes: for N >= LPR
// lane c holds values c*(N/LPR) + j in v[j], j < N/LPR; for N < LPR lane c holds
// value c / (LPR/N) in v[0]. Each halving step sends the half a lane does not
// keep, so N values cost N-1 shuffles instead of N*log2(LPR).
template <int N, int MASK>
__device__ __forceinline__ void transpose_reduce(float* v, int lane) {
  if constexpr (MASK >= 1) {
    if constexpr (N > 1) {
      const bool up = (lane & MASK) != 0;
#pragma unroll
      for (int j = 0; j < N / 2; ++j) {
        const float send = up ? v[j] : v[j + N / 2];
        const float keep = up ? v[j + N / 2] : v[j];
        v[j] = keep + __shfl_xor_sync(FULL_MASK, send, MASK);
      }
      transpose_reduce<N / 2, MASK / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(FULL_MASK, v[0], MASK);
      transpose_reduce<1, MASK / 2>(v, lane);
    }
  }
}

// Layout of the values after transpose_reduce<NV, LPR/2> for R rows x GP heads
// (value index = row * GP + head).
template <int NV, int LPR, int GP>
struct HeldValues {
  static constexpr int NH = NV >= LPR ? NV / LPR : 1;  // values held per lane
  __device__ __forceinline__ static int index(int c, int j) {
    if constexpr (NV >= LPR)
      return c * NH + j;
    else
      return c / (LPR / NV);
  }
  // Lane-bit masks that change the row but not the head of the held values:
  // a max/sum over rows is a shuffle over masks ROW_MASK_LO .. LPR/2.
  static constexpr int ROW_MASK_LO = NV >= LPR ? GP / NH : (LPR / NV) * GP;
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(FULL_MASK, x, m);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL_MASK, x, m));
  return x;
}

__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load_as_float(const float* p) { return *p; }

}  // namespace kvs
