// C ABI of libkvsparse: argument validation and kernel dispatch. Every check
// runs on the host before anything is launched; kernels are enqueued on the
// caller's stream and nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "attention.cuh"
#include "covariance.cuh"
#include "kvsparse.h"
#include "launch.h"
#include "select.cuh"
#include "summaries.cuh"

namespace kvs {

cudaError_t attn_launch_bf16_d64(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&, int,
                                  cudaStream_t);
cudaError_t attn_launch_bf16_d128(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&, int,
                                  cudaStream_t);
cudaError_t attn_launch_f32_d64(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&, int,
                                  cudaStream_t);
cudaError_t attn_launch_f32_d128(int, bool, const AttnParams&, const CUtensorMap&, const CUtensorMap&, int,
                                  cudaStream_t);
int attn_prepare_bf16_d64(int, bool, int);
int attn_prepare_bf16_d128(int, bool, int);
int attn_prepare_f32_d64(int, bool, int);
int attn_prepare_f32_d128(int, bool, int);
bool fused_fits_bf16_d64(int, int);
bool fused_fits_bf16_d128(int, int);
cudaError_t fused_launch_bf16_d64(int, const AttnParams&, const CUtensorMap&, const CUtensorMap&, int, cudaStream_t);
cudaError_t fused_launch_bf16_d128(int, const AttnParams&, const CUtensorMap&, const CUtensorMap&, int, cudaStream_t);
cudaError_t select_launch_bf16_d64(int, int, const SelParams&, int, cudaStream_t);
cudaError_t select_launch_bf16_d128(int, int, const SelParams&, int, cudaStream_t);
cudaError_t select_launch_f32_d64(int, int, const SelParams&, int, cudaStream_t);
cudaError_t select_launch_f32_d128(int, int, const SelParams&, int, cudaStream_t);

cudaError_t launch_attn(int dtype, int D, int G, bool use_mma, const AttnParams& p, const CUtensorMap& tk,
                        const CUtensorMap& tv, int grid, cudaStream_t st) {
  if (dtype == KV_BF16)
    return D == 64 ? attn_launch_bf16_d64(G, use_mma, p, tk, tv, grid, st)
                   : attn_launch_bf16_d128(G, use_mma, p, tk, tv, grid, st);
  return D == 64 ? attn_launch_f32_d64(G, false, p, tk, tv, grid, st) : attn_launch_f32_d128(G, false, p, tk, tv, grid, st);
}
int attn_ctas_per_sm(int dtype, int D, int G, bool use_mma, int dev) {
  if (dtype == KV_BF16)
    return D == 64 ? attn_prepare_bf16_d64(G, use_mma, dev) : attn_prepare_bf16_d128(G, use_mma, dev);
  return D == 64 ? attn_prepare_f32_d64(G, false, dev) : attn_prepare_f32_d128(G, false, dev);
}
bool fused_fits(int dtype, int D, int G, int NBcap) {
  if (dtype != KV_BF16) return false;
  return D == 64 ? fused_fits_bf16_d64(G, NBcap) : fused_fits_bf16_d128(G, NBcap);
}
cudaError_t launch_fused(int dtype, int D, int G, const AttnParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                         int grid, cudaStream_t st) {
  if (dtype != KV_BF16) return cudaErrorInvalidValue;
  return D == 64 ? fused_launch_bf16_d64(G, p, tk, tv, grid, st) : fused_launch_bf16_d128(G, p, tk, tv, grid, st);
}
cudaError_t launch_select(int dtype, int D, int G, int mode, const SelParams& p, int grid, cudaStream_t st) {
  if (dtype == KV_BF16)
    return D == 64 ? select_launch_bf16_d64(G, mode, p, grid, st) : select_launch_bf16_d128(G, mode, p, grid, st);
  return D == 64 ? select_launch_f32_d64(G, mode, p, grid, st) : select_launch_f32_d128(G, mode, p, grid, st);
}

template <typename T, int D>
static cudaError_t sums_td(const void* K, const void* V, const int32_t* seq_lens, float* k_sum, float* v_sum,
                           int32_t* counts, float* k_tot, float* v_tot, int NBH, int Hkv, int Ncap, int L, int NBcap,
                           cudaStream_t st) {
  constexpr int LPR = D / (16 / static_cast<int>(sizeof(T)));
  const int64_t total = 2LL * NBH * NBcap * LPR;
  const int64_t blocks = (total + 255) / 256;
  block_sums_kernel<T, D><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const T*>(K), static_cast<const T*>(V), seq_lens, k_sum, v_sum, counts, NBH, Hkv, Ncap, L, NBcap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t tot2 = 2LL * NBH * D;
  block_totals_kernel<<<static_cast<unsigned>((tot2 + 255) / 256), 256, 0, st>>>(k_sum, v_sum, k_tot, v_tot, NBH,
                                                                                  NBcap, D);
  return cudaGetLastError();
}

static cudaError_t launch_bounds(int D, const void* K, const int32_t* seq_lens, void* bounds, int NBH, int Hkv,
                                 int Ncap, int L, int NBcap, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(NBH) * NBcap * (D / 8);
  const unsigned blocks = static_cast<unsigned>((total + 255) / 256);
  const auto* k = static_cast<const __nv_bfloat16*>(K);
  auto* out = static_cast<__nv_bfloat16*>(bounds);
  if (D == 64)
    block_bounds_kernel<64><<<blocks, 256, 0, st>>>(k, seq_lens, out, NBH, Hkv, Ncap, L, NBcap);
  else
    block_bounds_kernel<128><<<blocks, 256, 0, st>>>(k, seq_lens, out, NBH, Hkv, Ncap, L, NBcap);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t cov_td(const void* K, const int32_t* seq_lens, float* xi, int NBH, int Hkv, int Ncap, int L,
                          int NBcap, int r, cudaStream_t st) {
  const size_t smem = cov_smem_bytes(L, D);
  static std::atomic<int> configured{0};  // one bit per device: smem limit raised
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured.load() & (1 << (dev & 31)))) {
    const cudaError_t e = cudaFuncSetAttribute(cov_factors_kernel<T, D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(cov_smem_bytes(COV_MAX_ROWS, D)));
    if (e != cudaSuccess) return e;
    configured.fetch_or(1 << (dev & 31));
  }
  const long long grid = static_cast<long long>(NBH) * NBcap;
  cov_factors_kernel<T, D, false><<<static_cast<unsigned>(grid), COV_THREADS, smem, st>>>(
      static_cast<const T*>(K), seq_lens, xi, Hkv, Ncap, L, NBcap, r, nullptr, 0, 0);
  return cudaGetLastError();
}

static cudaError_t launch_cov(int dtype, int D, const void* K, const int32_t* seq_lens, float* xi, int NBH, int Hkv,
                              int Ncap, int L, int NBcap, int r, cudaStream_t st) {
  if (dtype == KV_BF16)
    return D == 64 ? cov_td<__nv_bfloat16, 64>(K, seq_lens, xi, NBH, Hkv, Ncap, L, NBcap, r, st)
                   : cov_td<__nv_bfloat16, 128>(K, seq_lens, xi, NBH, Hkv, Ncap, L, NBcap, r, st);
  return D == 64 ? cov_td<float, 64>(K, seq_lens, xi, NBH, Hkv, Ncap, L, NBcap, r, st)
                 : cov_td<float, 128>(K, seq_lens, xi, NBH, Hkv, Ncap, L, NBcap, r, st);
}

cudaError_t launch_sums(int dtype, int D, const void* K, const void* V, const int32_t* seq_lens, float* k_sum,
                        float* v_sum, int32_t* counts, float* k_tot, float* v_tot, int NBH, int Hkv, int Ncap,
                        int L, int NBcap, cudaStream_t st) {
  if (dtype == KV_BF16) {
    if (D == 64)
      return sums_td<__nv_bfloat16, 64>(K, V, seq_lens, k_sum, v_sum, counts, k_tot, v_tot, NBH, Hkv, Ncap, L, NBcap,
                                        st);
    return sums_td<__nv_bfloat16, 128>(K, V, seq_lens, k_sum, v_sum, counts, k_tot, v_tot, NBH, Hkv, Ncap, L, NBcap,
                                       st);
  }
  if (D == 64)
    return sums_td<float, 64>(K, V, seq_lens, k_sum, v_sum, counts, k_tot, v_tot, NBH, Hkv, Ncap, L, NBcap, st);
  return sums_td<float, 128>(K, V, seq_lens, k_sum, v_sum, counts, k_tot, v_tot, NBH, Hkv, Ncap, L, NBcap, st);
}

}  // namespace kvs

namespace {

thread_local std::string g_last_error;

kv_status fail(kv_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

kv_status cuda_fail(cudaError_t e, const char* where) {
  return fail(KV_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by every entry point.
kv_status check_shape(const kv_shape* s) {
  if (!s) return fail(KV_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 0) return fail(KV_ERR_INVALID_ARG, "B = %d < 0", s->B);
  if (s->Hq < 1 || s->Hkv < 1 || s->Hq % s->Hkv != 0)
    return fail(KV_ERR_INVALID_ARG, "Hq = %d must be a positive multiple of Hkv = %d", s->Hq, s->Hkv);
  if (s->Ncap < 1) return fail(KV_ERR_INVALID_ARG, "Ncap = %d < 1", s->Ncap);
  if (s->block_size < 1) return fail(KV_ERR_INVALID_ARG, "block_size = %d < 1", s->block_size);
  if (s->dtype != KV_BF16 && s->dtype != KV_F32) return fail(KV_ERR_INVALID_ARG, "unknown dtype %d", (int)s->dtype);
  const int G = s->Hq / s->Hkv;
  if (G > 8) return fail(KV_ERR_UNSUPPORTED, "group size G = %d > 8", G);
  if (s->D != 64 && s->D != 128) return fail(KV_ERR_UNSUPPORTED, "head dim D = %d (supported: 64, 128)", s->D);
  const int L = s->block_size;
  if (L != 16 && L != 32 && L != 64 && L != 128)
    return fail(KV_ERR_UNSUPPORTED, "block_size = %d (supported: 16, 32, 64, 128)", L);
  const long long nb = (static_cast<long long>(s->Ncap) + L - 1) / L;
  if (nb > kvs::SEL_MAXNB) return fail(KV_ERR_UNSUPPORTED, "NBcap = %lld > %d", nb, kvs::SEL_MAXNB);
  if (static_cast<long long>(s->B) * s->Hkv > (1LL << 24))
    return fail(KV_ERR_UNSUPPORTED, "B * Hkv = %lld too large", static_cast<long long>(s->B) * s->Hkv);
  if (s->B > 0 && !s->seq_lens) return fail(KV_ERR_INVALID_ARG, "seq_lens is NULL");
  if (s->seq_lens && !aligned(s->seq_lens, 4)) return fail(KV_ERR_INVALID_ARG, "seq_lens not 4-byte aligned");
  return KV_OK;
}

kv_status need(const void* p, const char* name, size_t align = 16) {
  if (!p) return fail(KV_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(KV_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return KV_OK;
}

#define KV_TRY(expr)                 \
  do {                               \
    kv_status _st = (expr);          \
    if (_st != KV_OK) return _st;    \
  } while (0)

// bf16 caches use the tensor-core attention consumer unless the environment
// variable KVSPARSE_ATTN=fma selects the CUDA-core one (read once per process).
bool attention_uses_tensor_cores() {
  static const bool v = [] {
    const char* e = std::getenv("KVSPARSE_ATTN");
    return !(e && std::strcmp(e, "fma") == 0);
  }();
  return v;
}

// Block-mode attention over a bf16 cache with block size >= 32 runs the
// warp-specialised kernel (one CTA per SM, a producer warp streaming the kept
// chunks ahead of the tensor-core consumer warps) unless the environment
// variable KVSPARSE_ATTN is "v1" (or "fma"), which selects the per-worker-ring
// kernel (read once per process); other modes and shapes always run the latter.
bool attention_uses_gather() {
  static const bool v = [] {
    const char* e = std::getenv("KVSPARSE_ATTN");
    return !(e && (std::strcmp(e, "v1") == 0 || std::strcmp(e, "fma") == 0));
  }();
  return v;
}

// Tiled tensor map over a [rows][D] bf16 cache, 128-byte swizzle, zero fill past
// the last row. whole_rows == 0: 2-D, boxes of box_rows rows x 64 elements (128
// bytes; 32 rows for block copies, 1 row for gather4). whole_rows != 0 and D =
// 128: 3-D with the row's two 128-byte halves as the outermost dimension, so one
// box of {64, box_rows, 2} lands as two swizzled box_rows x 128-byte tiles, the
// first half then the second. Encoded through the driver entry point (no link
// against the driver library); the last few maps are cached, keyed by address,
// extent and shape.
kv_status encode_kv_map(const void* base, uint64_t rows, int D, int box_rows, CUtensorMap* out, int whole_rows = 0) {
  using Encode = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static Encode encode = nullptr;
  static std::mutex mu;
  struct Entry {
    const void* base;
    uint64_t rows;
    int D, box_rows, whole;
    CUtensorMap map;
  };
  static Entry cache[16];
  static int next_slot = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : cache)
    if (e.base == base && e.rows == rows && e.D == D && e.box_rows == box_rows && e.whole == whole_rows) {
      *out = e.map;
      return KV_OK;
    }
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess || !fn)
      return fail(KV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    encode = reinterpret_cast<Encode>(fn);
  }
  CUtensorMap m;
  CUresult r;
  if (whole_rows && D == 128) {
    const cuuint64_t dims[3] = {64, rows, 2};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, 128};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    r = encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    r = encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS) return fail(KV_ERR_CUDA, "tensor map encoding failed (CUresult %d)", static_cast<int>(r));
  cache[next_slot] = Entry{base, rows, D, box_rows, whole_rows, m};
  next_slot = (next_slot + 1) % 16;
  *out = m;
  return KV_OK;
}

int num_sms_current() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static int cache[64] = {0};
  int& c = cache[dev & 63];
  if (c == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    c = v;
  }
  return c;
}

// Selection done inside the attention kernel (fused decode step).
struct FusedSel {
  int k_top, force_first, force_last;
  int32_t* block_idx;
  int32_t* n_kept;
  float* scores;
};

// Can the fused decode step run this shape? (bf16 caches, tensor cores, the
// per-CTA layout fits, pair boundaries on 32-token range boundaries.)
bool fused_applies(const kv_shape* s, int kmax) {
  if (!attention_uses_tensor_cores() || s->dtype != KV_BF16) return false;
  const int NBcap = (s->Ncap + s->block_size - 1) / s->block_size;
  if (kmax <= 0 || (static_cast<long long>(kmax) * s->block_size) % kvs::RANGE_ALIGN != 0) return false;
  return kvs::fused_fits(s->dtype, s->D, s->Hq / s->Hkv, NBcap);
}

kv_status run_attention(const kv_shape* s, const void* q, float scale, const void* K, const void* V,
                        const int32_t* block_idx, const int32_t* n_kept, int kmax, const float* k_sum,
                        const float* v_sum, const int32_t* counts, const float* k_tot, const float* v_tot,
                        int use_proxy, const int32_t* tok_idx, const float* w, int m, int mode, float* out,
                        float* lse, void* ws, size_t ws_bytes, kv_stream_t stream, const FusedSel* fs = nullptr,
                        bool check_only = false) {
  const int G = s->Hq / s->Hkv;
  const int NBH = s->B * s->Hkv;
  const int NBcap = (s->Ncap + s->block_size - 1) / s->block_size;
  if (!std::isfinite(scale)) return fail(KV_ERR_INVALID_ARG, "scale is not finite");
  KV_TRY(need(q, "q"));
  KV_TRY(need(K, "K"));
  KV_TRY(need(V, "V"));
  KV_TRY(need(out, "out"));
  if (lse) KV_TRY(need(lse, "lse", 4));
  KV_TRY(need(ws, "workspace", 256));
  const size_t want = kv_workspace_bytes(s);
  if (ws_bytes < want) return fail(KV_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", ws_bytes, want);
  int P = 0;
  if (mode == kvs::ATTN_BLOCKS) {
    if (kmax < 0) return fail(KV_ERR_INVALID_ARG, "kmax = %d < 0", kmax);
    if (kmax > NBcap) return fail(KV_ERR_INVALID_ARG, "kmax = %d > NBcap = %d", kmax, NBcap);
    KV_TRY(need(block_idx, "block_idx", 4));
    KV_TRY(need(n_kept, "n_kept", 4));
    if (use_proxy) {
      KV_TRY(need(k_sum, "k_sum"));
      KV_TRY(need(v_sum, "v_sum"));
      KV_TRY(need(counts, "counts", 4));
      KV_TRY(need(k_tot, "k_tot"));
      KV_TRY(need(v_tot, "v_tot"));
    }
    P = (kmax > 0 ? kmax : 1) * s->block_size;
  } else if (mode == kvs::ATTN_WEIGHTED) {
    if (m < 0) return fail(KV_ERR_INVALID_ARG, "m = %d < 0", m);
    KV_TRY(need(tok_idx, "tok_idx", 4));
    KV_TRY(need(w, "w", 4));
    P = m > 0 ? m : 1;
    use_proxy = 0;
  } else {
    P = s->Ncap;
    use_proxy = 0;
  }
  if (NBH == 0) return KV_OK;
  const int sms = num_sms_current();
  if (sms <= 0) return fail(KV_ERR_CUDA, "no CUDA device available");
  int dev = 0;
  cudaGetDevice(&dev);
  // tensor cores for bf16 caches in every mode (gathered coreset rows arrive by
  // gather4 tensor copies)
  const bool use_mma = attention_uses_tensor_cores() && s->dtype == KV_BF16;
  if (fs && !use_mma) return fail(KV_ERR_UNSUPPORTED, "the fused decode step needs the tensor-core path");
  const int cps = kvs::attn_ctas_per_sm(s->dtype, s->D, G, use_mma, dev);
  if (cps <= 0) return fail(KV_ERR_CUDA, "attention kernel does not fit on an SM");
  if (use_mma && static_cast<uint64_t>(NBH) * s->Ncap > 0x7fffffffull)
    return fail(KV_ERR_UNSUPPORTED, "B * Hkv * Ncap = %llu rows is too many",
                static_cast<unsigned long long>(static_cast<uint64_t>(NBH) * s->Ncap));
  if (check_only) return KV_OK;
  kvs::AttnParams p{};
  p.q = q;
  p.K = K;
  p.V = V;
  p.seq_lens = s->seq_lens;
  p.block_idx = block_idx;
  p.n_kept = n_kept;
  p.kmax = kmax;
  p.k_sum = k_sum;
  p.v_sum = v_sum;
  p.counts = counts;
  p.k_tot = k_tot;
  p.v_tot = v_tot;
  p.tok_idx = tok_idx;
  p.w = w;
  p.m = m;
  p.out = out;
  p.lse = lse;
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  p.status = reinterpret_cast<uint32_t*>(wsb);
  p.counters = reinterpret_cast<uint32_t*>(wsb + kvs::ws_counters_off());
  p.recs = reinterpret_cast<float*>(wsb + kvs::ws_records_off(NBH));
  p.proxy_recs = reinterpret_cast<float*>(wsb + kvs::ws_proxy_off(NBH, G, s->D));
  p.B = s->B;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.Ncap = s->Ncap;
  p.L = s->block_size;
  p.log2L = 0;
  while ((1 << p.log2L) < s->block_size) ++p.log2L;
  p.NBcap = NBcap;
  p.mode = mode;
  p.use_proxy = use_proxy ? 1 : 0;
  p.qscale = scale * 1.4426950408889634f;
  if (fs) {
    // one CTA per pair: its workers split the pair's kept tokens
    p.part.NBH = NBH;
    p.part.P = P;
    p.part.TT = static_cast<int64_t>(NBH) * P;
    p.part.C = NBH * kvs::ATTN_NW;
    p.part.tq = p.part.TT / p.part.C;
    p.part.tr = static_cast<int>(p.part.TT % p.part.C);
    p.k_top = fs->k_top;
    p.force_first = fs->force_first ? 1 : 0;
    p.force_last = fs->force_last ? 1 : 0;
    p.sel_block_idx = fs->block_idx;
    p.sel_n_kept = fs->n_kept;
    p.sel_scores = fs->scores;
  } else {
    p.part = kvs::make_partition(NBH, P, static_cast<int64_t>(sms) * cps * kvs::ATTN_NW);
  }
  const bool gather = !fs && use_mma && mode == kvs::ATTN_BLOCKS && s->block_size >= 32 && attention_uses_gather();
  const int ga_rows = s->block_size >= 64 ? 64 : 32;  // rows a chunk of the warp-specialised kernel
  CUtensorMap tk, tv;
  std::memset(&tk, 0, sizeof(tk));
  std::memset(&tv, 0, sizeof(tv));
  if (use_mma) {
    const uint64_t rows = static_cast<uint64_t>(NBH) * s->Ncap;
    if (rows > 0x7fffffffull) return fail(KV_ERR_UNSUPPORTED, "B * Hkv * Ncap = %llu rows is too many", (unsigned long long)rows);
    if (gather) {
      KV_TRY(encode_kv_map(K, rows, s->D, ga_rows, &tk, 1));
      KV_TRY(encode_kv_map(V, rows, s->D, ga_rows, &tv, 1));
    } else {
      const int box_rows = mode == kvs::ATTN_WEIGHTED ? 1 : 32;  // gather4 needs a one-row box
      KV_TRY(encode_kv_map(K, rows, s->D, box_rows, &tk));
      KV_TRY(encode_kv_map(V, rows, s->D, box_rows, &tv));
    }
  }
  cudaError_t e;
  if (gather) {
    const long long T = static_cast<long long>(NBH) * (kmax > 0 ? kmax : 1) * (s->block_size / ga_rows);
    const int grid = static_cast<int>(std::min<long long>(sms, T));
    e = kvs::launch_gather(s->D, G, ga_rows, p, tk, tv, grid, reinterpret_cast<cudaStream_t>(stream));
  } else {
    e = fs ? kvs::launch_fused(s->dtype, s->D, G, p, tk, tv, NBH, reinterpret_cast<cudaStream_t>(stream))
           : kvs::launch_attn(s->dtype, s->D, G, use_mma, p, tk, tv, kvs::part_grid(p.part),
                              reinterpret_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, fs ? "fused decode step launch" : "attention launch");
  return KV_OK;
}

}  // namespace

namespace kvs {
// Every argument check of kv_sparse_decode_attn, with nothing enqueued.
kv_status sparse_attn_check(const kv_shape* shape, const void* q, float scale, const void* K, const void* V,
                            const int32_t* block_idx, const int32_t* n_kept, int kmax, const float* k_sum,
                            const float* v_sum, const int32_t* counts, const float* k_tot, const float* v_tot,
                            int use_tail_proxy, const int32_t* tok_idx, const float* w, int m, float* out, float* lse,
                            void* workspace, size_t ws_bytes) {
  KV_TRY(check_shape(shape));
  const int mode = tok_idx ? kvs::ATTN_WEIGHTED : kvs::ATTN_BLOCKS;
  return run_attention(shape, q, scale, K, V, block_idx, n_kept, kmax, k_sum, v_sum, counts, k_tot, v_tot,
                       use_tail_proxy, tok_idx, w, m, mode, out, lse, workspace, ws_bytes, nullptr, nullptr, true);
}
}  // namespace kvs

extern "C" {

kv_status kv_build_block_summaries(const kv_shape* shape, const void* K, const void* V, float* k_sum, float* v_sum,
                                   int32_t* counts, float* k_tot, float* v_tot, kv_stream_t stream) {
  KV_TRY(check_shape(shape));
  KV_TRY(need(K, "K"));
  KV_TRY(need(V, "V"));
  KV_TRY(need(k_sum, "k_sum"));
  KV_TRY(need(v_sum, "v_sum"));
  KV_TRY(need(counts, "counts", 4));
  KV_TRY(need(k_tot, "k_tot"));
  KV_TRY(need(v_tot, "v_tot"));
  const int NBH = shape->B * shape->Hkv;
  if (NBH == 0) return KV_OK;
  const int NBcap = (shape->Ncap + shape->block_size - 1) / shape->block_size;
  cudaError_t e = kvs::launch_sums(shape->dtype, shape->D, K, V, shape->seq_lens, k_sum, v_sum, counts, k_tot, v_tot,
                                   NBH, shape->Hkv, shape->Ncap, shape->block_size, NBcap,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "summary launch");
  return KV_OK;
}

kv_status kv_build_block_key_means(const kv_shape* shape, const float* k_sum, const int32_t* counts, void* k_mean,
                                   kv_stream_t stream) {
  KV_TRY(check_shape(shape));
  KV_TRY(need(k_sum, "k_sum"));
  KV_TRY(need(counts, "counts", 4));
  KV_TRY(need(k_mean, "k_mean"));
  const int NBH = shape->B * shape->Hkv;
  const int NBcap = (shape->Ncap + shape->block_size - 1) / shape->block_size;
  if (NBH == 0 || NBcap == 0) return KV_OK;
  const int64_t rows = static_cast<int64_t>(NBH) * NBcap;
  const int64_t work = rows * (shape->D / 8);
  const int sms = num_sms_current();
  if (sms <= 0) return fail(KV_ERR_CUDA, "no CUDA device available");
  const int64_t want = (work + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
  kvs::block_mean16_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      k_sum, counts, static_cast<__nv_bfloat16*>(k_mean), rows, shape->Hkv, NBcap, shape->D);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "key-mean launch");
  return KV_OK;
}

kv_status kv_build_block_bounds(const kv_shape* shape, const void* K, void* k_bounds, kv_stream_t stream) {
  KV_TRY(check_shape(shape));
  if (shape->dtype != KV_BF16) return fail(KV_ERR_UNSUPPORTED, "block bounds are built for bf16 caches only");
  KV_TRY(need(K, "K"));
  KV_TRY(need(k_bounds, "k_bounds"));
  const int NBH = shape->B * shape->Hkv;
  if (NBH == 0) return KV_OK;
  const int NBcap = (shape->Ncap + shape->block_size - 1) / shape->block_size;
  cudaError_t e = kvs::launch_bounds(shape->D, K, shape->seq_lens, k_bounds, NBH, shape->Hkv, shape->Ncap,
                                     shape->block_size, NBcap, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bounds launch");
  return KV_OK;
}

kv_status kv_build_block_cov_factors(const kv_shape* shape, const void* K, int rank, float* k_xi,
                                     kv_stream_t stream) {
  KV_TRY(check_shape(shape));
  if (rank < 1 || rank > kvs::COV_MAX_RANK) return fail(KV_ERR_INVALID_ARG, "rank = %d outside 1..%d", rank,
                                                         kvs::COV_MAX_RANK);
  if (shape->block_size > kvs::COV_MAX_ROWS)
    return fail(KV_ERR_UNSUPPORTED, "covariance factors are built for block sizes up to %d", kvs::COV_MAX_ROWS);
  KV_TRY(need(K, "K"));
  KV_TRY(need(k_xi, "k_xi"));
  const int NBH = shape->B * shape->Hkv;
  const int NBcap = (shape->Ncap + shape->block_size - 1) / shape->block_size;
  if (NBH == 0 || NBcap == 0) return KV_OK;
  if (static_cast<long long>(NBH) * NBcap > 0x7fffffffLL) return fail(KV_ERR_UNSUPPORTED, "too many blocks");
  cudaError_t e = kvs::launch_cov(shape->dtype, shape->D, K, shape->seq_lens, k_xi, NBH, shape->Hkv, shape->Ncap,
                                  shape->block_size, NBcap, rank, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "covariance factors launch");
  return KV_OK;
}

}  // extern "C"

namespace {
// CTAs per pair for the few-pairs selector (0: the one-CTA kernel): the summary and
// bf16-mean scorers with k_top <= 16, when at least two CTAs per pair fit on the SMs.
// KVSPARSE_SELECT_SPLIT=0 in the environment (read once) keeps the one-CTA kernel.
int split_select_ctas(int sel_mode, int k_top, int NBH) {
  static const bool disabled = [] {
    const char* v = std::getenv("KVSPARSE_SELECT_SPLIT");
    return v && v[0] == '0';
  }();
  if (disabled || (sel_mode != kvs::SEL_SUMMARY && sel_mode != kvs::SEL_MEAN16) || k_top > kvs::SEL_TOPK || NBH < 1)
    return 0;
  const int sms = num_sms_current();
  const int S = std::min(8, sms / NBH);
  return S >= 2 ? S : 0;
}

// Shared by the summary, exact-mass and Quest selections: argument checks and the
// launch. sel_mode is a kvs::SelMode.
kv_status select_any(const kv_shape* shape, const void* q, float scale, int sel_mode, const float* k_sum,
                     const void* k_bounds, const int32_t* counts, const void* K, int k_top, int force_first,
                     int force_last, int kmax, int32_t* block_idx, int32_t* n_kept, float* scores,
                     kv_stream_t stream, const float* k_xi = nullptr, int rank = 0, const void* k_mean16 = nullptr,
                     const uint8_t* xi4 = nullptr, const float* xi4_scale = nullptr, const float* Uq = nullptr,
                     int s_dim = 0) {
  KV_TRY(check_shape(shape));
  if (!std::isfinite(scale)) return fail(KV_ERR_INVALID_ARG, "scale is not finite");
  KV_TRY(need(q, "q"));
  if (sel_mode == kvs::SEL_SUMMARY || sel_mode == kvs::SEL_COBS) {
    KV_TRY(need(k_sum, "k_sum"));
    KV_TRY(need(counts, "counts", 4));
    if (sel_mode == kvs::SEL_COBS) {
      KV_TRY(need(k_xi, "k_xi"));
      if (rank < 1 || rank > kvs::COV_MAX_RANK)
        return fail(KV_ERR_INVALID_ARG, "rank = %d outside 1..%d", rank, kvs::COV_MAX_RANK);
    }
  } else if (sel_mode == kvs::SEL_EXACT) {
    KV_TRY(need(K, "K"));
  } else if (sel_mode == kvs::SEL_MEAN16 || sel_mode == kvs::SEL_COBS4) {
    if (shape->dtype != KV_BF16) return fail(KV_ERR_UNSUPPORTED, "bf16-mean scoring is built for bf16 caches only");
    KV_TRY(need(k_mean16, "k_mean"));
    KV_TRY(need(counts, "counts", 4));
    if (sel_mode == kvs::SEL_COBS4) {
      KV_TRY(need(xi4, "codes"));
      KV_TRY(need(xi4_scale, "code_scales", 4));
      if (Uq) KV_TRY(need(Uq, "U", 4));
      if (rank < 1 || rank > kvs::COV_MAX_RANK)
        return fail(KV_ERR_INVALID_ARG, "rank = %d outside 1..%d", rank, kvs::COV_MAX_RANK);
      if (Uq ? (s_dim < 1 || s_dim > shape->D) : s_dim != shape->D)
        return fail(KV_ERR_INVALID_ARG, "s = %d: 1..D with a basis, D without one", s_dim);
    }
  } else {
    if (shape->dtype != KV_BF16) return fail(KV_ERR_UNSUPPORTED, "Quest scoring reads bf16 bounds (bf16 caches only)");
    KV_TRY(need(k_bounds, "k_bounds"));
  }
  KV_TRY(need(block_idx, "block_idx", 4));
  KV_TRY(need(n_kept, "n_kept", 4));
  if (scores) KV_TRY(need(scores, "scores", 4));
  if (k_top < 0) return fail(KV_ERR_INVALID_ARG, "k_top = %d < 0", k_top);
  const int NBcap = (shape->Ncap + shape->block_size - 1) / shape->block_size;
  const int forced = (force_first ? 1 : 0) + (force_last ? 1 : 0);
  const long long need_k = std::min<long long>(NBcap, static_cast<long long>(k_top) + forced);
  if (kmax < need_k)
    return fail(KV_ERR_INVALID_ARG, "kmax = %d < min(NBcap, k_top + forced) = %lld", kmax, need_k);
  const int NBH = shape->B * shape->Hkv;
  if (NBH == 0) return KV_OK;
  kvs::SelParams p{};
  p.q = q;
  p.k_sum = k_sum;
  p.k_bounds = k_bounds;
  p.k_mean16 = k_mean16;
  p.k_xi = k_xi;
  p.cobs_r = rank;
  p.xi4 = xi4;
  p.xi4_scale = xi4_scale;
  p.Uq = Uq;
  p.s_dim = s_dim;
  p.SP = (s_dim + 31) & ~31;
  p.counts = counts;
  p.K = K;
  p.seq_lens = shape->seq_lens;
  p.block_idx = block_idx;
  p.n_kept = n_kept;
  p.scores = scores;
  p.B = shape->B;
  p.Hq = shape->Hq;
  p.Hkv = shape->Hkv;
  p.Ncap = shape->Ncap;
  p.L = shape->block_size;
  p.NBcap = NBcap;
  p.k_top = k_top;
  p.force_first = force_first ? 1 : 0;
  p.force_last = force_last ? 1 : 0;
  p.kmax = kmax;
  p.qscale = scale * 1.4426950408889634f;
  const int G = shape->Hq / shape->Hkv;
  // few pairs: split each pair's blocks over a cluster of CTAs
  const int S = split_select_ctas(sel_mode, k_top, NBH);
  cudaError_t e = S >= 2 ? kvs::launch_select_split(shape->dtype, shape->D, G, sel_mode, p, NBH, S,
                                                    reinterpret_cast<cudaStream_t>(stream))
                         : kvs::launch_select(shape->dtype, shape->D, G, sel_mode, p, NBH,
                                              reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  return KV_OK;
}
}  // namespace

extern "C" {

kv_status kv_select_blocks(const kv_shape* shape, const void* q, float scale, kv_score_mode mode,
                           const float* k_sum, const int32_t* counts, const void* K, int k_top, int force_first,
                           int force_last, int kmax, int32_t* block_idx, int32_t* n_kept, float* scores,
                           kv_stream_t stream) {
  if (mode != KV_SCORE_SUMMARY && mode != KV_SCORE_EXACT_MASS)
    return fail(KV_ERR_INVALID_ARG, "unknown score mode %d", (int)mode);
  return select_any(shape, q, scale, mode == KV_SCORE_SUMMARY ? kvs::SEL_SUMMARY : kvs::SEL_EXACT, k_sum, nullptr,
                    counts, K, k_top, force_first, force_last, kmax, block_idx, n_kept, scores, stream);
}

kv_status kv_select_blocks_mean16(const kv_shape* shape, const void* q, float scale, const void* k_mean,
                                  const int32_t* counts, int k_top, int force_first, int force_last, int kmax,
                                  int32_t* block_idx, int32_t* n_kept, float* scores, kv_stream_t stream) {
  return select_any(shape, q, scale, kvs::SEL_MEAN16, nullptr, nullptr, counts, nullptr, k_top, force_first,
                    force_last, kmax, block_idx, n_kept, scores, stream, nullptr, 0, k_mean);
}

kv_status kv_select_blocks_cobs(const kv_shape* shape, const void* q, float scale, const float* k_sum,
                                const int32_t* counts, const float* k_xi, int rank, int k_top, int force_first,
                                int force_last, int kmax, int32_t* block_idx, int32_t* n_kept, float* scores,
                                kv_stream_t stream) {
  return select_any(shape, q, scale, kvs::SEL_COBS, k_sum, nullptr, counts, nullptr, k_top, force_first, force_last,
                    kmax, block_idx, n_kept, scores, stream, k_xi, rank);
}

kv_status kv_select_blocks_cobs_fp4(const kv_shape* shape, const void* q, float scale, const void* k_mean,
                                    const int32_t* counts, const float* U, int s, const uint8_t* codes,
                                    const float* code_scales, int rank, int k_top, int force_first, int force_last,
                                    int kmax, int32_t* block_idx, int32_t* n_kept, float* scores, kv_stream_t stream) {
  return select_any(shape, q, scale, kvs::SEL_COBS4, nullptr, nullptr, counts, nullptr, k_top, force_first, force_last,
                    kmax, block_idx, n_kept, scores, stream, nullptr, rank, k_mean, codes, code_scales, U, s);
}

kv_status kv_select_blocks_quest(const kv_shape* shape, const void* q, float scale, const void* k_bounds, int k_top,
                                 int force_first, int force_last, int kmax, int32_t* block_idx, int32_t* n_kept,
                                 float* scores, kv_stream_t stream) {
  return select_any(shape, q, scale, kvs::SEL_QUEST, nullptr, k_bounds, nullptr, nullptr, k_top, force_first,
                    force_last, kmax, block_idx, n_kept, scores, stream);
}

kv_status kv_sparse_decode_attn(const kv_shape* shape, const void* q, float scale, const void* K, const void* V,
                                const int32_t* block_idx, const int32_t* n_kept, int kmax, const float* k_sum,
                                const float* v_sum, const int32_t* counts, const float* k_tot, const float* v_tot,
                                int use_tail_proxy, const int32_t* tok_idx, const float* w, int m, float* out,
                                float* lse, void* workspace, size_t ws_bytes, kv_stream_t stream) {
  KV_TRY(check_shape(shape));
  const int mode = tok_idx ? kvs::ATTN_WEIGHTED : kvs::ATTN_BLOCKS;
  return run_attention(shape, q, scale, K, V, block_idx, n_kept, kmax, k_sum, v_sum, counts, k_tot, v_tot,
                       use_tail_proxy, tok_idx, w, m, mode, out, lse, workspace, ws_bytes, stream);
}

kv_status kv_dense_decode_attn(const kv_shape* shape, const void* q, float scale, const void* K, const void* V,
                               float* out, float* lse, void* workspace, size_t ws_bytes, kv_stream_t stream) {
  KV_TRY(check_shape(shape));
  return run_attention(shape, q, scale, K, V, nullptr, nullptr, 0, nullptr, nullptr, nullptr, nullptr, nullptr, 0,
                       nullptr, nullptr, 0, kvs::ATTN_DENSE, out, lse, workspace, ws_bytes, stream);
}

kv_status kv_decode_step(const kv_shape* shape, const void* q, float scale, const void* K, const void* V,
                         const float* k_sum, const float* v_sum, const int32_t* counts, const float* k_tot,
                         const float* v_tot, int k_top, int force_first, int force_last, int kmax, int use_tail_proxy,
                         int32_t* block_idx, int32_t* n_kept, float* scores, float* out, float* lse, void* workspace,
                         size_t ws_bytes, kv_step_how how, kv_stream_t stream) {
  KV_TRY(check_shape(shape));
  if (how != KV_STEP_AUTO && how != KV_STEP_TWO_KERNELS && how != KV_STEP_FUSED)
    return fail(KV_ERR_INVALID_ARG, "unknown decode-step form %d", static_cast<int>(how));
  if (how != KV_STEP_FUSED || !fused_applies(shape, kmax)) {
    KV_TRY(kv_select_blocks(shape, q, scale, KV_SCORE_SUMMARY, k_sum, counts, nullptr, k_top, force_first, force_last,
                            kmax, block_idx, n_kept, scores, stream));
    return kv_sparse_decode_attn(shape, q, scale, K, V, block_idx, n_kept, kmax, k_sum, v_sum, counts, k_tot, v_tot,
                                 use_tail_proxy, nullptr, nullptr, 0, out, lse, workspace, ws_bytes, stream);
  }
  // the selection's argument checks (the attention's follow in run_attention)
  if (!std::isfinite(scale)) return fail(KV_ERR_INVALID_ARG, "scale is not finite");
  KV_TRY(need(k_sum, "k_sum"));
  KV_TRY(need(counts, "counts", 4));
  KV_TRY(need(block_idx, "block_idx", 4));
  KV_TRY(need(n_kept, "n_kept", 4));
  if (scores) KV_TRY(need(scores, "scores", 4));
  if (k_top < 0) return fail(KV_ERR_INVALID_ARG, "k_top = %d < 0", k_top);
  const int NBcap = (shape->Ncap + shape->block_size - 1) / shape->block_size;
  const int forced = (force_first ? 1 : 0) + (force_last ? 1 : 0);
  const long long need_k = std::min<long long>(NBcap, static_cast<long long>(k_top) + forced);
  if (kmax < need_k)
    return fail(KV_ERR_INVALID_ARG, "kmax = %d < min(NBcap, k_top + forced) = %lld", kmax, need_k);
  const FusedSel fs{k_top, force_first, force_last, block_idx, n_kept, scores};
  return run_attention(shape, q, scale, K, V, block_idx, n_kept, kmax, k_sum, v_sum, counts, k_tot, v_tot,
                       use_tail_proxy, nullptr, nullptr, 0, kvs::ATTN_BLOCKS, out, lse, workspace, ws_bytes, stream,
                       &fs);
}

size_t kv_workspace_bytes(const kv_shape* shape) {
  if (!shape || shape->Hkv < 1 || shape->Hq < shape->Hkv || shape->B < 0 || shape->D < 1) return 0;
  const int G = shape->Hq / shape->Hkv;
  return kvs::ws_total(shape->B * shape->Hkv, G, shape->D);
}

kv_status kv_workspace_init(void* workspace, size_t ws_bytes, kv_stream_t stream) {
  KV_TRY(need(workspace, "workspace", 256));
  if (ws_bytes < 256) return fail(KV_ERR_INVALID_ARG, "workspace too small (%zu bytes)", ws_bytes);
  cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "workspace memset");
  return KV_OK;
}

kv_status kv_workspace_status(const void* workspace, uint32_t* status_out, kv_stream_t stream) {
  KV_TRY(need(workspace, "workspace", 256));
  if (!status_out) return fail(KV_ERR_INVALID_ARG, "status_out is NULL");
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t v = 0;
  e = cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status copy");
  *status_out = v;
  if (v != 0) return fail(KV_ERR_DEVICE_CHECK, "device checks failed: status 0x%x", v);
  return KV_OK;
}

const char* kv_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"

namespace kvs {
// Lets other translation units of the library report a message through
// kv_last_error().
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace kvs
