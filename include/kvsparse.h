/*
 * kvsparse.h -- C ABI of the reduced-KV softmax decode-attention library
 * (libkvsparse.so, CUDA kernels for sm_100a).
 *
 * The method, per decode step of one layer:
 *   1. Once after prefill, every block of L cached tokens is summarised by its
 *      key sum, value sum and token count (kv_build_block_summaries).
 *   2. Each KV head scores its blocks for the current query group and keeps the
 *      top-k by the GQA-normalised group score (kv_select_blocks).
 *   3. Attention runs exactly over the kept blocks' tokens plus one count-aware
 *      proxy token standing for the unread tail (kv_sparse_decode_attn), or over
 *      an explicitly weighted coreset; kv_dense_decode_attn is exact attention
 *      over every token, the baseline.
 *
 * Conventions shared by every entry point
 *   - Pointers named K, V, q, k_sum, ... are DEVICE pointers unless stated.
 *     The library calls no allocator; the caller owns every buffer (the one
 *     exception, kv_sparse_decode_attn_noalloc, uses a fixed array inside the
 *     library instead of a caller workspace).
 *   - Layouts are dense row-major, C order:
 *       q        [B][Hq][D]         dtype of the shape
 *       K, V     [B][Hkv][Ncap][D]  dtype of the shape
 *       out      [B][Hq][D]         fp32
 *       lse      [B][Hq]            fp32, natural log of the softmax normaliser
 *     Query head g reads KV head g / G, G = Hq / Hkv.
 *   - Every call is asynchronous on `stream` and returns before the kernels run.
 *     Argument errors are reported BEFORE anything is launched.
 *   - Sizes: D in {64, 128}; 1 <= G <= 8; L (block_size) in {16, 32, 64, 128};
 *     dtype bf16 or fp32; NBcap = ceil(Ncap / L) <= 4096. Other shapes return
 *     KV_ERR_UNSUPPORTED. Every device pointer must be 16-byte aligned.
 *   - Values that live on the device (seq_lens, block indices, token indices)
 *     cannot be checked by the host. The kernels check them and never read out
 *     of bounds: a bad entry is skipped and a bit is set in the workspace status
 *     word (kv_workspace_status), after which results are unspecified.
 *   - Thread safety: calls are re-entrant. The last error message is kept per
 *     host thread (kv_last_error). Calls that share one workspace must be
 *     ordered on the device (same stream, or events); overlapping ones race.
 */
#ifndef KVSPARSE_H
#define KVSPARSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* kv_stream_t;

typedef enum {
  KV_OK = 0,
  KV_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size; nothing launched  */
  KV_ERR_UNSUPPORTED = 2,   /* valid but not built: D, G, L, dtype or NBcap         */
  KV_ERR_CUDA = 3,          /* a CUDA call or launch failed (see kv_last_error)      */
  KV_ERR_DEVICE_CHECK = 4   /* kv_workspace_status found a device-side check failed  */
} kv_status;

typedef enum { KV_BF16 = 0, KV_F32 = 1 } kv_dtype;

typedef enum {
  KV_SCORE_SUMMARY = 0,     /* first-order mean-pool score from the block sums       */
  KV_SCORE_EXACT_MASS = 1   /* exact block log-mass from all block keys (OSA)        */
} kv_score_mode;

/* Device-status bits written into the workspace by the attention kernels. */
#define KV_DEV_BAD_BLOCK_INDEX  0x1u  /* block index out of range or not ascending   */
#define KV_DEV_BAD_TOKEN_INDEX  0x2u  /* coreset token index outside [0, seq_len)    */
#define KV_DEV_BAD_SEQ_LEN      0x4u  /* seq_len outside [0, Ncap]                   */
#define KV_DEV_BAD_N_KEPT       0x8u  /* n_kept outside [0, kmax]                    */
#define KV_DEV_WAIT_TIMEOUT     0x10u /* a bounded wait on a copy gave up            */

typedef struct {
  int B;                    /* sequences in the batch, >= 0                          */
  int Hq;                   /* query heads                                           */
  int Hkv;                  /* KV heads; Hq % Hkv == 0                               */
  int D;                    /* head dimension                                        */
  int Ncap;                 /* allocated tokens per (sequence, KV head), >= 1        */
  int block_size;           /* L, tokens per block                                   */
  kv_dtype dtype;           /* element type of q, K and V                            */
  const int32_t* seq_lens;  /* device [B]: tokens actually cached, 0..Ncap           */
} kv_shape;

/*
 * kv_build_block_summaries -- per-block key sum, value sum and token count.
 *
 * Source: "COBS: Cumulant Order Block Sparse Attention", the affine score (18)
 * (mean-pool summary: phi_b = block mean key, a_b = ln L) and the paragraph that
 * stores the mean key per block; "OpenAttention reads 1% of the KV cache --
 * Count-aware tail proxy" (the proxy needs the unread tail's mean key and value,
 * obtained from the totals minus the kept blocks' sums).
 *
 * Writes, for every (b, h, block) with block < NBcap:
 *   k_sum, v_sum [B][Hkv][NBcap][D] fp32  sums over the block's tokens < seq_len
 *   counts       [B][NBcap] int32         min(L, seq_len - block*L) clamped at 0
 *   k_tot, v_tot [B][Hkv][D] fp32         sums over all tokens < seq_len
 * Blocks at or past ceil(seq_len / L) get zero sums and count 0. Accumulation is
 * fp32; the totals are summed from the block sums in a fixed order, so results
 * are bit-reproducible. Run once after prefill (and again if the cache changes).
 */
kv_status kv_build_block_summaries(const kv_shape* shape, const void* K, const void* V,
                                   float* k_sum, float* v_sum, int32_t* counts,
                                   float* k_tot, float* v_tot, kv_stream_t stream);

/*
 * kv_select_blocks -- per-KV-head block choice for one decode step.
 *
 * Source: "COBS: Cumulant Order Block Sparse Attention" -- Equation (5), the
 * GQA-normalised group score (a sum over the group's query heads of per-head
 * block softmax probabilities, normaliser Z^(g,h) of (5)); the first-order
 * mean-pool estimate of ln m_b (text after Equation (8), affine score (18)); the
 * OSA paragraph for KV_SCORE_EXACT_MASS.
 *
 *   summary mode:  s[g,b] = scale * q_g . (k_sum_b / n_b) + ln n_b
 *   exact mode:    s[g,b] = ln sum_{r in b} exp(scale * q_g . k_r)   (reads all K)
 *   S[b] = sum_{g in group} exp(s[g,b] - ln sum_b' exp(s[g,b']))      over valid b'
 *
 * Forced blocks (block 0 if force_first, block ceil(n/L)-1 if force_last) are
 * always kept and do not compete. The other valid blocks are ranked by
 * (S descending, block index ascending) and the first min(k_top, candidates)
 * are kept.
 *
 *   q          device [B][Hq][D], dtype of the shape
 *   scale      softmax scale applied to q.k (e.g. 1/sqrt(D))
 *   k_sum      device, from kv_build_block_summaries (summary mode; may be NULL
 *              in exact mode)
 *   counts     device [B][NBcap] from kv_build_block_summaries (both modes)
 *   K          device cache (exact mode only; may be NULL in summary mode)
 *   kmax       row stride of block_idx; must be >= min(NBcap, k_top + forced)
 *   block_idx  device out [B][Hkv][kmax] int32: kept block indices, ascending;
 *              entries past n_kept are left unchanged
 *   n_kept     device out [B][Hkv] int32
 *   scores     device out [B][Hkv][NBcap] fp32 S[b] (0 for invalid blocks), or NULL
 */
kv_status kv_select_blocks(const kv_shape* shape, const void* q, float scale,
                           kv_score_mode mode, const float* k_sum, const int32_t* counts,
                           const void* K, int k_top, int force_first, int force_last,
                           int kmax, int32_t* block_idx, int32_t* n_kept, float* scores,
                           kv_stream_t stream);

/*
 * kv_build_block_key_means -- the block mean keys at bf16 precision, the block
 * summary COBS stores for first-order scoring. Source: "COBS: Cumulant Order
 * Block Sparse Attention", the quantisation paragraph (the block mean is kept at
 * bf16 precision) and the mean-pool score after Equation (8).
 *
 *   k_sum   device [B][Hkv][NBcap][D] fp32 key sums (kv_build_block_summaries)
 *   counts  device [B][NBcap] int32 token counts (same call)
 *   k_mean  device out [B][Hkv][NBcap][D] bf16, 16-byte aligned: the correctly
 *           rounded fp32 quotient k_sum / n_b rounded to the nearest bf16 (ties
 *           to even); zeros where n_b = 0.
 * Half the bytes of the fp32 sums for the scorer to stream. Run once after
 * prefill (after kv_build_block_summaries, on the same stream).
 */
kv_status kv_build_block_key_means(const kv_shape* shape, const float* k_sum, const int32_t* counts,
                                   void* k_mean, kv_stream_t stream);

/*
 * kv_select_blocks_mean16 -- kv_select_blocks (summary mode) scoring from the
 * bf16 block means instead of the fp32 sums. Source: "COBS: Cumulant Order Block
 * Sparse Attention", text after Equation (8), Equation (5), the quantisation
 * paragraph:
 *
 *   s[g,b] = scale * q_g . k_mean_b + ln n_b        (k_mean_b the bf16 mean)
 *   S[b]   = sum_{g in group} exp(s[g,b] - ln sum_b' exp(s[g,b']))  over valid b'
 *
 * Reads NBcap * (2 D + 4) bytes per (sequence, KV head) instead of
 * NBcap * (4 D + 4). The rounding of the mean moves each logit by at most
 * scale * sum_d |q_d| |mean_d| 2^-8, so the kept set can differ from the
 * fp32-sum ranking where two candidates score that close. Forcing, ranking,
 * kmax, block_idx, n_kept and scores are as in kv_select_blocks. bf16 caches only
 * (KV_ERR_UNSUPPORTED otherwise).
 */
kv_status kv_select_blocks_mean16(const kv_shape* shape, const void* q, float scale, const void* k_mean,
                                  const int32_t* counts, int k_top, int force_first, int force_last,
                                  int kmax, int32_t* block_idx, int32_t* n_kept, float* scores,
                                  kv_stream_t stream);

/*
 * kv_build_wildcat_coreset -- a weighted coreset of every (sequence, KV head)'s
 * keys, for the weighted-coreset mode of kv_sparse_decode_attn. Source:
 * "WildCat: Near-Linear Attention in Theory and Practice", abstract (the coreset is
 * selected by randomly pivoted Cholesky and weighted to minimise the
 * reconstruction error). Readings: the kernel is exp(scale k_i . k_j) on the first
 * seq_len keys (evaluated shifted by scale * max_i |k_i|^2; the shift cancels);
 * the weights minimise the kernel distance between the sum over all tokens and the
 * weighted coreset (A_SS w = A_{S,:} 1); a negative weight is clipped to 0.
 *
 *   K        device cache [B][Hkv][Ncap][D] (bf16 or fp32), 16-byte aligned
 *   scale    the softmax scale, > 0
 *   m        coreset size per (sequence, KV head), 1 <= m <= min(4096, Ncap)
 *   ctas_per_pair  CTAs (a thread-block cluster) per (sequence, KV head), 1..8, or 0
 *            for min(8, SMs / pairs); the pivots differ between cluster sizes only
 *            where fp32 rounding of the running sums decides a draw
 *   u        device [B][Hkv][m] fp32 uniforms in (0, 1): u[.][t] draws pivot t as the
 *            first token whose running sum of the residual diagonal reaches u times
 *            its total (randomness is an input, so results are reproducible)
 *   tok_idx  device out [B][Hkv][m] int32: the pivots in the order drawn
 *   w        device out [B][Hkv][m] fp32: their weights (>= 0)
 *   n_sel    device out [B][Hkv] int32 (or NULL): pivots drawn; fewer than m when
 *            the residual vanishes (entries past it: index 0, weight 0, which the
 *            attention leaves out)
 *   workspace  device, kv_wildcat_workspace_bytes(shape, m) bytes, 16-byte aligned
 *            (per (sequence, KV head): the factor and the residual diagonal, m + 1
 *            rows of Ncap floats with Ncap rounded up to a multiple of 32, and 8 x m
 *            partial column sums)
 * The cluster of a pair runs the m pivot steps (each a draw from the residual
 * diagonal and one pass over the keys for a residual kernel column); run once after
 * prefill. Bytes per pair and step: the n keys plus t + 1 factor rows of n floats.
 * KV_ERR_INVALID_ARG for bad sizes or pointers, KV_ERR_UNSUPPORTED for D not 64/128
 * or Ncap above 2^20.
 */
kv_status kv_build_wildcat_coreset(const kv_shape* shape, const void* K, float scale, int m,
                                   int ctas_per_pair, const float* u, int32_t* tok_idx, float* w, int32_t* n_sel,
                                   void* workspace, size_t ws_bytes, kv_stream_t stream);

/* Workspace bytes kv_build_wildcat_coreset needs for this shape and m (0 if invalid). */
size_t kv_wildcat_workspace_bytes(const kv_shape* shape, int m);

/*
 * kv_build_block_bounds -- per-block, per-channel key minimum and maximum (the
 * axis-aligned bounding box of each block's keys). Source: "COBS: Cumulant Order
 * Block Sparse Attention", the Quest paragraph (a block is scored by the largest
 * inner product any point of its key box could reach).
 *
 *   K         device cache [B][Hkv][Ncap][D] bf16 (bf16 caches only)
 *   k_bounds  device out [B][Hkv][NBcap][D][2] bf16: (min, max) of channel d over
 *             the block's tokens < seq_len, as adjacent pairs; blocks at or past
 *             ceil(seq_len / L) get zeros. Must be 16-byte aligned. The bounds
 *             are exact (min and max of bf16 values are bf16 values).
 * Returns KV_ERR_UNSUPPORTED for an fp32 cache. Run once after prefill.
 */
kv_status kv_build_block_bounds(const kv_shape* shape, const void* K, void* k_bounds,
                                kv_stream_t stream);

/*
 * kv_select_blocks_quest -- kv_select_blocks with the Quest box bound as the
 * per-head block logit. Source: "COBS: Cumulant Order Block Sparse Attention",
 * the Quest paragraph and Equation (5):
 *
 *   s[g,b] = scale * sum_d max(q_g[d] * min_b[d], q_g[d] * max_b[d])
 *   S[b]   = sum_{g in group} exp(s[g,b] - ln sum_b' exp(s[g,b']))  over valid b'
 *
 * The bound carries no ln n_b count term (the paragraph scores the box's largest
 * inner product alone). Forcing, ranking, kmax, block_idx, n_kept and scores are
 * as in kv_select_blocks. k_bounds: kv_build_block_bounds output. bf16 only
 * (KV_ERR_UNSUPPORTED otherwise).
 */
kv_status kv_select_blocks_quest(const kv_shape* shape, const void* q, float scale,
                                 const void* k_bounds, int k_top, int force_first,
                                 int force_last, int kmax, int32_t* block_idx,
                                 int32_t* n_kept, float* scores, kv_stream_t stream);

/*
 * kv_build_block_cov_factors -- per-block covariance factors for second-order
 * block scoring. Source: "COBS: Cumulant Order Block Sparse Attention" -- the
 * cumulant expansion (8) truncated at second order and the low-rank spectral
 * decomposition (13) of the within-block key covariance.
 *
 *   K      device cache [B][Hkv][Ncap][D] (bf16 or fp32)
 *   rank   r, 1..8: eigendirections kept per block
 *   k_xi   device out [B][Hkv][NBcap][r][D] fp32, 16-byte aligned: xi_i =
 *          sqrt(lambda_i) u_i for the r largest eigenvalues lambda_i (descending)
 *          of the block's population covariance (sum over its n_b keys of
 *          (k - mean)(k - mean)^T / n_b). The sign of each xi_i is arbitrary;
 *          directions past the covariance's rank, blocks with fewer than two
 *          keys and blocks at or past ceil(seq_len / L) are zero.
 * block_size must be <= 64 (KV_ERR_UNSUPPORTED otherwise). Eigenvectors come from
 * a float64 Jacobi diagonalisation of each block's Gram matrix. Run once after
 * prefill (and again if the cache changes).
 */
kv_status kv_build_block_cov_factors(const kv_shape* shape, const void* K, int rank, float* k_xi,
                                     kv_stream_t stream);

/*
 * kv_select_blocks_cobs -- kv_select_blocks with the second-order block logit.
 * Source: "COBS: Cumulant Order Block Sparse Attention", text after Equation (8)
 * (the second-order estimator), the low-rank form (13) and Equation (5):
 *
 *   s[g,b] = scale * q_g . (k_sum_b / n_b) + (scale^2 / 2) sum_i (q_g . xi_bi)^2
 *            + ln n_b
 *   S[b]   = sum_{g in group} exp(s[g,b] - ln sum_b' exp(s[g,b']))  over valid b'
 *
 * k_sum, counts: kv_build_block_summaries output; k_xi, rank: from
 * kv_build_block_cov_factors. Forcing, ranking, kmax, block_idx, n_kept and
 * scores are as in kv_select_blocks.
 */
kv_status kv_select_blocks_cobs(const kv_shape* shape, const void* q, float scale, const float* k_sum,
                                const int32_t* counts, const float* k_xi, int rank, int k_top,
                                int force_first, int force_last, int kmax, int32_t* block_idx,
                                int32_t* n_kept, float* scores, kv_stream_t stream);

/*
 * The stored second-order descriptor. Source: "COBS: Cumulant Order Block Sparse
 * Attention" -- the subspace paragraph (keep each block's covariance only within
 * the span U_Q of the top s eigenvectors of the query second moment E[q q^T], store
 * the rank-r factors of B_b = U_Q^T Sigma_b U_Q, score with the projected query
 * U_Q^T q; s set from the rank capturing 90% of the query spectral energy, averaged
 * over heads) and the quantisation paragraph (the factors in E2M1 FP4 with one fp32
 * scale per factor, the block mean at bf16).
 *
 * kv_build_query_basis -- per KV head h, the eigenvectors of the query second moment
 * C_h = mean over the Nc calibration positions and the group's Hq / Hkv query heads
 * of q q^T (float64 accumulation and Jacobi diagonalisation).
 *   Qc       device [Nc][Hq][D] (bf16 or fp32 per dtype), 16-byte aligned
 *   evecs    device out [Hkv][D][D] fp32: row j of head h is the unit eigenvector of
 *            evals[h][j] (sign arbitrary)
 *   evals    device out [Hkv][D] fp32, descending (ties to the lower index)
 *   workspace  device, kv_query_basis_workspace_bytes(Hkv, D) bytes (float64 scratch)
 * D must be 64 or 128 (KV_ERR_UNSUPPORTED); Hq a multiple of Hkv.
 */
kv_status kv_build_query_basis(const void* Qc, kv_dtype dtype, int Nc, int Hq, int Hkv, int D, float* evecs,
                               float* evals, void* workspace, size_t ws_bytes, kv_stream_t stream);
size_t kv_query_basis_workspace_bytes(int Hkv, int D);

/*
 * kv_query_subspace_rank -- host function: s = ceil(mean over heads of s_h), s_h the
 * smallest count of leading eigenvalues of head h whose sum reaches `energy` (0..1]
 * of the head's total. evals: HOST [Hkv][D] fp32, descending (kv_build_query_basis's,
 * copied back). Returns s, or -1 for bad arguments.
 */
int kv_query_subspace_rank(const float* evals, int Hkv, int D, double energy);

/*
 * kv_build_block_cov_factors_ss -- per block, the r largest eigenpairs of
 * B_b = U Sigma_b U^T as scaled eigenvectors xi_i = sqrt(lambda_i) u_i (s values),
 * Sigma_b the population covariance of the block's keys.
 *   U      device [Hkv][s][D] fp32: rows the subspace basis (the first s rows of
 *          kv_build_query_basis's evecs per head)
 *   s      1..D
 *   xi_ss  device out [B][Hkv][NBcap][rank][SP] fp32, SP = s rounded up to 32 (values
 *          past s, directions past B_b's rank, blocks with fewer than two keys and
 *          blocks past the sequence are zero), 16-byte aligned
 * block_size <= 64 and D in {64, 128} (KV_ERR_UNSUPPORTED otherwise); rank 1..8.
 */
kv_status kv_build_block_cov_factors_ss(const kv_shape* shape, const void* K, const float* U, int s, int rank,
                                        float* xi_ss, kv_stream_t stream);

/*
 * kv_quantize_fp4 -- E2M1 FP4 codes of nvec vectors of len fp32 values, one fp32 scale
 * per vector: scale = max|x| / 6; each x_j / scale (an IEEE fp32 division) goes to
 * the nearest of the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6, a tie to the code with
 * mantissa bit 0, the sign in bit 3 (zero is code 0).
 *   x       device [nvec][len] fp32, 16-byte aligned; len a multiple of 32, <= 4096
 *   codes   device out [nvec][len / 2] bytes: element 2j in the low nibble
 *   scales  device out [nvec] fp32 (0 for an all-zero vector)
 */
kv_status kv_quantize_fp4(const float* x, long long nvec, int len, uint8_t* codes, float* scales,
                          kv_stream_t stream);

/*
 * kv_select_blocks_cobs_fp4 -- kv_select_blocks with the second-order block logit read
 * from the stored descriptor:
 *   s[g,b] = scale * q_g . mean_b + (scale^2 / 2) sum_i (q~_g . xi_bi)^2 + ln n_b,
 *   q~_g = U q_g (s values; the full space, q~ = q, when U is NULL and s = D),
 *   xi_bi = code_scales[b][i] * e2m1(codes[b][i]),
 * and Equation (5) over the group's heads as in kv_select_blocks.
 *   k_mean       device [B][Hkv][NBcap][D] bf16 block means (kv_build_block_key_means)
 *   counts       device [B][NBcap] int32 (kv_build_block_summaries)
 *   U, s         device [Hkv][s][D] fp32 basis, or NULL with s = D
 *   codes        device [B][Hkv][NBcap][rank][SP / 2] E2M1 codes (kv_quantize_fp4 of
 *                kv_build_block_cov_factors_ss's output, or of full-space factors),
 *                SP = s rounded up to 32, 16-byte aligned
 *   code_scales  device [B][Hkv][NBcap][rank] fp32
 * bf16 caches only (KV_ERR_UNSUPPORTED otherwise); rank 1..8. Forcing, ranking, kmax,
 * block_idx, n_kept and scores are as in kv_select_blocks.
 */
kv_status kv_select_blocks_cobs_fp4(const kv_shape* shape, const void* q, float scale, const void* k_mean,
                                    const int32_t* counts, const float* U, int s, const uint8_t* codes,
                                    const float* code_scales, int rank, int k_top, int force_first, int force_last,
                                    int kmax, int32_t* block_idx, int32_t* n_kept, float* scores, kv_stream_t stream);

/*
 * Query-guided clusters with one proxy each and an error-gated read budget. Source:
 * "OpenAttention reads 1% of the KV cache" -- section "Three helpers that make the
 * proxy accurate" (QGC: keys projected onto the top eigenvectors of the queries and
 * clustered by k-means in 16 dimensions once after prefill; ErrorGate: the exact-read
 * budget split across clusters in proportion to the error each proxy would leave,
 * estimated from cached mean and variance tokens at 1.5 KV rows a cluster, charged
 * to the read; QGS: the top tokens inside each cluster from low-bit projections) and
 * section "Skipping reviews without losing the verdict" (the count-aware mean proxy;
 * a proxy's weight error is its mass times the spread of the weights it hides).
 * A decode step is kv_select_qgc, kv_sparse_decode_attn in weighted mode over the
 * read list, then kv_merge_qgc_proxies.
 *
 * kv_build_qgc -- once after prefill, per (sequence, KV head):
 *   P        device [Hkv][16][D] fp32: the projection rows (the 16 leading rows of
 *            kv_build_query_basis's evecs per head)
 *   C        clusters, 1..64 (min(C, seq_len) are used); iters: Lloyd iterations, 1..100
 *   z16      device out [B][Hkv][Ncap][16] bf16: P k (fp32, then bf16) in member
 *            order: entry m is the projection of token perm[m] (zero past seq_len),
 *            so every cluster's projections are one contiguous run
 *   labels   device out [B][Hkv][Ncap] int32: cluster of each token (-1 past seq_len)
 *   perm     device out [B][Hkv][Ncap] int32: the tokens grouped by cluster, ascending
 *            inside a cluster (-1 past seq_len); offs: [B][Hkv][C + 1] int32 starts
 *   counts   device out [B][Hkv][C] int32
 *   k_sum, v_sum, k_sq  device out [B][Hkv][C][D] fp32: per cluster the key and value
 *            sums and the per-channel key sum of squares (the mean and variance tokens)
 *   workspace  device, kv_qgc_workspace_bytes(shape) bytes (fp32 coordinates)
 * k-means: float64, starts at tokens ((2c + 1) n) // (2C'), ties to the lower cluster,
 * the clusters are the last assignment.
 */
kv_status kv_build_qgc(const kv_shape* shape, const void* K, const void* V, const float* P, int C, int iters,
                       void* z16, int32_t* labels, int32_t* perm, int32_t* offs, int32_t* counts, float* k_sum,
                       float* v_sum, float* k_sq, void* workspace, size_t ws_bytes, kv_stream_t stream);
size_t kv_qgc_workspace_bytes(const kv_shape* shape);

/*
 * kv_select_qgc -- per query: per cluster c, from the mean and variance tokens,
 *   mu_g = scale q_g . mean_c, s2_g = scale^2 sum_d q_gd^2 var_cd,
 *   E_c = sum_g n_c e^mu_g (e^(s2_g / 2) - 1) / sum_c' n_c' e^(mu_g + s2_g / 2)
 * (the mean-logit proxy's shortfall against the cluster's expected mass under normal
 * logits, per head normalised and summed over the group); the exact-read budget
 * R = floor(budget n) - ceil(1.5 live clusters) split as r_c = min(n_c, floor(R E_c /
 * sum E)); in every cluster the r_c tokens of largest t_i = sum_g exp(scale (P q_g) .
 * z16_i - LSE_g) (ties to the lower index).
 *   budget     read fraction in [0, 1]; max_read >= floor(budget Ncap)
 *   tok_idx, w device out [B][Hkv][max_read]: the read tokens grouped by cluster with
 *              weight 1, then index 0 / weight 0 (kv_sparse_decode_attn's weighted mode)
 *   n_read     device out [B][Hkv] int32
 *   proxy_k, proxy_v  device out [B][Hkv][C][D] fp32: per cluster the mean key and
 *              value of its unread tokens (cluster sums minus the read rows)
 *   proxy_n    device out [B][Hkv][C] int32: unread tokens per cluster (0: no proxy)
 *   workspace  device, kv_qgc_select_workspace_bytes(shape) bytes (token scores)
 * q bf16 or fp32 per shape->dtype; G <= 8.
 */
kv_status kv_select_qgc(const kv_shape* shape, const void* q, float scale, const float* P, int C, const void* z16,
                        const int32_t* perm, const int32_t* offs, const int32_t* counts, const float* k_sum,
                        const float* v_sum, const float* k_sq, const void* K, const void* V, float budget,
                        int max_read, int32_t* tok_idx, float* w, int32_t* n_read, float* proxy_k, float* proxy_v,
                        int32_t* proxy_n, void* workspace, size_t ws_bytes, kv_stream_t stream);
size_t kv_qgc_select_workspace_bytes(const kv_shape* shape);

/*
 * kv_merge_qgc_proxies -- folds the cluster proxies into the attention over the read
 * tokens, in place: with the read tokens' out [B][Hq][D] and lse [B][Hq] (from
 * kv_sparse_decode_attn; lse is required) and proxy logits l_c = scale q . proxy_k_c +
 * ln proxy_n_c, out <- (e^lse out + sum_c e^l_c proxy_v_c) / (e^lse + sum_c e^l_c) and
 * lse <- ln(e^lse + sum_c e^l_c), evaluated with a max shift.
 */
kv_status kv_merge_qgc_proxies(const kv_shape* shape, const void* q, float scale, int C, const float* proxy_k,
                               const float* proxy_v, const int32_t* proxy_n, float* out, float* lse,
                               kv_stream_t stream);

/*
 * kv_sparse_decode_attn -- softmax attention over a reduced KV cache.
 *
 * Block mode (tok_idx == NULL). Source: "OpenAttention reads 1% of the KV cache
 * -- Count-aware tail proxy", section "Skipping reviews without losing the
 * verdict": exact attention over the kept blocks' tokens plus, if use_tail_proxy,
 * one virtual token for the n_T unread tokens whose value is their mean value and
 * whose logit is scale * q . (their mean key) + ln n_T (their mean logit plus the
 * log of their count). The tail means come from the block sums:
 * (k_tot - sum of kept k_sum) / n_T. With use_tail_proxy = 0 the tail is dropped
 * and the kept tokens are renormalised (top-k discard).
 *   block_idx [B][Hkv][kmax], n_kept [B][Hkv]: kept blocks, strictly ascending,
 *   each < ceil(seq_len / L) (kv_select_blocks output, or the caller's own).
 *   k_sum, v_sum, counts, k_tot, v_tot: kv_build_block_summaries output; needed
 *   only when use_tail_proxy != 0 (else may be NULL).
 *
 * Weighted-coreset mode (tok_idx != NULL). Source: "WildCat: Near-Linear
 * Attention in Theory and Practice", abstract: attention over a small weighted
 * coreset, token i entering the softmax with logit scale * q . k_i + ln w_i.
 *   tok_idx [B][Hkv][m] int32 token positions (< seq_len), w [B][Hkv][m] fp32
 *   weights (>= 0; 0 excludes the token). No proxy; block arguments ignored.
 *
 *   out [B][Hq][D] fp32; lse [B][Hq] fp32 or NULL. A head with no token and no
 *   proxy gets out = 0 and lse = -inf.
 *   workspace: device, >= kv_workspace_bytes(shape) bytes, zeroed once before
 *   its first use (kv_workspace_init); every call leaves it ready for the next.
 */
kv_status kv_sparse_decode_attn(const kv_shape* shape, const void* q, float scale,
                                const void* K, const void* V,
                                const int32_t* block_idx, const int32_t* n_kept, int kmax,
                                const float* k_sum, const float* v_sum, const int32_t* counts,
                                const float* k_tot, const float* v_tot, int use_tail_proxy,
                                const int32_t* tok_idx, const float* w, int m,
                                float* out, float* lse, void* workspace, size_t ws_bytes,
                                kv_stream_t stream);

/*
 * kv_dense_decode_attn -- exact softmax attention over every cached token, the
 * baseline the reduced path is measured against. Source: "COBS: Cumulant Order
 * Block Sparse Attention", the read-traffic accounting ("Dense reads the whole
 * KV cache"); "OpenAttention reads 1% of the KV cache", section "The news" (the
 * decode-attention speed comparison against dense attention).
 * Arguments as in kv_sparse_decode_attn.
 */
kv_status kv_dense_decode_attn(const kv_shape* shape, const void* q, float scale,
                               const void* K, const void* V, float* out, float* lse,
                               void* workspace, size_t ws_bytes, kv_stream_t stream);

/*
 * kv_decode_step -- one decode step of the reduced path: kv_select_blocks in
 * summary mode followed by kv_sparse_decode_attn in block mode, with the same
 * results. Sources: as for those two calls ("COBS: Cumulant Order Block Sparse
 * Attention", Equation (5) and the mean-pool score after Equation (8);
 * "OpenAttention reads 1% of the KV cache", "Skipping reviews without losing the
 * verdict" for the tail proxy).
 *   Arguments: those of kv_select_blocks (k_sum, counts, k_top, force_first,
 *   force_last, kmax, block_idx and n_kept as outputs, scores optional) and of
 *   kv_sparse_decode_attn in block mode (v_sum, k_tot, v_tot, use_tail_proxy,
 *   out, lse, workspace). block_idx / n_kept are written and then read by the
 *   attention, so they must not be read by another stream until the call's work
 *   completes.
 *   how: KV_STEP_TWO_KERNELS (also KV_STEP_AUTO) launches the selector and the
 *   attention kernel back to back (the attention grid is scheduled while the
 *   selector finishes). KV_STEP_FUSED runs one kernel in which each CTA selects
 *   the blocks of one (sequence, KV head) and then attends to them (no cross-CTA
 *   dependency); it applies to bf16 caches on the tensor-core path when the
 *   per-CTA layout fits (three ring slots: G <= 4 at D = 128; block logits of the
 *   pair in one 18 KB slot) and kmax * block_size is a multiple of 32, and falls
 *   back to two kernels otherwise. On B200 the two-kernel form is the faster one
 *   at the shapes measured, so it is the default.
 *   Errors: the union of the two calls' argument errors, reported before any
 *   launch; KV_ERR_INVALID_ARG for an unknown `how`.
 */
typedef enum { KV_STEP_AUTO = 0, KV_STEP_TWO_KERNELS = 1, KV_STEP_FUSED = 2 } kv_step_how;

kv_status kv_decode_step(const kv_shape* shape, const void* q, float scale, const void* K, const void* V,
                         const float* k_sum, const float* v_sum, const int32_t* counts, const float* k_tot,
                         const float* v_tot, int k_top, int force_first, int force_last, int kmax,
                         int use_tail_proxy, int32_t* block_idx, int32_t* n_kept, float* scores, float* out,
                         float* lse, void* workspace, size_t ws_bytes, kv_step_how how, kv_stream_t stream);

/*
 * kv_workspace_bytes -- device workspace the attention entry points need for
 * this shape (split partial results, arrival counters, a status word). The size
 * depends only on B, Hkv, G and D. Returns 0 for an invalid shape pointer.
 */
size_t kv_workspace_bytes(const kv_shape* shape);

/*
 * kv_workspace_init -- zeroes the counters and the status word of a workspace
 * (an async memset on `stream`). Needed once after allocation; calls leave the
 * counters at zero, and the status word keeps its bits until the next init.
 */
kv_status kv_workspace_init(void* workspace, size_t ws_bytes, kv_stream_t stream);

/*
 * kv_workspace_status -- synchronises `stream`, then copies the workspace status
 * word (KV_DEV_* bits) to *status_out (host pointer). Returns KV_ERR_DEVICE_CHECK
 * if any bit is set, KV_OK otherwise.
 */
kv_status kv_workspace_status(const void* workspace, uint32_t* status_out, kv_stream_t stream);

/*
 * kv_sparse_decode_attn_noalloc -- kv_sparse_decode_attn for callers that cannot
 * allocate device memory (a plugin or operator that is handed only its inputs and
 * outputs, or a process that forbids allocation once it is serving). The pages
 * have no counterpart of this entry point: it only changes where the kernel's
 * scratch lives.
 *
 * Same arguments and results as kv_sparse_decode_attn, without the workspace:
 * the scratch comes from a fixed 16 MiB array inside the library (held on every
 * GPU that loads it, until exit). Shapes whose kv_workspace_bytes exceeds 16 MiB
 * are rejected with KV_ERR_INVALID_ARG. The first call on a device looks up the
 * array's device address (make it before any stream capture). Each call checks
 * every argument first (a rejected call enqueues nothing), then clears the
 * array's counters with an async memset on `stream`; calls share the array,
 * so calls that overlap on the GPU race -- order them on one stream or with
 * events. Nothing is allocated. Device-check status bits are not reported.
 */
kv_status kv_sparse_decode_attn_noalloc(const kv_shape* shape, const void* q, float scale,
                                        const void* K, const void* V,
                                        const int32_t* block_idx, const int32_t* n_kept, int kmax,
                                        const float* k_sum, const float* v_sum,
                                        const int32_t* counts, const float* k_tot,
                                        const float* v_tot, int use_tail_proxy,
                                        const int32_t* tok_idx, const float* w, int m,
                                        float* out, float* lse, kv_stream_t stream);

/*
 * kv_selftest_wait_timeout -- checks the kernels' failure detection on the
 * device without a fault. The pages have no counterpart: every wait of the
 * kernels on a copy is bounded, and one that runs out sets KV_DEV_WAIT_TIMEOUT
 * in the status word and returns instead of hanging; this call runs that same
 * bounded wait in a one-warp kernel.
 *
 *   status     device uint32, 4-byte aligned: KV_DEV_WAIT_TIMEOUT is OR-ed in
 *              when the wait gives up (other bits untouched).
 *   waited_ok  device uint32, 4-byte aligned: set to 1 if the wait completed,
 *              0 if it gave up.
 *   limit_ns   the wait's limit, 0 < limit_ns <= 2e9 (wall time, %globaltimer).
 *   arrive     nonzero: the barrier's phase completes (an arrival with no bytes
 *              expected) and the wait succeeds; zero: the phase expects 16 bytes
 *              that no copy delivers (none is issued), so the wait runs out.
 *
 * Asynchronous on `stream`; KV_ERR_INVALID_ARG for bad pointers or limits.
 */
kv_status kv_selftest_wait_timeout(uint32_t* status, uint32_t* waited_ok, uint64_t limit_ns, int arrive,
                                   kv_stream_t stream);

/*
 * kv_stream_read -- a measurement reference with no counterpart on the pages:
 * reads `bytes` from src once, as a plain streaming kernel (16-byte loads, four
 * in flight per thread, eight 256-thread CTAs per SM) and produces nothing. Timed
 * like the attention kernel, it gives the time one launch needs just to move the
 * same number of bytes from HBM, launch and ramp included.
 *
 *   src    device, 16-byte aligned; bytes a multiple of 16
 *   sink   device uint32, 4-byte aligned (written only if the folded words hit a
 *          fixed constant, so the loads cannot be optimised away)
 * Asynchronous on `stream`; KV_ERR_INVALID_ARG for bad pointers or sizes.
 */
kv_status kv_stream_read(const void* src, size_t bytes, uint32_t* sink, kv_stream_t stream);

/* Message of the last failed call on this host thread ("" if none). */
const char* kv_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVSPARSE_H */
