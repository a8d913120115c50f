"""Float64 CPU oracle for reduced-KV softmax decode attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or runs this
module; only the tests, the smoke check and the benchmark's CPU-baseline leg do.
It shares no code with the CUDA path: it is plain NumPy in float64, written step by
step from the pages, with no blocking, fusion or reordering beyond what each
definition states.

Sources (page title, then section / equation):
  [COBS]  "COBS: Cumulant Order Block Sparse Attention" -- block masses and block
          probabilities (Equation 1 and the text around it), the per-KV-head GQA
          score (Equation 5 and the normaliser Z^(g,h) of (5)), the first-order
          mean-pool score (affine score (18): phi_b = mean key, a_b = ln L), OSA
          exact-mass ranking (the OSA paragraph), and the Quest min/max score it
          analyses (the paragraph on escaping the first-order ceiling: per block
          the element-wise minimum and maximum of the keys, scored by the largest
          inner product any point of that box can reach); the second-order
          estimator (truncating the cumulant expansion (8) at second order: the
          block log-mass as ln L plus the first two cumulants of sigma q.k over
          the block's keys) with the covariance kept as its top r scaled
          eigenvectors (the low-rank spectral decomposition (13): each
          eigenvector times the square root of its eigenvalue).
  [OA]    "OpenAttention reads 1% of the KV cache -- Count-aware tail proxy",
          section "Skipping reviews without losing the verdict" (the proxy token)
          and section "A worked example with named numbers".
  [WC]    "WildCat: Near-Linear Attention in Theory and Practice", abstract
          (attention over a small weighted coreset).

Readings where the pages are silent or garbled (each is also listed in the design
notes of the repository):
  R1  The GQA group score is the sum over the group's query heads of per-head
      block softmax probabilities, normalised over all valid blocks (forced ones
      included).
  R2  The count term is the natural log of the block's actual token count n_b
      (ln L for full blocks).
  R3  Logits are sigma * q.k with sigma passed in (1/sqrt(D), or 1 when q is
      already scaled).
  R4  Query head g reads KV head floor(g / G).
  R5  Forced blocks (first and/or last) do not compete and do not count toward k.
  R6  Ties are broken by lowest block index.
  R7  The proxy logit is sigma * q . (mean tail key) + ln n_T, which equals the
      mean tail logit plus ln n_T by linearity; with an empty tail there is no
      proxy.
  R8  Weighted mode: logit + ln w_i, no proxy; w_i = 0 excludes the token.
  R9  An empty softmax (no token, no proxy) gives out = 0 and lse = -inf.
  R10 Near tie: (S_(k) - S_(k+1)) / S_(k) < 1e-3 between the k-th and (k+1)-th
      candidate scores.
  R11 Quest scoring: the box bound sigma * sum_j max(q_j min_j, q_j max_j) takes
      the place of the block log-mass estimate in the Equation 5 group score
      (per-head block softmax probabilities summed over the group), with no count
      term; forced blocks and ties as in R5 and R6.
  R12 Second-order scoring: the block's keys are the distribution whose
      cumulants enter, so the covariance is the population one over the n_b keys
      (divided by n_b) and ln L becomes ln n_b as in R2; the estimate
      sigma q.mean + (sigma^2 / 2) q^T Sigma_r q + ln n_b, with Sigma_r = sum of the
      top r xi_i xi_i^T, is the block logit in the Equation 5 group score. The
      full-space factors are used (no query subspace, no FP4 quantisation).
  R13 bf16 block means: the mean key is rounded to the nearest bfloat16 value
      (ties to even) and used in place of the exact mean in the first-order
      score; everything else as in R1 to R6.
  R14 WildCat coreset (the abstract names randomly pivoted Cholesky and weights
      that minimise reconstruction error, not the kernel or the error): the kernel
      is the exponential kernel of attention on the keys, exp(sigma k_i . k_j)
      (shifted by a constant, which cancels); the error is the kernel (feature
      space) distance between the sum over all tokens and the weighted coreset,
      whose minimiser solves A_SS w = A_{S,:} 1; negative weights are clipped to
      0; the uniforms of the pivot draws are inputs.
  R15 COBS stored descriptor (the subspace and quantisation paragraphs): U_Q is
      the top-s eigenvectors of each KV head's query second moment, the mean of
      q q^T over calibration positions and the group's query heads, stored at
      fp32; s = ceil(mean over heads of the smallest rank reaching 90% of the
      head's trace); the factors are the scaled top-r eigenvectors of
      U_Q^T Sigma_b U_Q; E2M1 codes take one scale per factor, max|x| / 6, the
      nearest magnitude with ties to the even code, decided in float32; the
      block mean is the bf16 mean of R13.
  R16 QGC + ErrorGate (OpenAttention, "Three helpers"): the projection is the
      top-16 query eigenvectors of R15, stored at fp32; k-means is Lloyd's
      iteration in float64 from evenly spaced tokens, the clusters being the
      last assignment; the mean and variance tokens are per cluster the key and
      value means and the per-channel key variance; a proxy's error is the
      lognormal gap n e^mu (e^(s2/2) - 1) between its cluster's expected mass and
      the mean-logit proxy's mass, normalised per head and summed over the group;
      the read budget floor(budget n) less 1.5 rows a cluster is split as
      floor(R E_c / sum E) capped at the cluster size; inside a cluster the top
      tokens by the Equation 5 combination of per-head softmax scores from the bf16
      projections; one count-aware proxy per cluster of its unread tokens.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

NEAR_TIE_REL = 1e-3


# --------------------------------------------------------------------------- blocks
def blocks_of(n: int, L: int) -> List[Tuple[int, int]]:
    """Contiguous blocks of L tokens over [0, n); the last one may be short."""
    return [(s, min(s + L, n)) for s in range(0, n, L)]


def block_summaries_one(K: np.ndarray, V: np.ndarray, n: int, L: int, NBcap: int):
    """Per-block key sum, value sum and token count for one (sequence, KV head),
    plus whole-sequence totals. The mean key k_sum/n_b is the mean-pool summary
    [COBS, affine score (18)]; the sums feed the tail proxy [OA].

    K, V: [Ncap][D] float64. Returns k_sum, v_sum [NBcap][D], counts [NBcap],
    k_tot, v_tot [D]. Blocks at or beyond ceil(n/L) are zero with count 0.
    """
    D = K.shape[1]
    k_sum = np.zeros((NBcap, D))
    v_sum = np.zeros((NBcap, D))
    counts = np.zeros(NBcap, dtype=np.int64)
    for b, (s, e) in enumerate(blocks_of(n, L)):
        k_sum[b] = K[s:e].sum(axis=0)
        v_sum[b] = V[s:e].sum(axis=0)
        counts[b] = e - s
    return k_sum, v_sum, counts, K[:n].sum(axis=0), V[:n].sum(axis=0)


def build_block_summaries(K, V, seq_lens, L):
    """Batched block summaries. K, V: [B][Hkv][Ncap][D] float64."""
    B, Hkv, Ncap, D = K.shape
    NBcap = (Ncap + L - 1) // L
    k_sum = np.zeros((B, Hkv, NBcap, D))
    v_sum = np.zeros((B, Hkv, NBcap, D))
    counts = np.zeros((B, NBcap), dtype=np.int64)
    k_tot = np.zeros((B, Hkv, D))
    v_tot = np.zeros((B, Hkv, D))
    for b in range(B):
        for h in range(Hkv):
            ks, vs, c, kt, vt = block_summaries_one(K[b, h], V[b, h], int(seq_lens[b]), L, NBcap)
            k_sum[b, h], v_sum[b, h], k_tot[b, h], v_tot[b, h] = ks, vs, kt, vt
            counts[b] = c
    return k_sum, v_sum, counts, k_tot, v_tot


def block_bounds_one(K: np.ndarray, n: int, L: int, NBcap: int):
    """Per-block, per-channel minimum and maximum of the keys of one (sequence, KV
    head): the axis-aligned bounding box of each block's keys [COBS, the Quest
    paragraph]. Blocks past the sequence stay 0."""
    D = K.shape[1]
    kmin = np.zeros((NBcap, D))
    kmax = np.zeros((NBcap, D))
    for b, (s, e) in enumerate(blocks_of(n, L)):
        kmin[b] = K[s:e].min(axis=0)
        kmax[b] = K[s:e].max(axis=0)
    return kmin, kmax


def quest_logits(qg: np.ndarray, kmin: np.ndarray, kmax: np.ndarray, sigma: float):
    """s_hat[g][b] = sigma * the largest q_g . k over the box [kmin_b, kmax_b]: a
    linear function is largest at the corner that takes, channel by channel, the
    end whose product with q is larger [COBS, the Quest paragraph]."""
    G = qg.shape[0]
    NB = kmin.shape[0]
    out = np.empty((G, NB))
    for g in range(G):
        out[g] = sigma * np.maximum(qg[g] * kmin, qg[g] * kmax).sum(axis=1)
    return out


def block_cov_factors_one(K: np.ndarray, n: int, L: int, NBcap: int, r: int):
    """Per block, the top r scaled eigenvectors xi_i = sqrt(lambda_i) u_i of the
    covariance of the block's keys (population covariance, divided by the count),
    eigenvalues in descending order [COBS, the low-rank spectral decomposition
    (13); reading R12]. Returns xi [NBcap][r][D] and the eigenvalues [NBcap][r];
    blocks past the sequence, and directions past the covariance's rank, stay 0."""
    D = K.shape[1]
    xi = np.zeros((NBcap, r, D))
    lam = np.zeros((NBcap, r))
    for b, (s, e) in enumerate(blocks_of(n, L)):
        X = K[s:e] - K[s:e].mean(axis=0)
        cov = X.T @ X / (e - s)
        w, U = np.linalg.eigh(cov)  # ascending
        for i in range(min(r, D)):
            li = max(float(w[D - 1 - i]), 0.0)
            lam[b, i] = li
            xi[b, i] = math.sqrt(li) * U[:, D - 1 - i]
    return xi, lam


def cobs_logits(qg: np.ndarray, k_sum: np.ndarray, counts: np.ndarray, xi: np.ndarray, sigma: float):
    """s_hat[g][b] = sigma q_g . mean_b + (sigma^2 / 2) sum_i (q_g . xi_bi)^2 + ln n_b:
    the cumulant expansion of the block log-mass truncated at second order, with
    the covariance in its rank-r form [COBS, text after Equation (8) and (13);
    reading R12]."""
    G = qg.shape[0]
    NB = k_sum.shape[0]
    out = np.empty((G, NB))
    for b in range(NB):
        nb = int(counts[b])
        mean = k_sum[b] / nb
        for g in range(G):
            quad = float(np.sum((xi[b] @ qg[g]) ** 2))
            out[g, b] = sigma * float(qg[g] @ mean) + 0.5 * sigma * sigma * quad + math.log(nb)
    return out


def query_basis(Qc: np.ndarray, Hkv: int):
    """The eigenvectors of each KV head's query second moment [COBS, the subspace
    paragraph: U_Q holds the top s eigenvectors of E[q q^T]; reading R15]. The
    second moment of KV head h is the mean of q q^T over the calibration positions
    and the query heads of its group. Qc: [Nc][Hq][D]. Returns (evals [Hkv][D] in
    descending order, evecs [Hkv][D][D] whose row j is the unit eigenvector of
    evals[h][j])."""
    Nc, Hq, D = Qc.shape
    G = Hq // Hkv
    evals = np.zeros((Hkv, D))
    evecs = np.zeros((Hkv, D, D))
    for h in range(Hkv):
        X = np.asarray(Qc[:, h * G:(h + 1) * G, :], dtype=np.float64).reshape(-1, D)
        C = X.T @ X / X.shape[0]
        w, U = np.linalg.eigh(C)  # ascending
        evals[h] = w[::-1]
        evecs[h] = U[:, ::-1].T
    return evals, evecs


def subspace_rank(evals: np.ndarray, energy: float = 0.9):
    """The subspace dimension s [COBS, the subspace paragraph: s is set per layer
    from the rank capturing 90% of the query spectral energy, averaged over heads;
    reading R15]: per head the smallest s_h whose leading eigenvalues sum to at least
    `energy` of the trace, then s = ceil(mean over heads of s_h). Returns (s, [s_h])."""
    sh = []
    for lam in np.asarray(evals, dtype=np.float64):
        tot = float(np.sum(lam))
        acc, pick = 0.0, len(lam)
        for j, x in enumerate(lam):
            acc += float(x)
            if acc >= energy * tot:
                pick = j + 1
                break
        sh.append(pick)
    return int(math.ceil(sum(sh) / len(sh))), sh


def block_cov_factors_ss_one(K: np.ndarray, n: int, L: int, NBcap: int, r: int, U: np.ndarray):
    """Per block, the top r scaled eigenvectors of the covariance kept within the
    query subspace [COBS, the subspace paragraph: B_b = U_Q^T Sigma_b U_Q, rank-r
    spectral decomposition in the projected space; reading R15]. U: [s][D], rows the
    basis (U_Q^T). Returns xi [NBcap][r][s] (xi_i = sqrt(lambda_i) u_i for the r
    largest eigenvalues of B_b, descending) and the eigenvalues [NBcap][r]; blocks
    past the sequence and directions past B_b's rank stay 0."""
    U = np.asarray(U, dtype=np.float64)
    s_dim = U.shape[0]
    xi = np.zeros((NBcap, r, s_dim))
    lam = np.zeros((NBcap, r))
    for b, (st, e) in enumerate(blocks_of(n, L)):
        X = K[st:e] - K[st:e].mean(axis=0)
        Bm = U @ (X.T @ X / (e - st)) @ U.T
        w, V = np.linalg.eigh(Bm)  # ascending
        for i in range(min(r, s_dim)):
            li = max(float(w[s_dim - 1 - i]), 0.0)
            lam[b, i] = li
            xi[b, i] = math.sqrt(li) * V[:, s_dim - 1 - i]
    return xi, lam


E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # magnitudes of codes 0..7


def fp4_e2m1_quantize(x):
    """E2M1 FP4 codes of one vector with one fp32 scale [COBS, the quantisation
    paragraph: the scaled eigenvectors in E2M1 FP4 with one fp32 scale each;
    reading R15]. The scale is max|x| / 6 (6 is the largest E2M1 magnitude); each
    x_j / scale goes to the nearest E2M1 magnitude, a tie to the code with mantissa
    bit 0 (the even code), with the sign in bit 3 (zero keeps code 0). The scale and
    the quotients are float32 operations, the precision in which the kernel takes the
    same decisions. Returns (codes uint8 [len] in 0..15, scale float32)."""
    x32 = np.asarray(x, dtype=np.float32)
    codes = np.zeros(x32.shape, dtype=np.uint8)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0.0)
    scale = np.float32(amax / np.float32(6.0))
    if not scale > 0:
        return codes, np.float32(0.0)
    for j, v in enumerate(x32):
        a = abs(float(np.float32(v / scale)))
        best, bd = 0, None
        for c, gv in enumerate(E2M1_GRID):
            dist = abs(a - gv)
            if bd is None or dist < bd or (dist == bd and c % 2 == 0):
                best, bd = c, dist
        codes[j] = best | (8 if (v < 0 and best != 0) else 0)
    return codes, scale


def fp4_e2m1_decode(codes, scale) -> np.ndarray:
    """The values of E2M1 codes times their scale (float64)."""
    c = np.asarray(codes, dtype=np.int64)
    mag = np.array(E2M1_GRID)[c & 7]
    return np.where(c & 8, -mag, mag) * float(scale)


def cobs_subspace_logits(qg: np.ndarray, mean: np.ndarray, counts: np.ndarray, xi: np.ndarray, sigma: float,
                         U=None):
    """s_hat[g][b] = sigma q_g . mean_b + (sigma^2 / 2) sum_i (q~_g . xi_bi)^2 + ln n_b
    with the projected query q~ = U q (U None: the full space, q~ = q) [COBS, the
    projected quadratic form after (13), exact when the query lies in the subspace].
    mean: [NB][D] the stored block means; xi: [NB][r][s] the stored factors."""
    G = qg.shape[0]
    NB = mean.shape[0]
    qt = qg if U is None else qg @ np.asarray(U, dtype=np.float64).T
    out = np.full((G, NB), -math.inf)
    for b in range(NB):
        nb = int(counts[b])
        if nb <= 0:
            continue
        for g in range(G):
            quad = float(np.sum((xi[b] @ qt[g]) ** 2))
            out[g, b] = sigma * float(qg[g] @ mean[b]) + 0.5 * sigma * sigma * quad + math.log(nb)
    return out


# --------------------------------------------------------------------------- QGC + ErrorGate
def qgc_project(K: np.ndarray, n: int, P: np.ndarray) -> np.ndarray:
    """z_i = P k_i, the keys' coordinates on the top eigenvectors of the queries,
    stored at fp32 [OA, "Three helpers that make the proxy accurate": keys are
    projected onto the top eigenvectors of the queries; reading R16]. P: [16][D]."""
    return (np.asarray(K[:n], dtype=np.float64) @ np.asarray(P, dtype=np.float64).T).astype(np.float32)


def qgc_kmeans(Z32: np.ndarray, C: int, iters: int):
    """k-means in the projection [OA, "Three helpers": k-means in 16 dimensions, once
    after prefill; reading R16], Lloyd's iteration in float64 on the fp32 coordinates:
    C' = min(C, n) centroids start at the tokens ((2c + 1) n) // (2 C'); each iteration
    assigns every token to the nearest centroid (squared distance summed over the
    coordinates in order; ties to the lower cluster) and moves every non-empty
    cluster's centroid to its members' mean. Returns (labels [n] of the last
    assignment, centroids [C'][16])."""
    Z = np.asarray(Z32, dtype=np.float64)
    n = Z.shape[0]
    Ce = min(C, n)
    if Ce == 0:
        return np.zeros(0, dtype=np.int64), np.zeros((0, Z.shape[1] if Z.ndim == 2 else 16))
    cent = np.stack([Z[((2 * c + 1) * n) // (2 * Ce)] for c in range(Ce)])
    labels = np.zeros(n, dtype=np.int64)
    for _ in range(iters):
        d = np.zeros((n, Ce))
        for c in range(Ce):
            diff = Z - cent[c]
            acc = np.zeros(n)
            for j in range(Z.shape[1]):
                acc = acc + diff[:, j] * diff[:, j]
            d[:, c] = acc
        labels = np.argmin(d, axis=1)
        for c in range(Ce):
            m = labels == c
            if m.any():
                cent[c] = Z[m].mean(axis=0)
    return labels, cent


def qgc_cluster_stats(K: np.ndarray, V: np.ndarray, n: int, labels: np.ndarray, C: int):
    """The cached tokens of every cluster [OA, "Three helpers": the mean and variance
    tokens; reading R16]: count [C], key sum [C][D], value sum [C][D] and per-channel
    key sum of squares [C][D] (mean = sum / count, variance = squares / count - mean^2)."""
    D = K.shape[1]
    cnt = np.zeros(C, dtype=np.int64)
    ks, vs, kq = np.zeros((C, D)), np.zeros((C, D)), np.zeros((C, D))
    for i in range(n):
        c = int(labels[i])
        cnt[c] += 1
        ks[c] += K[i]
        vs[c] += V[i]
        kq[c] += K[i] * K[i]
    return cnt, ks, vs, kq


def errorgate_errors(qg: np.ndarray, cnt, ks, kq, sigma: float) -> np.ndarray:
    """The estimated weight error each cluster's proxy would leave [OA, "Skipping
    reviews without losing the verdict": a proxy's unnormalised weight error is its
    mass times the spread of the weights it hides; "Three helpers": ErrorGate
    estimates it from the cached mean and variance tokens; reading R16]. With the
    cluster's logits read as normal with mean mu_gc = sigma q_g . mean_c and variance
    s2_gc = sigma^2 sum_d q_gd^2 var_cd, the mean-logit proxy's mass n_c e^mu falls
    short of the cluster's expected mass n_c e^(mu + s2/2) by
    E_gc = n_c e^mu_gc (e^(s2_gc / 2) - 1); per head it is divided by the estimated
    total Zhat_g = sum_c n_c e^(mu_gc + s2_gc / 2) and summed over the group's heads.
    Empty clusters get 0. Returns E [C]."""
    C = len(cnt)
    G = qg.shape[0]
    mu = np.full((G, C), -math.inf)
    s2 = np.zeros((G, C))
    for c in range(C):
        if cnt[c] <= 0:
            continue
        mean = ks[c] / cnt[c]
        var = np.maximum(kq[c] / cnt[c] - mean * mean, 0.0)
        for g in range(G):
            mu[g, c] = sigma * float(qg[g] @ mean)
            s2[g, c] = sigma * sigma * float(np.sum(qg[g] * qg[g] * var))
    E = np.zeros(C)
    for g in range(G):
        live = cnt > 0
        if not live.any():
            continue
        M = float(np.max(mu[g, live] + 0.5 * s2[g, live]))
        zhat = float(np.sum(cnt[live] * np.exp(mu[g, live] + 0.5 * s2[g, live] - M)))
        for c in range(C):
            if cnt[c] > 0:
                E[c] += cnt[c] * math.exp(mu[g, c] - M) * math.expm1(0.5 * s2[g, c]) / zhat
    return E


def errorgate_split(E: np.ndarray, cnt, R: int):
    """Exact reads per cluster [OA, "Three helpers": ErrorGate splits the exact-read
    budget across clusters in proportion to the error each proxy would leave; reading
    R23]: r_c = min(n_c, floor(R E_c / sum E)); all 0 when sum E = 0. Also returns the
    near-integer flag: some R E_c / sum E within 1e-4 (relative) of an integer below
    n_c, where float rounding may decide the floor."""
    tot = float(np.sum(E))
    r = np.zeros(len(E), dtype=np.int64)
    near = False
    if tot <= 0.0 or R <= 0:
        return r, near
    for c in range(len(E)):
        x = R * float(E[c]) / tot
        fl = math.floor(x)
        r[c] = min(int(cnt[c]), fl)
        if fl < cnt[c] and (x - fl < 1e-4 * max(1.0, x) or fl + 1 - x < 1e-4 * max(1.0, x)):
            near = True
    return r, near


def qgs_token_scores(qg: np.ndarray, Z16: np.ndarray, P: np.ndarray, sigma: float) -> np.ndarray:
    """Token scores inside the clusters [OA, "Three helpers": QGS picks the top tokens
    inside each cluster from low-bit projections; reading R16]: with the projections
    stored at bf16 (Z16) and the query projected the same way (P q_g),
    t_i = sum_g exp(sigma (P q_g) . z_i - LSE_g), LSE_g over all tokens (the group
    combination of Equation 5, per token)."""
    qt = np.asarray(qg, dtype=np.float64) @ np.asarray(P, dtype=np.float64).T
    lg = sigma * (np.asarray(Z16, dtype=np.float64) @ qt.T)  # [n][G]
    t = np.zeros(lg.shape[0])
    for g in range(lg.shape[1]):
        t += np.exp(lg[:, g] - logsumexp(lg[:, g]))
    return t


def qgc_select(t: np.ndarray, labels: np.ndarray, r) -> Tuple[List[int], bool]:
    """The read tokens: in every cluster c the r_c largest scores (ties to the lower
    index); ascending. Also a near-tie flag: inside some cluster the r_c-th and the
    next score within 1e-3 (relative)."""
    out: List[int] = []
    near = False
    for c in range(len(r)):
        mem = [int(i) for i in np.nonzero(labels == c)[0]]
        if r[c] <= 0 or not mem:
            continue
        mem.sort(key=lambda i: (-t[i], i))
        out += mem[:r[c]]
        if r[c] < len(mem):
            a, b = t[mem[r[c] - 1]], t[mem[r[c]]]
            if a - b <= 1e-3 * abs(a):
                near = True
    return sorted(out), near


def qgc_attend_one(qg, K, V, n, labels, read, C, sigma):
    """Softmax over the read tokens and one count-aware proxy per cluster with unread
    tokens: their mean key and value, logit sigma q . mean + ln count [OA, "Skipping
    reviews": the proxy is one virtual token with the tail's mean value and mean
    logit plus the log of its count; "Three helpers": one proxy per cluster]. Built
    directly from the unread tokens."""
    G, D = qg.shape[0], V.shape[1]
    rs = set(int(i) for i in read)
    out = np.zeros((G, D))
    lse = np.full(G, -math.inf)
    for g in range(G):
        logits, vals = [], []
        for i in sorted(rs):
            logits.append(sigma * float(qg[g] @ K[i]))
            vals.append(V[i])
        for c in range(C):
            un = [i for i in range(n) if int(labels[i]) == c and i not in rs]
            if not un:
                continue
            km = K[un].mean(axis=0)
            vm = V[un].mean(axis=0)
            logits.append(sigma * float(qg[g] @ km) + math.log(len(un)))
            vals.append(vm)
        if logits:
            out[g], lse[g] = softmax_attend(np.array(logits), np.array(vals))
    return out, lse


def qgc_read_budget(n: int, budget: float, C_live: int) -> int:
    """Exact rows a query may read: floor(budget n) less the cached mean and variance
    tokens, 1.5 KV rows a cluster, charged to the read [OA, "Three helpers"]; at least 0."""
    return max(0, int(math.floor(budget * n)) - int(math.ceil(1.5 * C_live)))


def qgc_decode_one(qg, K, V, n, P, C, iters, budget, sigma):
    """One (sequence, KV head) decode step of QGC + ErrorGate from scratch: the
    build (projection, k-means, cluster statistics) and the query (errors, split,
    in-cluster selection, attention with the proxies). Returns a dict with labels,
    counts, E, r, read, near_tie, out, lse."""
    Z32 = qgc_project(K, n, P)
    labels, _ = qgc_kmeans(Z32, C, iters)
    Ce = min(C, n)
    cnt, ks, vs, kq = qgc_cluster_stats(K, V, n, labels, Ce)
    E = errorgate_errors(qg, cnt, ks, kq, sigma)
    R = qgc_read_budget(n, budget, int(np.sum(cnt > 0)))
    r, near_split = errorgate_split(E, cnt, R)
    t = qgs_token_scores(qg, round_bf16(Z32.astype(np.float64)), P, sigma)
    read, near_sel = qgc_select(t, labels, r)
    out, lse = qgc_attend_one(qg, K, V, n, labels, read, Ce, sigma)
    return dict(labels=labels, counts=cnt, E=E, R=R, r=r, read=read, near_tie=near_split or near_sel,
                out=out, lse=lse, Z32=Z32, t=t)


# --------------------------------------------------------------------------- scores
def logsumexp(x: np.ndarray) -> float:
    """ln sum exp(x) with a max shift; -inf for an empty or all -inf input."""
    x = np.asarray(x, dtype=np.float64)
    if x.size == 0:
        return -math.inf
    m = np.max(x)
    if m == -math.inf:
        return -math.inf
    return float(m + math.log(np.sum(np.exp(x - m))))


def summary_logits(qg: np.ndarray, k_sum: np.ndarray, counts: np.ndarray, sigma: float):
    """First-order mean-pool estimate of the block log-mass [COBS, text after
    Equation (8): the first-order term is a mean-pool; affine score (18) with
    phi_b = mean key, a_b = ln L; reading R2 uses ln n_b]:

        s_hat[g, b] = sigma * q_g . (k_sum_b / n_b) + ln n_b

    qg: [G][D]; k_sum: [NB][D]; counts: [NB]. Blocks with n_b = 0 get -inf.
    """
    G = qg.shape[0]
    NB = k_sum.shape[0]
    out = np.full((G, NB), -math.inf)
    for b in range(NB):
        nb = int(counts[b])
        if nb <= 0:
            continue
        mean_key = k_sum[b] / nb
        out[:, b] = sigma * (qg @ mean_key) + math.log(nb)
    return out


def round_bf16(x) -> np.ndarray:
    """Nearest bfloat16 value of each float64 (8 significant bits, ties to even):
    the precision at which COBS keeps the block mean [COBS, the quantisation
    paragraph: one fp32 scale per eigenvector and the block mean at bf16].

    Written from the definition: with |x| in [2^e, 2^(e+1)) the bf16 grid has
    spacing 2^(e-7) (2^-133 below 2^-126, the subnormal range); x / spacing is
    rounded to the nearest integer, ties to even, and scaled back (both scalings
    by a power of two are exact in float64). Values past the largest finite bf16
    become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    fin = np.isfinite(x) & (x != 0)
    if np.any(fin):
        _, E = np.frexp(x[fin])                  # |x| = m 2^E, m in [0.5, 1)
        e = np.maximum(E - 1, -126)              # binade exponent, subnormals share -126
        spacing = np.ldexp(1.0, e - 7)
        r = np.rint(x[fin] / spacing) * spacing  # np.rint: round half to even
        r[np.abs(r) > BF16_MAX] = np.inf * np.sign(r[np.abs(r) > BF16_MAX])
        out[fin] = r
    return out


BF16_MAX = float((2.0 - 2.0 ** -7) * 2.0 ** 127)


def summary_mean16_logits(qg: np.ndarray, k_sum: np.ndarray, counts: np.ndarray, sigma: float):
    """The first-order mean-pool estimate with the block mean stored at bf16
    precision [COBS, text after Equation (8) and the quantisation paragraph]:

        s_hat[g, b] = sigma * q_g . bf16(k_sum_b / n_b) + ln n_b

    Blocks with n_b = 0 get -inf.
    """
    G = qg.shape[0]
    NB = k_sum.shape[0]
    out = np.full((G, NB), -math.inf)
    for b in range(NB):
        nb = int(counts[b])
        if nb <= 0:
            continue
        mean_key = round_bf16(k_sum[b] / nb)
        out[:, b] = sigma * (qg @ mean_key) + math.log(nb)
    return out


def exact_log_mass(qg: np.ndarray, K: np.ndarray, n: int, L: int, NB: int, sigma: float):
    """Exact block log-mass ln m_b = ln sum_{r in b} exp(sigma q.k_r), the quantity
    OSA ranks by [COBS, OSA paragraph; block mass m_b of Equation 1].

    qg: [G][D]; K: [Ncap][D]. Returns [G][NB] with -inf for empty blocks.
    """
    G = qg.shape[0]
    out = np.full((G, NB), -math.inf)
    for b, (s, e) in enumerate(blocks_of(n, L)):
        logits = sigma * (K[s:e] @ qg.T)          # [e-s][G]
        for g in range(G):
            out[g, b] = logsumexp(logits[:, g])
    return out


def group_score(shat: np.ndarray) -> np.ndarray:
    """GQA-normalised group score [COBS, Equation (5) and its normaliser Z^(g,h);
    reading R1]: S_b = sum_g exp(s_hat[g,b] - ln sum_b' exp(s_hat[g,b'])), i.e. the
    sum of the group's per-head block softmax probabilities.
    """
    G, NB = shat.shape
    S = np.zeros(NB)
    for g in range(G):
        lse = logsumexp(shat[g])
        if lse == -math.inf:
            continue
        S += np.exp(shat[g] - lse)
    return S


def select_blocks(S: np.ndarray, valid_nb: int, k: int, force_first: bool,
                  force_last: bool) -> Dict:
    """Top-k block choice per KV head [COBS: "maximized by the top-k blocks under"
    (5); readings R5, R6, R10].

    Forced blocks (first = 0, last = valid_nb - 1) are kept and do not compete.
    The others are ordered by (S descending, block index ascending) and the first
    min(k, |C|) are kept. Returns kept (ascending), the candidate order, and the
    near-tie flag at the k / k+1 boundary.
    """
    forced = set()
    if valid_nb > 0:
        if force_first:
            forced.add(0)
        if force_last:
            forced.add(valid_nb - 1)
    cand = [b for b in range(valid_nb) if b not in forced]
    order = sorted(cand, key=lambda b: (-S[b], b))
    chosen = order[:min(k, len(order))]
    near_tie = False
    if 0 < k < len(order):
        sk, sk1 = S[order[k - 1]], S[order[k]]
        near_tie = bool(sk <= 0 or (sk - sk1) / sk < NEAR_TIE_REL)
    kept = sorted(forced | set(chosen))
    return {"kept": kept, "order": order, "near_tie": near_tie, "forced": sorted(forced)}


# --------------------------------------------------------------------------- attention
def softmax_attend(logits: np.ndarray, values: np.ndarray):
    """out = sum_i softmax(logits)_i values_i and lse = ln sum_i exp(logits_i),
    with a max shift. logits: [T]; values: [T][D]. Entries with logit -inf do not
    contribute. Empty or all -inf -> (zeros, -inf) (reading R9)."""
    D = values.shape[1] if values.ndim == 2 else 0
    logits = np.asarray(logits, dtype=np.float64)
    if logits.size == 0 or np.max(logits) == -math.inf:
        return np.zeros(D), -math.inf
    m = np.max(logits)
    p = np.exp(logits - m)
    z = p.sum()
    out = (p[:, None] * values).sum(axis=0) / z
    return out, float(m + math.log(z))


def tail_proxy(qg: np.ndarray, K: np.ndarray, V: np.ndarray, n: int, L: int,
               kept: Sequence[int], sigma: float):
    """Count-aware tail proxy [OA, "Skipping reviews without losing the verdict";
    reading R7]: one virtual token whose value is the mean of the unread values and
    whose logit is the mean unread logit plus ln(count), computed here directly
    from the tail tokens.

    Returns (logits [G], value [D], n_T) or None when the tail is empty.
    """
    mask = np.ones(n, dtype=bool)
    for b in kept:
        mask[b * L:min(n, (b + 1) * L)] = False
    nT = int(mask.sum())
    if nT == 0:
        return None
    tail_logits = sigma * (K[:n][mask] @ qg.T)    # [nT][G]
    mean_logit = tail_logits.mean(axis=0)          # [G]
    value = V[:n][mask].mean(axis=0)
    return mean_logit + math.log(nT), value, nT


def sparse_attend_one(qg, K, V, n, L, kept, sigma, use_proxy=True):
    """Exact attention over the kept blocks' tokens plus, when use_proxy, the tail
    proxy as one more softmax entry [OA: the proxy "enters the softmax next to the
    exact tokens"]. Without the proxy this is top-k discard: the kept tokens are
    renormalised among themselves [COBS, text after Equation 1].

    qg: [G][D]; K, V: [Ncap][D]. Returns out [G][D], lse [G], proxy info.
    """
    G = qg.shape[0]
    D = V.shape[1]
    rows = []
    for b in sorted(kept):
        rows.extend(range(b * L, min(n, (b + 1) * L)))
    rows = np.asarray(rows, dtype=np.int64)
    proxy = tail_proxy(qg, K, V, n, L, kept, sigma) if use_proxy else None
    out = np.zeros((G, D))
    lse = np.full(G, -math.inf)
    for g in range(G):
        logits = sigma * (K[rows] @ qg[g]) if rows.size else np.zeros(0)
        vals = V[rows] if rows.size else np.zeros((0, D))
        if proxy is not None:
            logits = np.concatenate([logits, [proxy[0][g]]])
            vals = np.concatenate([vals, proxy[1][None, :]], axis=0)
        out[g], lse[g] = softmax_attend(logits, vals)
    return out, lse, proxy


def weighted_attend_one(qg, K, V, n, tok_idx, w, sigma):
    """Attention over an explicitly weighted coreset [WC, abstract]: token i enters
    the softmax with logit sigma q.k_i + ln w_i (reading R8). Tokens with w_i = 0
    or an index outside [0, n) are excluded."""
    G = qg.shape[0]
    D = V.shape[1]
    out = np.zeros((G, D))
    lse = np.full(G, -math.inf)
    idx = np.asarray(tok_idx, dtype=np.int64)
    w = np.asarray(w, dtype=np.float64)
    keep = (w > 0) & (idx >= 0) & (idx < n)
    idx, w = idx[keep], w[keep]
    for g in range(G):
        logits = sigma * (K[idx] @ qg[g]) + np.log(w)
        out[g], lse[g] = softmax_attend(logits, V[idx])
    return out, lse


def wildcat_kernel(K: np.ndarray, n: int, sigma: float) -> np.ndarray:
    """The kernel on the keys the coreset is chosen for [WC, abstract; reading R14]:
    A[i, j] = exp(sigma k_i . k_j - sigma M) over the first n keys, M = max_i |k_i|^2.
    The constant shift keeps every entry in (0, 1] (k_i . k_j <= M by Cauchy-Schwarz)
    and cancels in the pivot choice and in the weights."""
    Kn = np.asarray(K[:n], dtype=np.float64)
    if n == 0:
        return np.zeros((0, 0))
    M = float(np.max(np.sum(Kn * Kn, axis=1)))
    return np.exp(sigma * (Kn @ Kn.T) - sigma * M)


def rpcholesky(K: np.ndarray, n: int, sigma: float, u, m: int):
    """Randomly pivoted Cholesky on the key kernel [WC, abstract: the coreset is
    selected by randomly pivoted Cholesky]. Step t draws the pivot with probability
    proportional to the residual diagonal d (the kernel's diagonal minus what the
    factor so far explains): with the uniform u[t] in (0, 1), the pivot is the
    smallest i with d_0 + ... + d_i >= u[t] (d_0 + ... + d_{n-1}). The new factor
    column is the pivot's residual kernel column divided by the square root of its
    pivot entry, and d drops by its square. Stops early when the residual is zero.
    Returns the pivots (in order) and the factor F [n][t] with F F^T = A on the
    pivots' rows and columns."""
    S, F, _ = rpcholesky_steps(K, n, sigma, u, m)
    return S, F


def wildcat_kernel_cols(K: np.ndarray, n: int, sigma: float, cols) -> np.ndarray:
    """Columns `cols` of wildcat_kernel (an n x len(cols) array), evaluated from the
    same formula without forming the n x n matrix."""
    Kn = np.asarray(K[:n], dtype=np.float64)
    M = float(np.max(np.sum(Kn * Kn, axis=1)))
    return np.exp(sigma * (Kn @ Kn[list(cols)].T) - sigma * M)


def wildcat_kernel_diag(K: np.ndarray, n: int, sigma: float) -> np.ndarray:
    """The diagonal of wildcat_kernel: exp(sigma |k_i|^2 - sigma M)."""
    Kn = np.asarray(K[:n], dtype=np.float64)
    sq = np.sum(Kn * Kn, axis=1)
    return np.exp(sigma * sq - sigma * float(np.max(sq)))


def rpcholesky_steps(K: np.ndarray, n: int, sigma: float, u, m: int, pivots=None):
    """The steps of rpcholesky, also returning each step's residual diagonal (before
    the step's pivot is drawn). With pivots given, those are taken in order instead
    of the draws (to replay another implementation's choices). The kernel is
    evaluated a column at a time, so long sequences fit in memory."""
    d = wildcat_kernel_diag(K, n, sigma) if n else np.zeros(0)
    F = np.zeros((n, m))
    S: List[int] = []
    resid = []
    for t in range(m):
        tot = float(np.sum(d))
        if n == 0 or tot <= 0.0 or (pivots is not None and t >= len(pivots)):
            break
        resid.append(d.copy())
        if pivots is None:
            c = np.cumsum(d)
            s = int(np.searchsorted(c, float(u[t]) * tot, side="left"))
            s = min(s, n - 1)
        else:
            s = int(pivots[t])
        g = wildcat_kernel_cols(K, n, sigma, [s])[:, 0] - F[:, :t] @ F[s, :t]
        if g[s] <= 0.0:
            break
        F[:, t] = g / math.sqrt(g[s])
        d = np.maximum(d - F[:, t] ** 2, 0.0)
        d[s] = 0.0
        S.append(s)
    return S, F[:, :len(S)], resid


def wildcat_weights(K: np.ndarray, n: int, sigma: float, S) -> Tuple[np.ndarray, np.ndarray]:
    """The coreset weights [WC, abstract: "weight the elements optimally to
    minimise reconstruction error"; reading R14]: the w minimising the kernel
    distance || sum_{i<n} phi(k_i) - sum_{j in S} w_j phi(k_j) ||^2, i.e. the
    solution of A_SS w = A_{S,:} 1. Returns (w, w clipped at 0); the attention
    takes ln w, so a negative weight drops its token."""
    S = list(S)
    if not S:
        return np.zeros(0), np.zeros(0)
    AS = wildcat_kernel_cols(K, n, sigma, S)  # A[:, S], n x |S|
    w = np.linalg.solve(AS[S, :], AS.sum(axis=0))
    return w, np.maximum(w, 0.0)


def dense_attend_one(qg, K, V, n, sigma):
    """Exact softmax attention over all n tokens [COBS: "Dense reads the whole KV
    cache"]."""
    G = qg.shape[0]
    D = V.shape[1]
    out = np.zeros((G, D))
    lse = np.full(G, -math.inf)
    for g in range(G):
        out[g], lse[g] = softmax_attend(sigma * (K[:n] @ qg[g]), V[:n])
    return out, lse


# --------------------------------------------------------------------------- batched
def select_batch(q, K, seq_lens, L, sigma, k, force_first, force_last, mode,
                 k_sum=None, counts=None, bh=None, rank=4, stored_xi=None, stored_U=None):
    """Block choice for every (sequence, KV head), or for the listed ones.

    q: [B][Hq][D]; K: [B][Hkv][Ncap][D] float64 (needed for exact-mass mode and to
    build summaries when k_sum is not given). Returns a dict keyed by (b, h) with
    kept, near_tie, S and s_hat.
    """
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    Ncap = K.shape[2]
    G = Hq // Hkv
    NBcap = (Ncap + L - 1) // L
    res = {}
    pairs = bh if bh is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for (b, h) in pairs:
        n = int(seq_lens[b])
        nb = (n + L - 1) // L
        qg = q[b, h * G:(h + 1) * G]
        if mode in ("summary", "summary_mean16"):
            if k_sum is None:
                ks, _, c, _, _ = block_summaries_one(K[b, h], K[b, h], n, L, NBcap)
            else:
                ks, c = k_sum[b, h], counts[b]
            fn = summary_logits if mode == "summary" else summary_mean16_logits
            shat = fn(qg, ks[:nb], c[:nb], sigma)
        elif mode == "exact_mass":
            shat = exact_log_mass(qg, K[b, h], n, L, nb, sigma)
        elif mode == "quest":
            kmin, kmax = block_bounds_one(K[b, h], n, L, NBcap)
            shat = quest_logits(qg, kmin[:nb], kmax[:nb], sigma)
        elif mode == "cobs":
            ks, _, c, _, _ = block_summaries_one(K[b, h], K[b, h], n, L, NBcap)
            xi, _ = block_cov_factors_one(K[b, h], n, L, NBcap, rank)
            shat = cobs_logits(qg, ks[:nb], c[:nb], xi[:nb], sigma)
        elif mode == "cobs_stored":
            # the stored descriptor: bf16 block means and the given factors
            # (stored_xi[(b, h)]: [NB][r][s], e.g. FP4-decoded) in the subspace of
            # stored_U[h] ([s][D]; None: the full space)
            if k_sum is None:
                ks, _, c, _, _ = block_summaries_one(K[b, h], K[b, h], n, L, NBcap)
            else:
                ks, c = k_sum[b, h], counts[b]
            mean = np.zeros((nb, D))
            for j in range(nb):
                if int(c[j]) > 0:
                    mean[j] = round_bf16(ks[j] / int(c[j]))
            Uh = None if stored_U is None else stored_U[h]
            shat = cobs_subspace_logits(qg, mean, c[:nb], stored_xi[(b, h)][:nb], sigma, Uh)
        else:
            raise ValueError(mode)
        S = group_score(shat)
        sel = select_blocks(S, nb, k, force_first, force_last)
        sel["S"] = S
        sel["s_hat"] = shat
        res[(b, h)] = sel
    return res


def sparse_batch(q, K, V, seq_lens, L, sigma, kept: Dict, use_proxy=True, bh=None):
    """out [B][Hq][D], lse [B][Hq] for the given kept-block lists (dict keyed by
    (b, h)); rows not listed in bh stay NaN."""
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    pairs = bh if bh is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for (b, h) in pairs:
        o, l, _ = sparse_attend_one(q[b, h * G:(h + 1) * G], K[b, h], V[b, h],
                                    int(seq_lens[b]), L, kept[(b, h)], sigma, use_proxy)
        out[b, h * G:(h + 1) * G], lse[b, h * G:(h + 1) * G] = o, l
    return out, lse


def weighted_batch(q, K, V, seq_lens, tok_idx, w, sigma, bh=None):
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    pairs = bh if bh is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for (b, h) in pairs:
        o, l = weighted_attend_one(q[b, h * G:(h + 1) * G], K[b, h], V[b, h],
                                   int(seq_lens[b]), tok_idx[b, h], w[b, h], sigma)
        out[b, h * G:(h + 1) * G], lse[b, h * G:(h + 1) * G] = o, l
    return out, lse


def dense_batch(q, K, V, seq_lens, sigma, bh=None):
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    pairs = bh if bh is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for (b, h) in pairs:
        o, l = dense_attend_one(q[b, h * G:(h + 1) * G], K[b, h], V[b, h],
                                int(seq_lens[b]), sigma)
        out[b, h * G:(h + 1) * G], lse[b, h * G:(h + 1) * G] = o, l
    return out, lse


def decode_step(q, K, V, seq_lens, L, sigma, k, force_first, force_last,
                score_mode="summary", use_proxy=True, bh=None):
    """One decode step of one layer for every sequence: block choice per KV head,
    then attention over the kept blocks plus the tail proxy."""
    sel = select_batch(q, K, seq_lens, L, sigma, k, force_first, force_last,
                       score_mode, bh=bh)
    kept = {key: v["kept"] for key, v in sel.items()}
    out, lse = sparse_batch(q, K, V, seq_lens, L, sigma, kept, use_proxy, bh=bh)
    return sel, out, lse
