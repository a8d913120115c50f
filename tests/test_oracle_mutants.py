"""Planted mistakes: each mutant breaks one oracle function in a plausible way
(a dropped term, a wrong sign or index, a wrong reduction) and at least one pin
must fail on it. This checks that the pins can see such mistakes."""
import math

import numpy as np
import pytest

import oracle_pins as P
from oracle import oracle as O


def _mut_proxy_no_log_count(orig):
    def f(qg, K, V, n, L, kept, sigma):
        r = orig(qg, K, V, n, L, kept, sigma)
        return None if r is None else (r[0] - math.log(r[2]), r[1], r[2])
    return f


def _mut_proxy_sum_value(orig):
    def f(qg, K, V, n, L, kept, sigma):
        r = orig(qg, K, V, n, L, kept, sigma)
        return None if r is None else (r[0], r[1] * r[2], r[2])
    return f


def _mut_summary_no_log(orig):
    def f(qg, k_sum, counts, sigma):
        out = orig(qg, k_sum, counts, sigma)
        c = np.asarray(counts, dtype=np.float64)
        return np.where(c > 0, out - np.log(np.maximum(c, 1)), out)
    return f


def _mut_summary_sum_not_mean(orig):
    def f(qg, k_sum, counts, sigma):
        return orig(qg, k_sum * np.maximum(np.asarray(counts)[:, None], 1), counts, sigma)
    return f


def _mut_round_bf16_truncate(orig):
    def f(x):
        x = np.asarray(x, dtype=np.float64)
        out = np.array(x, copy=True)
        fin = np.isfinite(x) & (x != 0)
        _, E = np.frexp(x[fin])
        sp = np.ldexp(1.0, np.maximum(E - 1, -126) - 7)
        out[fin] = np.trunc(x[fin] / sp) * sp
        return out
    return f


def _mut_round_bf16_ties_up(orig):
    def f(x):
        x = np.asarray(x, dtype=np.float64)
        out = np.array(x, copy=True)
        fin = np.isfinite(x) & (x != 0)
        _, E = np.frexp(x[fin])
        sp = np.ldexp(1.0, np.maximum(E - 1, -126) - 7)
        out[fin] = np.floor(x[fin] / sp + 0.5) * sp
        return out
    return f


def _mut_rpchol_greedy(orig):
    def f(K, n, sigma, u, m):
        return _greedy(K, n, sigma, m)
    return f


def _greedy(K, n, sigma, m):
    A = O.wildcat_kernel(K, n, sigma)
    d = np.diag(A).copy()
    F = np.zeros((n, m))
    S = []
    for t in range(m):
        if d.sum() <= 0:
            break
        s_ = int(np.argmax(d))
        g = A[:, s_] - F[:, :t] @ F[s_, :t]
        F[:, t] = g / math.sqrt(g[s_])
        d = np.maximum(d - F[:, t] ** 2, 0.0)
        d[s_] = 0.0
        S.append(s_)
    return S, F[:, :len(S)]


def _mut_rpchol_no_downdate(orig):
    def f(K, n, sigma, u, m):
        A = O.wildcat_kernel(K, n, sigma)
        d = np.diag(A).copy()
        F = np.zeros((n, m))
        S = []
        for t in range(m):
            tot = d.sum()
            if tot <= 0:
                break
            s_ = min(int(np.searchsorted(np.cumsum(d), u[t] * tot)), n - 1)
            g = A[:, s_].copy()
            F[:, t] = g / math.sqrt(g[s_])
            d = np.maximum(d - F[:, t] ** 2, 0.0)
            d[s_] = 0.0
            S.append(s_)
        return S, F[:, :len(S)]
    return f


def _mut_wildcat_uniform_weights(orig):
    def f(K, n, sigma, S):
        w = np.full(len(S), n / max(1, len(S)))
        return w, w
    return f


def _mut_wildcat_kernel_no_sigma(orig):
    def f(K, n, sigma):
        return orig(K, n, 1.0)
    return f


def _mut_group_score_logits(orig):
    def f(shat):
        return np.where(np.isfinite(shat), shat, 0.0).sum(axis=0)
    return f


def _mut_select_high_index(orig):
    def f(S, valid_nb, k, ff, fl):
        r = orig(-np.asarray(S)[::-1] * -1 if False else S, valid_nb, k, ff, fl)
        forced = set(r["forced"])
        cand = [b for b in range(valid_nb) if b not in forced]
        order = sorted(cand, key=lambda b: (-S[b], -b))
        r["order"] = order
        r["kept"] = sorted(forced | set(order[:min(k, len(order))]))
        return r
    return f


def _mut_exact_mass_max(orig):
    def f(qg, K, n, L, NB, sigma):
        out = np.full((qg.shape[0], NB), -math.inf)
        for b, (s, e) in enumerate(O.blocks_of(n, L)):
            out[:, b] = (sigma * (K[s:e] @ qg.T)).max(axis=0)
        return out
    return f


def _mut_cobs_no_half(orig):
    def f(qg, k_sum, counts, xi, sigma):
        out = orig(qg, k_sum, counts, xi, sigma)
        for b in range(k_sum.shape[0]):
            for g in range(qg.shape[0]):
                out[g, b] += 0.5 * sigma * sigma * float(np.sum((xi[b] @ qg[g]) ** 2))
        return out
    return f


def _mut_cobs_unsquared(orig):
    def f(qg, k_sum, counts, xi, sigma):
        out = orig(qg, k_sum, counts, xi, sigma)
        for b in range(k_sum.shape[0]):
            for g in range(qg.shape[0]):
                p = xi[b] @ qg[g]
                out[g, b] += 0.5 * sigma * sigma * float(np.sum(p) - np.sum(p ** 2))
        return out
    return f


def _mut_cov_sample(orig):
    def f(K, n, L, NBcap, r):
        xi, lam = orig(K, n, L, NBcap, r)
        for b, (s, e) in enumerate(O.blocks_of(n, L)):
            c = e - s
            if c > 1:
                xi[b] *= math.sqrt(c / (c - 1))
                lam[b] *= c / (c - 1)
        return xi, lam
    return f


def _mut_cov_smallest(orig):
    def f(K, n, L, NBcap, r):
        D = K.shape[1]
        xi_all, lam_all = orig(K, n, L, NBcap, D)
        return xi_all[:, ::-1][:, :r].copy(), lam_all[:, ::-1][:, :r].copy()
    return f


def _mut_quest_max_end_only(orig):
    def f(qg, kmin, kmax, sigma):
        return np.stack([sigma * (qg[g] * kmax).sum(axis=1) for g in range(qg.shape[0])])
    return f


def _mut_bounds_swapped(orig):
    def f(K, n, L, NBcap):
        a, b = orig(K, n, L, NBcap)
        return b, a
    return f


def _mut_weighted_no_log(orig):
    def f(qg, K, V, n, idx, w, sigma):
        w = np.asarray(w, dtype=np.float64)
        return orig(qg, K, V, n, idx, np.where(w > 0, 1.0, 0.0), sigma)
    return f


def _mut_summaries_count(orig):
    def f(K, V, n, L, NBcap):
        ks, vs, c, kt, vt = orig(K, V, n, L, NBcap)
        c = c.copy()
        c[c > 0] = L
        return ks, vs, c, kt, vt
    return f


def _mut_softmax_no_norm(orig):
    def f(logits, values):
        o, l = orig(logits, values)
        return o * 1.01, l
    return f


def _mut_logsumexp_shift(orig):
    def f(x):
        v = orig(x)
        return v if v == -math.inf else v + 1e-3
    return f



def _mut_fp4_ties_away(orig):
    def f(x):
        x32 = np.asarray(x, dtype=np.float32)
        codes = np.zeros(x32.shape, dtype=np.uint8)
        amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0.0)
        scale = np.float32(amax / np.float32(6.0))
        if not scale > 0:
            return codes, np.float32(0.0)
        for j, v in enumerate(x32):
            a = abs(float(np.float32(v / scale)))
            best, bd = 0, None
            for c, gv in enumerate(O.E2M1_GRID):
                dist = abs(a - gv)
                if bd is None or dist <= bd:  # a tie goes to the larger magnitude
                    best, bd = c, dist
            codes[j] = best | (8 if (v < 0 and best != 0) else 0)
        return codes, scale
    return f


def _mut_fp4_scale_by_4(orig):
    def f(x):
        x32 = np.asarray(x, dtype=np.float32)
        amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0.0)
        scale = np.float32(amax / np.float32(4.0))  # the largest magnitude lands on 4, not 6
        codes = np.zeros(x32.shape, dtype=np.uint8)
        if not scale > 0:
            return codes, np.float32(0.0)
        for j, v in enumerate(x32):
            a = abs(float(np.float32(v / scale)))
            best = min(range(8), key=lambda c: (abs(a - O.E2M1_GRID[c]), c % 2))
            codes[j] = best | (8 if (v < 0 and best != 0) else 0)
        return codes, scale
    return f


def _mut_query_basis_first_head(orig):
    def f(Qc, Hkv):
        G = Qc.shape[1] // Hkv
        return orig(Qc[:, ::G, :], Hkv)
    return f


def _mut_subspace_rank_floor(orig):
    def f(evals, energy=0.9):
        s, sh = orig(evals, energy)
        return int(math.floor(sum(sh) / len(sh))), sh
    return f


def _mut_subspace_logits_unprojected(orig):
    def f(qg, mean, counts, xi, sigma, U=None):
        if U is None:
            return orig(qg, mean, counts, xi, sigma, None)
        # the query's first s coordinates instead of its projection
        return orig(qg, mean, counts, xi, sigma, np.eye(xi.shape[-1], qg.shape[1]))
    return f


def _mut_ss_factors_full_space_projected(orig):
    def f(K, n, L, NBcap, r, U):
        # project the full-space top-r directions instead of decomposing U Sigma U^T
        xf, lf = O.block_cov_factors_one(K, n, L, NBcap, r)
        xs = np.einsum("brd,sd->brs", xf, np.asarray(U, dtype=np.float64))
        return xs, np.sum(xs * xs, axis=2)
    return f


def _mut_kmeans_no_update(orig):
    def f(Z32, C, iters):
        return orig(Z32, C, min(iters, 1))  # the centroids stop after one move
    return f


def _mut_kmeans_first_tokens(orig):
    def f(Z32, C, iters):
        Z = np.asarray(Z32, dtype=np.float64)
        n = Z.shape[0]
        Ce = min(C, n)
        cent = Z[:Ce].copy()  # starts at the first tokens
        labels = np.zeros(n, dtype=np.int64)
        for _ in range(iters):
            d = ((Z[:, None, :] - cent[None]) ** 2).sum(axis=2)
            labels = np.argmin(d, axis=1)
            for c in range(Ce):
                if (labels == c).any():
                    cent[c] = Z[labels == c].mean(axis=0)
        return labels, cent
    return f


def _mut_errorgate_no_minus_one(orig):
    def f(qg, cnt, ks, kq, sigma):
        E = orig(qg, cnt, ks, kq, sigma)
        return E + np.where(np.asarray(cnt) > 0, 1.0, 0.0) * qg.shape[0] / max(1, int(np.sum(np.asarray(cnt) > 0)))
    return f


def _mut_split_uncapped(orig):
    def f(E, cnt, R):
        return orig(E, [10 ** 9] * len(cnt), R)
    return f


def _mut_qgs_no_normaliser(orig):
    def f(qg, Z16, P, sigma):
        qt = np.asarray(qg, dtype=np.float64) @ np.asarray(P, dtype=np.float64).T
        lg = sigma * (np.asarray(Z16, dtype=np.float64) @ qt.T)
        return np.exp(lg).sum(axis=1)
    return f


def _mut_qgc_proxy_no_count(orig):
    def f(qg, K, V, n, labels, read, C, sigma):
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
                if un:
                    logits.append(sigma * float(qg[g] @ K[un].mean(axis=0)))  # no ln count
                    vals.append(V[un].mean(axis=0))
            if logits:
                out[g], lse[g] = O.softmax_attend(np.array(logits), np.array(vals))
        return out, lse
    return f

MUTANTS = {
    "tail_proxy/no ln count": ("tail_proxy", _mut_proxy_no_log_count),
    "tail_proxy/sum not mean": ("tail_proxy", _mut_proxy_sum_value),
    "summary_logits/no ln n_b": ("summary_logits", _mut_summary_no_log),
    "summary_logits/sum not mean": ("summary_logits", _mut_summary_sum_not_mean),
    "mean16/no ln n_b": ("summary_mean16_logits", _mut_summary_no_log),
    "mean16/sum not mean": ("summary_mean16_logits", _mut_summary_sum_not_mean),
    "round_bf16/truncates": ("round_bf16", _mut_round_bf16_truncate),
    "rpcholesky/greedy pivots": ("rpcholesky", _mut_rpchol_greedy),
    "rpcholesky/no downdate": ("rpcholesky", _mut_rpchol_no_downdate),
    "wildcat/uniform weights": ("wildcat_weights", _mut_wildcat_uniform_weights),
    "wildcat/kernel without scale": ("wildcat_kernel", _mut_wildcat_kernel_no_sigma),
    "round_bf16/ties up": ("round_bf16", _mut_round_bf16_ties_up),
    "group_score/sums logits": ("group_score", _mut_group_score_logits),
    "select_blocks/high-index ties": ("select_blocks", _mut_select_high_index),
    "exact_log_mass/max not lse": ("exact_log_mass", _mut_exact_mass_max),
    "weighted/no ln w": ("weighted_attend_one", _mut_weighted_no_log),
    "summaries/count": ("block_summaries_one", _mut_summaries_count),
    "softmax/unnormalised": ("softmax_attend", _mut_softmax_no_norm),
    "logsumexp/offset": ("logsumexp", _mut_logsumexp_shift),
    "quest/max end only": ("quest_logits", _mut_quest_max_end_only),
    "quest/bounds swapped": ("block_bounds_one", _mut_bounds_swapped),
    "cobs/no one half": ("cobs_logits", _mut_cobs_no_half),
    "cobs/projections not squared": ("cobs_logits", _mut_cobs_unsquared),
    "cobs/sample covariance (n - 1)": ("block_cov_factors_one", _mut_cov_sample),
    "cobs/smallest eigendirections": ("block_cov_factors_one", _mut_cov_smallest),
    "fp4/ties away from zero": ("fp4_e2m1_quantize", _mut_fp4_ties_away),
    "fp4/scale max over 4": ("fp4_e2m1_quantize", _mut_fp4_scale_by_4),
    "query_basis/first head of the group": ("query_basis", _mut_query_basis_first_head),
    "subspace_rank/mean rounded down": ("subspace_rank", _mut_subspace_rank_floor),
    "subspace_logits/query not projected": ("cobs_subspace_logits", _mut_subspace_logits_unprojected),
    "ss_factors/projected full-space directions": ("block_cov_factors_ss_one", _mut_ss_factors_full_space_projected),
    "kmeans/centroids stop moving": ("qgc_kmeans", _mut_kmeans_no_update),
    "kmeans/starts at the first tokens": ("qgc_kmeans", _mut_kmeans_first_tokens),
    "errorgate/mass not the gap": ("errorgate_errors", _mut_errorgate_no_minus_one),
    "errorgate/split not capped": ("errorgate_split", _mut_split_uncapped),
    "qgs/no per-head normaliser": ("qgs_token_scores", _mut_qgs_no_normaliser),
    "qgc/proxy without ln count": ("qgc_attend_one", _mut_qgc_proxy_no_count),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_pin_fails_on_mutant(name, monkeypatch):
    attr, make = MUTANTS[name]
    monkeypatch.setattr(O, attr, make(getattr(O, attr)))
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {name}"
