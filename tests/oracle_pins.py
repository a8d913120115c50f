"""Pins for the float64 oracle: each function checks the oracle against something
other than itself -- a brute-force loop in plain Python floats, a closed form, an
invariant the pages state, or the numbers of the pages' worked example -- and raises
AssertionError on a mismatch. The tests call them as they are, and the planted-mistake
test calls them against deliberately broken copies of oracle functions.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-12


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3g}"


def _rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- brute force helpers
def _py_dense(qg, K, V, n, sigma):
    """Softmax attention written as nested Python loops over floats."""
    G, D = len(qg), len(qg[0])
    outs, lses = [], []
    for g in range(G):
        logits = []
        for r in range(n):
            s = 0.0
            for d in range(D):
                s += float(qg[g][d]) * float(K[r][d])
            logits.append(sigma * s)
        m = max(logits)
        ws = [math.exp(x - m) for x in logits]
        z = sum(ws)
        o = [sum(ws[r] * float(V[r][d]) for r in range(n)) / z for d in range(D)]
        outs.append(o)
        lses.append(m + math.log(z))
    return outs, lses


# ----------------------------------------------------------------------------- pins
def pin_dense_bruteforce(seed=0):
    r = _rng(seed)
    G, D, n = 3, 5, 23
    qg, K, V = r.normal(size=(G, D)), r.normal(size=(n + 4, D)), r.normal(size=(n + 4, D))
    o, l = O.dense_attend_one(qg, K, V, n, 0.7)
    po, pl = _py_dense(qg.tolist(), K.tolist(), V.tolist(), n, 0.7)
    _close(o, po, what="dense out")
    _close(l, pl, what="dense lse")


def pin_summaries_closed_form(seed=1):
    r = _rng(seed)
    D, Ncap, L = 4, 37, 8
    for n in (0, 1, 8, 29, 37):
        K, V = r.normal(size=(Ncap, D)), r.normal(size=(Ncap, D))
        NBcap = (Ncap + L - 1) // L
        ks, vs, c, kt, vt = O.block_summaries_one(K, V, n, L, NBcap)
        for b in range(NBcap):
            cnt = 0
            sk = [0.0] * D
            sv = [0.0] * D
            for t in range(b * L, (b + 1) * L):
                if t < n:
                    cnt += 1
                    for d in range(D):
                        sk[d] += float(K[t][d])
                        sv[d] += float(V[t][d])
            assert int(c[b]) == cnt, f"count of block {b} at n={n}"
            _close(ks[b], sk, what="k_sum")
            _close(vs[b], sv, what="v_sum")
        _close(kt, [sum(float(K[t][d]) for t in range(n)) for d in range(D)], what="k_tot")
        _close(vt, [sum(float(V[t][d]) for t in range(n)) for d in range(D)], what="v_tot")


def pin_exact_mass_bruteforce(seed=2):
    r = _rng(seed)
    G, D, n, L = 2, 3, 21, 6
    qg, K = r.normal(size=(G, D)), r.normal(size=(n, D))
    nb = (n + L - 1) // L
    lm = O.exact_log_mass(qg, K, n, L, nb, 0.9)
    for g in range(G):
        for b in range(nb):
            tot = 0.0
            for t in range(b * L, min(n, (b + 1) * L)):
                tot += math.exp(0.9 * sum(float(qg[g][d]) * float(K[t][d]) for d in range(D)))
            _close(lm[g, b], math.log(tot), what="ln m_b")


def pin_block_decomposition(seed=3):
    """COBS, text around Equation 1: the dense output is the P_b-weighted mixture of
    the block centroids v^c_b, with P_b = m_b / Z."""
    r = _rng(seed)
    G, D, n, L = 2, 4, 45, 8
    qg, K, V = r.normal(size=(G, D)), r.normal(size=(n, D)), r.normal(size=(n, D))
    o, _ = O.dense_attend_one(qg, K, V, n, 1.0)
    for g in range(G):
        masses, cents = [], []
        for (s, e) in O.blocks_of(n, L):
            ws = [math.exp(float(qg[g] @ K[t])) for t in range(s, e)]
            m = sum(ws)
            masses.append(m)
            cents.append([sum(ws[i] * float(V[s + i][d]) for i in range(e - s)) / m
                          for d in range(D)])
        Z = sum(masses)
        mix = [sum(masses[b] / Z * cents[b][d] for b in range(len(masses))) for d in range(D)]
        _close(o[g], mix, what="block decomposition")


def pin_discard_error_identity(seed=4):
    """COBS, text after Equation 1: o - o_S = (1/(1 - tau)) sum_{b not in S} P_b
    (v^c_b - o), tau the dropped mass. o_S is the oracle's discard-mode output."""
    r = _rng(seed)
    G, D, n, L = 1, 3, 40, 5
    qg, K, V = r.normal(size=(G, D)), r.normal(size=(n, D)), r.normal(size=(n, D))
    kept = [0, 3, 6]
    o, _ = O.dense_attend_one(qg, K, V, n, 1.0)
    oS, _, _ = O.sparse_attend_one(qg, K, V, n, L, kept, 1.0, use_proxy=False)
    ws = [math.exp(float(qg[0] @ K[t])) for t in range(n)]
    Z = sum(ws)
    tau = 0.0
    rhs = [0.0] * D
    for b, (s, e) in enumerate(O.blocks_of(n, L)):
        if b in kept:
            continue
        m = sum(ws[s:e])
        P = m / Z
        tau += P
        cent = [sum(ws[t] * float(V[t][d]) for t in range(s, e)) / m for d in range(D)]
        for d in range(D):
            rhs[d] += P * (cent[d] - float(o[0][d]))
    rhs = [x / (1.0 - tau) for x in rhs]
    _close(o[0] - oS[0], rhs, what="discard error identity")


def pin_all_kept_equals_dense(seed=5):
    r = _rng(seed)
    G, D, n, L = 2, 6, 61, 8
    q = r.normal(size=(1, G, D))
    K, V = r.normal(size=(1, 1, n, D)), r.normal(size=(1, 1, n, D))
    nb = (n + L - 1) // L
    sel, out, lse = O.decode_step(q, K, V, [n], L, 0.5, nb, False, False)
    assert sel[(0, 0)]["kept"] == list(range(nb))
    do, dl = O.dense_batch(q, K, V, [n], 0.5)
    _close(out, do, what="all kept out")
    _close(lse, dl, what="all kept lse")


def pin_proxy_exact_equal_tail(seed=6):
    """OA: the proxy represents the tail exactly when every tail token has the same
    logit. Tail keys differ from each other but share their projection on q."""
    r = _rng(seed)
    D, n, L = 5, 50, 10
    q = r.normal(size=(1, D))
    qhat = q[0] / np.linalg.norm(q[0])
    K = r.normal(size=(n, D))
    V = r.normal(size=(n, D))
    kept = [1, 3]
    for t in range(n):
        if t // L not in kept:
            u = K[t] - (K[t] @ qhat) * qhat          # component orthogonal to q
            K[t] = 0.3 * qhat + u                    # every tail logit = 0.3 |q| sigma
    o, l, proxy = O.sparse_attend_one(q, K, V, n, L, kept, 0.8, use_proxy=True)
    do, dl = O.dense_attend_one(q, K, V, n, 0.8)
    _close(o, do, what="proxy exact out")
    _close(l, dl, what="proxy exact lse")


def pin_proxy_logit_is_mean_plus_log_count(seed=7):
    """OA: proxy logit = mean tail logit + ln(count), so its weight is count times
    the weight of a mean-logit token; its value is the mean of the tail values."""
    r = _rng(seed)
    G, D, n, L = 2, 4, 33, 4
    qg, K, V = r.normal(size=(G, D)), r.normal(size=(n, D)), r.normal(size=(n, D))
    kept = [0, 5]
    logit, value, nT = O.tail_proxy(qg, K, V, n, L, kept, 0.6)
    tail = [t for t in range(n) if t // L not in kept]
    assert nT == len(tail)
    for g in range(G):
        ls = [0.6 * sum(float(qg[g][d]) * float(K[t][d]) for d in range(D)) for t in tail]
        mean_l = sum(ls) / len(ls)
        _close(logit[g], mean_l + math.log(len(tail)), what="proxy logit")
        _close(math.exp(logit[g]), len(tail) * math.exp(mean_l), what="proxy weight")
    _close(value, [sum(float(V[t][d]) for t in tail) / len(tail) for d in range(D)],
           what="proxy value")


def pin_jensen(seed=8):
    """Proxy weight <= true tail mass (equality iff equal tail logits, OA), and the
    mean-pool score <= exact log-mass (COBS: mean pooling matches only the zeroth
    and first cumulant terms)."""
    r = _rng(seed)
    G, D, n, L = 3, 6, 90, 9
    qg, K, V = r.normal(size=(G, D)), r.normal(size=(n, D)), r.normal(size=(n, D))
    kept = [2, 7]
    logit, _, _ = O.tail_proxy(qg, K, V, n, L, kept, 1.0)
    tail = [t for t in range(n) if t // L not in kept]
    for g in range(G):
        mass = sum(math.exp(float(qg[g] @ K[t])) for t in tail)
        assert math.exp(logit[g]) <= mass * (1 + 1e-12)
        assert math.exp(logit[g]) < mass * (1 - 1e-6), "random tail should be strict"
    nb = (n + L - 1) // L
    ks, _, c, _, _ = O.block_summaries_one(K, V, n, L, nb)
    sh = O.summary_logits(qg, ks, c, 1.0)
    lm = O.exact_log_mass(qg, K, n, L, nb, 1.0)
    assert np.all(sh <= lm + 1e-12), "summary score above exact log-mass"
    assert np.all(sh < lm - 1e-9), "random blocks should be strict"


def pin_integer_weights_duplication(seed=9):
    """WC form: exp(s + ln w) = w exp(s), so integer w equals w-fold duplication."""
    r = _rng(seed)
    G, D, n = 2, 5, 40
    qg, K, V = r.normal(size=(G, D)), r.normal(size=(n, D)), r.normal(size=(n, D))
    idx = r.choice(n, size=12, replace=False)
    w = r.integers(1, 5, size=12).astype(np.float64)
    o, l = O.weighted_attend_one(qg, K, V, n, idx, w, 0.9)
    rows = [int(i) for i, c in zip(idx, w) for _ in range(int(c))]
    Kd, Vd = K[rows], V[rows]
    po, pl = _py_dense(qg.tolist(), Kd.tolist(), Vd.tolist(), len(rows), 0.9)
    _close(o, po, what="weighted == duplicated out")
    _close(l, pl, what="weighted == duplicated lse")


def pin_zero_weight_excluded(seed=10):
    r = _rng(seed)
    G, D, n = 1, 3, 20
    qg, K, V = r.normal(size=(G, D)), r.normal(size=(n, D)), r.normal(size=(n, D))
    idx = np.array([1, 4, 7, 9])
    w = np.array([2.0, 0.0, 1.0, 3.0])
    o, l = O.weighted_attend_one(qg, K, V, n, idx, w, 1.0)
    o2, l2 = O.weighted_attend_one(qg, K, V, n, idx[[0, 2, 3]], w[[0, 2, 3]], 1.0)
    _close(o, o2, what="zero weight")
    _close(l, l2, what="zero weight lse")


def pin_summary_equals_exact_for_constant_blocks(seed=13):
    """When every key of a block is the same vector k, m_b = n_b exp(sigma q.k)
    exactly, so the mean-pool score must equal the exact log-mass (the Jensen
    equality case); ragged last block included."""
    r = _rng(seed)
    G, D, n, L = 3, 4, 27, 8
    qg = r.normal(size=(G, D))
    K = np.zeros((n, D))
    for b, (s, e) in enumerate(O.blocks_of(n, L)):
        K[s:e] = r.normal(size=D)
    nb = (n + L - 1) // L
    ks, _, c, _, _ = O.block_summaries_one(K, K, n, L, nb)
    sh = O.summary_logits(qg, ks, c, 0.7)
    for g in range(G):
        for b, (s, e) in enumerate(O.blocks_of(n, L)):
            want = math.log((e - s) * math.exp(0.7 * float(qg[g] @ K[s])))
            _close(sh[g, b], want, what="constant-block summary score")


def pin_group_score_invariants(seed=11):
    """Each head's block probabilities sum to one, so sum_b S_b = G; for G = 1 the
    ranking equals the ranking by s_hat (COBS: for G = 1, keeping the top-k by m_b,
    equivalently by ln m_b)."""
    r = _rng(seed)
    for G in (1, 4, 7):
        sh = r.normal(size=(G, 30)) * 3
        S = O.group_score(sh)
        _close(S.sum(), G, what="sum of S")
        assert np.all(S >= 0) and np.all(S <= G)
        # brute-force probabilities for one head
        z = sum(math.exp(x) for x in sh[0])
        if G == 1:
            _close(S, [math.exp(x) / z for x in sh[0]], what="G=1 probabilities")
            a = O.select_blocks(S, 30, 7, False, False)["order"]
            b = sorted(range(30), key=lambda i: (-sh[0][i], i))
            assert a == b, "G=1 order differs from s_hat order"


def pin_topk_bruteforce(seed=12):
    """The kept set maximises the summed score over all k-subsets of the competing
    blocks; among equal sums the lexicographically smallest index set wins."""
    r = _rng(seed)
    for trial in range(6):
        nb = 9
        S = np.round(r.random(nb) * 4) / 4 if trial % 2 else r.random(nb)
        for ff, fl in ((False, False), (True, True), (True, False)):
            forced = set([0] if ff else []) | set([nb - 1] if fl else [])
            cand = [b for b in range(nb) if b not in forced]
            for k in (1, 3, 5, len(cand), len(cand) + 2):
                best = None
                for sub in itertools.combinations(cand, min(k, len(cand))):
                    # ties in the sum are broken by the per-element (score, index) order
                    key = (sorted([(-S[b], b) for b in sub]),)
                    if best is None or key < best[0]:
                        best = (key, sub)
                want = sorted(forced | set(best[1]))
                got = O.select_blocks(S, nb, k, ff, fl)["kept"]
                assert got == want, f"top-k {got} != brute force {want}"
                assert sum(S[b] for b in got if b not in forced) >= \
                    max(sum(S[b] for b in sub) for sub in
                        itertools.combinations(cand, min(k, len(cand)))) - 1e-15


def pin_near_tie_flag():
    S = np.array([0.5, 0.30, 0.2999, 0.1])
    assert O.select_blocks(S, 4, 2, False, False)["near_tie"]
    assert not O.select_blocks(S, 4, 1, False, False)["near_tie"]
    assert not O.select_blocks(S, 4, 4, False, False)["near_tie"]


def pin_worked_example():
    """OA, "A worked example with named numbers": 10,000 tokens; 100 exact tokens
    hold 60%; a 9,900-token tail with equal logits holds 40%."""
    with open(os.path.join(GOLDEN, "openattention_worked_example.json")) as f:
        ex = json.load(f)
    n, n_ex, n_tail = ex["context_tokens"], ex["exact_tokens"], ex["tail_tokens"]
    assert n_ex + n_tail == n
    # one channel: logit = key value; exact tokens share logit a, the tail logit 0
    a = math.log(ex["exact_mass"] / ex["tail_mass"] * n_tail / n_ex)
    K = np.zeros((n, 1))
    K[:n_ex, 0] = a
    V = np.zeros((n, 2))
    V[:n_ex, 0] = 1.0            # channel 0 reads the exact tokens' share
    V[n_ex:, 1] = 1.0            # channel 1 reads the tail's share
    q = np.ones((1, 1))
    L = n_ex
    dense, _ = O.dense_attend_one(q, K, V, n, 1.0)
    _close(dense[0], [ex["exact_mass"], ex["tail_mass"]], what="toy masses")
    disc, _, _ = O.sparse_attend_one(q, K, V, n, L, [0], 1.0, use_proxy=False)
    infl = disc[0][0] / dense[0][0]
    assert abs(infl - 1 / 0.6) < 1e-12 and round(infl, 2) == ex["discard_inflation_about"]
    prox, _, p = O.sparse_attend_one(q, K, V, n, L, [0], 1.0, use_proxy=True)
    _close(prox[0], [ex["exact_mass"], ex["proxy_tail_mass_kept"]], what="proxy keeps 40%")
    assert p[2] == n_tail
    # scaled-up sample through the weighted mode: 50 tail tokens with weight 198
    s = ex["sample_tokens"]
    scale = n_tail / s
    assert scale == ex["sample_scale_up"]
    hit = s / n_tail
    assert round(hit, 3) == ex["sample_hit_probability_about"]
    assert round(1 - hit, 3) == ex["sample_miss_fraction_about"]
    idx = np.concatenate([np.arange(n_ex), n_ex + np.arange(s) * 7])
    w = np.concatenate([np.ones(n_ex), np.full(s, scale)])
    wo, _ = O.weighted_attend_one(q, K, V, n, idx, w, 1.0)
    _close(wo[0], [ex["exact_mass"], ex["tail_mass"]], what="scaled sample mass")


def pin_empty_inputs():
    D = 3
    K = np.zeros((8, D))
    o, l = O.dense_attend_one(np.ones((2, D)), K, K, 0, 1.0)
    assert np.all(o == 0) and np.all(l == -math.inf)
    o, l = O.weighted_attend_one(np.ones((1, D)), K, K, 8, [1, 2], [0.0, 0.0], 1.0)
    assert np.all(o == 0) and l[0] == -math.inf
    sel = O.select_blocks(np.zeros(0), 0, 3, True, True)
    assert sel["kept"] == []
    sel = O.select_blocks(np.array([0.7]), 1, 3, True, True)
    assert sel["kept"] == [0]


def pin_quest_box_corners(seed=14):
    """Quest bound = the largest q . corner over every corner of the block's
    bounding box (brute force over 2^D corners), and the bounds are the
    channel-wise min / max by loops."""
    r = _rng(seed)
    G, D, n, L = 2, 5, 23, 7
    qg, K = r.normal(size=(G, D)), r.normal(size=(n, D))
    NB = (n + L - 1) // L
    kmin, kmax = O.block_bounds_one(K, n, L, NB)
    for b in range(NB):
        rows = range(b * L, min(n, (b + 1) * L))
        for d in range(D):
            _close(kmin[b, d], min(float(K[t][d]) for t in rows), what="min")
            _close(kmax[b, d], max(float(K[t][d]) for t in rows), what="max")
    sq = O.quest_logits(qg, kmin, kmax, 0.7)
    for g in range(G):
        for b in range(NB):
            best = -math.inf
            for mask in range(1 << D):
                corner = [kmax[b, d] if (mask >> d) & 1 else kmin[b, d] for d in range(D)]
                best = max(best, sum(float(qg[g][d]) * corner[d] for d in range(D)))
            _close(sq[g, b], 0.7 * best, what="quest corner max")


def pin_quest_upper_bound(seed=15):
    """Every key of a block lies in its box, so the Quest score bounds each
    token's logit from above; a one-key block's box is that key, so the bound is
    that logit."""
    r = _rng(seed)
    G, D, n, L = 3, 8, 61, 8
    qg, K = r.normal(size=(G, D)), r.normal(size=(n, D))
    NB = (n + L - 1) // L
    kmin, kmax = O.block_bounds_one(K, n, L, NB)
    sq = O.quest_logits(qg, kmin, kmax, 0.5)
    for b in range(NB):
        lg = 0.5 * (K[b * L:min(n, (b + 1) * L)] @ qg.T)
        assert np.all(sq[:, b] >= lg.max(axis=0) - 1e-12), "quest bound below a token logit"
        assert np.all(sq[:, b] > lg.max(axis=0) + 1e-9), "quest bound equal to the max logit on a random block"
    k1 = K[:1]
    kmin1, kmax1 = O.block_bounds_one(k1, 1, L, 1)
    _close(O.quest_logits(qg, kmin1, kmax1, 0.5)[:, 0], 0.5 * (k1 @ qg.T)[0], what="one-key block")


# ----------------------------------------------------------------- second-order (COBS) scorer
def _py_cov_quadratic(K, s, e, q):
    """q^T Sigma q of the keys K[s:e], Sigma the population covariance, by loops."""
    n = e - s
    D = len(q)
    mean = [sum(float(K[r][j]) for r in range(s, e)) / n for j in range(D)]
    tot = 0.0
    for r in range(s, e):
        d = sum(float(q[j]) * (float(K[r][j]) - mean[j]) for j in range(D))
        tot += d * d
    return tot / n, mean


def pin_cobs_full_rank_is_exact_quadratic(seed=16):
    # with r = D the stored factors carry the whole covariance: the logit equals
    # sigma q.mean + (sigma^2 / 2) q^T Sigma q + ln n computed by loops
    g = _rng(seed)
    D, L, n = 6, 12, 30  # blocks of 12, 12 and 6 keys
    K = g.normal(size=(n, D)) * g.uniform(0.3, 2.0, size=D)
    qg = g.normal(size=(2, D))
    NB = 3
    ks, _, c, _, _ = O.block_summaries_one(K, K, n, L, NB)
    xi, _ = O.block_cov_factors_one(K, n, L, NB, D)
    sig = 0.8
    sh = O.cobs_logits(qg, ks, c, xi, sig)
    for b, (s, e) in enumerate(O.blocks_of(n, L)):
        for gi in range(2):
            quad, mean = _py_cov_quadratic(K, s, e, qg[gi])
            ref = sig * sum(float(qg[gi][j]) * mean[j] for j in range(D)) + 0.5 * sig * sig * quad + math.log(e - s)
            _close(sh[gi, b], ref, 1e-11, what="second-order logit, full rank")


def pin_cobs_rank_one_block(seed=17):
    # keys on a line through their mean: the covariance has rank 1, so r = 1
    # already holds all of it, the first eigenvalue is var(t) |v|^2 and the rest 0
    g = _rng(seed)
    D, n = 5, 16
    mu = g.normal(size=D)
    v = g.normal(size=D)
    t = g.normal(size=n)
    K = mu[None, :] + t[:, None] * v[None, :]
    xi1, lam = O.block_cov_factors_one(K, n, n, 1, 3)
    var_t = float(np.mean((t - t.mean()) ** 2))
    _close(lam[0, 0], var_t * float(v @ v), 1e-11, what="rank-one eigenvalue")
    _close(lam[0, 1:], np.zeros(2), 1e-11, what="eigenvalues past the rank")
    q = g.normal(size=D)
    quad, _ = _py_cov_quadratic(K, 0, n, q)
    _close(float((xi1[0, 0] @ q) ** 2), quad, 1e-11, what="rank-one quadratic form")


def pin_cobs_two_point_closed_form(seed=18):
    # keys mean +- v in equal numbers: the exact log-mass is ln n + x0 + ln cosh(x)
    # with x0 = sigma q.mean, x = sigma q.v; the second-order estimate replaces
    # ln cosh(x) by x^2 / 2
    g = _rng(seed)
    D, half = 4, 5
    mu = g.normal(size=D)
    v = 0.7 * g.normal(size=D)
    K = np.concatenate([mu[None, :] + v[None, :]] * half + [mu[None, :] - v[None, :]] * half)
    n = 2 * half
    q = g.normal(size=(1, D))
    sig = 0.9
    ks, _, c, _, _ = O.block_summaries_one(K, K, n, n, 1)
    xi, _ = O.block_cov_factors_one(K, n, n, 1, 2)
    est = O.cobs_logits(q, ks, c, xi, sig)[0, 0]
    exact = O.exact_log_mass(q, K, n, n, 1, sig)[0, 0]
    x0 = sig * float(q[0] @ mu)
    x = sig * float(q[0] @ v)
    _close(exact, math.log(n) + x0 + math.log(math.cosh(x)), 1e-12, what="two-point exact mass")
    _close(est - exact, 0.5 * x * x - math.log(math.cosh(x)), 1e-12, what="two-point second-order gap")


def pin_cobs_error_order(seed=19):
    # keys mean + eps z: the first-order (mean-pool) error shrinks like eps^2, the
    # second-order one like eps^3 (the third cumulant is the first term dropped)
    g = _rng(seed)
    D, n = 6, 24
    mu = g.normal(size=D)
    Z = g.normal(size=(n, D))
    q = g.normal(size=(1, D))
    sig = 1.0

    def errs(eps):
        K = mu[None, :] + eps * Z
        ks, _, c, _, _ = O.block_summaries_one(K, K, n, n, 1)
        xi, _ = O.block_cov_factors_one(K, n, n, 1, D)
        exact = O.exact_log_mass(q, K, n, n, 1, sig)[0, 0]
        first = O.summary_logits(q, ks, c, sig)[0, 0]
        second = O.cobs_logits(q, ks, c, xi, sig)[0, 0]
        return abs(exact - first), abs(exact - second)

    e1a, e2a = errs(0.02)
    e1b, e2b = errs(0.01)
    assert 3.6 < e1a / e1b < 4.4, f"first-order error ratio {e1a / e1b:.3f} (eps^2 expects 4)"
    assert 6.5 < e2a / e2b < 9.5, f"second-order error ratio {e2a / e2b:.3f} (eps^3 expects 8)"
    assert e2a < 0.1 * e1a, "the second-order estimate is not closer than the first-order one"


def pin_cobs_eigen_structure(seed=20):
    # scaled eigenvectors: mutually orthogonal, |xi_i|^2 = lambda_i descending, and
    # with r = D their outer products sum to the covariance (by loops)
    g = _rng(seed)
    D, n = 5, 9
    K = g.normal(size=(n, D)) * g.uniform(0.5, 2.0, size=D)
    xi, lam = O.block_cov_factors_one(K, n, n, 1, D)
    X = xi[0]
    gram = X @ X.T
    _close(gram - np.diag(np.diag(gram)), np.zeros((D, D)), 1e-11, what="orthogonal factors")
    _close(np.diag(gram), lam[0], 1e-11, what="|xi|^2 = eigenvalue")
    assert all(lam[0, i] >= lam[0, i + 1] - 1e-15 for i in range(D - 1)), "eigenvalues not descending"
    for a in range(D):
        for b2 in range(D):
            ca = sum((float(K[r][a]) - float(np.mean(K[:, a]))) * (float(K[r][b2]) - float(np.mean(K[:, b2])))
                     for r in range(n)) / n
            _close(float(np.sum(X[:, a] * X[:, b2])), ca, 1e-11, what="sum of xi xi^T = covariance")


def _bf16_bits(x: float) -> int:
    """Upper 16 bits of the float32 encoding of x (x must be a float32 value)."""
    import struct
    return struct.unpack("<I", struct.pack("<f", x))[0] >> 16


def _bf16_value(bits: int) -> float:
    import struct
    return struct.unpack("<f", struct.pack("<I", (bits & 0xffff) << 16))[0]


def pin_round_bf16_nearest_even(seed=21):
    """round_bf16 against a brute-force search over the bf16 grid: the result is a
    bf16 value, no bf16 value is nearer, and of two equally near ones the even
    encoding wins."""
    r = _rng(seed)
    xs = list(r.normal(size=300) * np.exp(r.uniform(-30, 30, size=300)))
    # exact midpoints between neighbouring bf16 values (ties), both parities
    for bits in (0x3f80, 0x3f81, 0x4049, 0x404a, 0xbf80, 0xc0a3, 0x0001, 0x0080):
        lo, hi = _bf16_value(bits), _bf16_value(bits + 1)
        xs.append((lo + hi) / 2)
    xs += [0.0, 1.0, -2.5, 3.0e38, 1e-40]
    got = O.round_bf16(np.array(xs))
    for x, g in zip(xs, got):
        if x == 0.0:
            assert g == 0.0
            continue
        if abs(x) > O.BF16_MAX * (1 + 2.0 ** -9):
            assert math.isinf(g)
            continue
        g32 = float(np.float32(g))
        assert g32 == g, f"{x!r}: {g!r} is not a float32 value"
        b = _bf16_bits(g32)
        assert _bf16_value(b) == g, f"{x!r}: {g!r} is not a bf16 value"
        # neighbours on the grid (same sign): none nearer, ties to the even code
        for nb in (b - 1, b + 1):
            if (nb & 0x7fff) in (0x7f80,) or nb < 0 or nb > 0xffff or (nb ^ b) & 0x8000:
                continue
            v = _bf16_value(nb)
            if math.isinf(v):
                continue
            dg, dv = abs(g - x), abs(v - x)
            assert dg <= dv, f"{x!r}: {g!r} is not the nearest bf16 value ({v!r} is nearer)"
            if dg == dv:
                assert b % 2 == 0, f"{x!r}: tie not broken to the even code"


def pin_mean16_score(seed=22):
    """The bf16-mean score equals the exact-mean score when every block mean is a
    bf16 value, and otherwise differs by at most sigma * sum_j |q_j| |mean_j| 2^-8
    (the relative rounding bound of an 8-bit significand)."""
    r = _rng(seed)
    G, D, L, NB = 3, 16, 4, 9
    # keys on a coarse dyadic grid whose block sums divide exactly: means are bf16
    K = np.round(r.normal(size=(NB * L, D)) * 4) / 4
    counts = np.full(NB, L)
    k_sum = K.reshape(NB, L, D).sum(axis=1)
    means = k_sum / L
    assert np.array_equal(O.round_bf16(means), means), "test means must be bf16 values"
    qg = r.normal(size=(G, D))
    _close(O.summary_mean16_logits(qg, k_sum, counts, 0.3), O.summary_logits(qg, k_sum, counts, 0.3),
           1e-14, what="bf16-representable means")
    # general keys: the bound, and the bound is not loose by orders of magnitude
    K = r.normal(size=(NB * L, D)) * np.exp(r.normal(size=D))
    counts = np.array([L] * (NB - 1) + [3])
    k_sum = np.zeros((NB, D))
    for b in range(NB):
        k_sum[b] = K[b * L:b * L + counts[b]].sum(axis=0)
    a = O.summary_mean16_logits(qg, k_sum, counts, 0.3)
    e = O.summary_logits(qg, k_sum, counts, 0.3)
    for b in range(NB):
        mean = k_sum[b] / counts[b]
        for g in range(G):
            bound = 0.3 * float(np.sum(np.abs(qg[g]) * np.abs(mean))) * 2.0 ** -8
            assert abs(a[g, b] - e[g, b]) <= bound * (1 + 1e-12), (b, g)
    assert np.max(np.abs(a - e)) > 0, "rounding must change some score"


def pin_wildcat_kernel_bruteforce(seed=23):
    """The key kernel, entry by entry in Python floats."""
    r = _rng(seed)
    K = r.normal(size=(9, 5))
    sigma = 0.4
    A = O.wildcat_kernel(K, 7, sigma)
    M = max(sum(float(x) * float(x) for x in K[i]) for i in range(7))
    for i in range(7):
        for j in range(7):
            dot = sum(float(K[i][d]) * float(K[j][d]) for d in range(5))
            _close(A[i, j], math.exp(sigma * dot - sigma * M), 1e-13, what="kernel entry")
    assert np.all(A <= 1.0 + 1e-15) and A.shape == (7, 7)


def pin_rpcholesky_pivot_rule(seed=24):
    """Each pivot is the inverse-CDF draw of u over the residual diagonal, which is
    recomputed here by brute force from the pivots before it (diag(A) minus the
    squares of the factor columns, each column the residual kernel column over the
    square root of its pivot entry)."""
    r = _rng(seed)
    n, m = 40, 12
    K = r.normal(size=(n, 6))
    u = r.uniform(size=m)
    sigma = 0.3
    S, F = O.rpcholesky(K, n, sigma, u, m)
    A = O.wildcat_kernel(K, n, sigma)
    cols = []
    for t, s_t in enumerate(S):
        d = [A[i][i] - sum(c[i] ** 2 for c in cols) for i in range(n)]
        for j in S[:t]:
            d[j] = 0.0
        d = [max(x, 0.0) for x in d]
        tot = sum(d)
        acc, want = 0.0, None
        for i in range(n):
            acc += d[i]
            if acc >= u[t] * tot:
                want = i
                break
        assert s_t == want, (t, s_t, want)
        res = [A[i][s_t] - sum(c[i] * c[s_t] for c in cols) for i in range(n)]
        cols.append([x / math.sqrt(res[s_t]) for x in res])
    _close(F, np.array(cols).T, 1e-10, what="factor columns")


def pin_rpcholesky_interpolates(seed=25):
    """F F^T reproduces the kernel on the pivots' rows; the residual diagonal is
    non-negative and zero on the pivots; the pivots are distinct."""
    r = _rng(seed)
    n = 120
    K = r.normal(size=(n, 8))
    S, F = O.rpcholesky(K, n, 0.25, r.uniform(size=30), 30)
    A = O.wildcat_kernel(K, n, 0.25)
    assert len(set(S)) == len(S) == 30
    _close((F @ F.T)[S], A[S], 1e-10, what="interpolation on pivot rows")
    res = np.diag(A) - np.sum(F * F, axis=1)
    assert np.min(res) > -1e-10 and np.max(np.abs(res[S])) < 1e-10


def pin_wildcat_all_points_is_exact(seed=26):
    """With every token a pivot the optimal weights are all 1, and the weighted
    coreset attention is dense attention."""
    r = _rng(seed)
    n, D = 14, 4
    K, V = r.normal(size=(n, D)), r.normal(size=(n, D))
    qg = r.normal(size=(2, D))
    S, _ = O.rpcholesky(K, n, 0.5, r.uniform(size=n), n)
    assert sorted(S) == list(range(n))
    w, wc = O.wildcat_weights(K, n, 0.5, S)
    _close(w, np.ones(n), 1e-8, what="weights with every token kept")
    o, l = O.weighted_attend_one(qg, K, V, n, S, wc, 0.5)
    od, ld = O.dense_attend_one(qg, K, V, n, 0.5)
    _close(o, od, 1e-8, what="coreset of all tokens = dense")
    _close(l, ld, 1e-8, what="lse")


def pin_wildcat_identical_tokens(seed=27):
    """n identical tokens: one pivot explains the kernel, its weight is n, and the
    coreset attention equals dense attention over the n copies."""
    r = _rng(seed)
    n, D = 25, 6
    k, v = r.normal(size=D), r.normal(size=D)
    K, V = np.tile(k, (n, 1)), np.tile(v, (n, 1))
    qg = r.normal(size=(3, D))
    S, _ = O.rpcholesky(K, n, 0.7, r.uniform(size=5), 5)
    assert len(S) == 1
    w, wc = O.wildcat_weights(K, n, 0.7, S)
    _close(w, [float(n)], 1e-10, what="weight of the single pivot")
    o, l = O.weighted_attend_one(qg, K, V, n, S, wc, 0.7)
    od, ld = O.dense_attend_one(qg, K, V, n, 0.7)
    _close(o, od, 1e-10, what="identical tokens")
    _close(l, ld, 1e-10, what="lse")


def pin_wildcat_weights_optimal(seed=28):
    """The weights minimise the kernel distance: the objective
    w^T A_SS w - 2 w^T A_{S,:} 1 (written out with Python sums) is not lowered by
    moving any single weight either way."""
    r = _rng(seed)
    n = 30
    K = r.normal(size=(n, 5))
    S, _ = O.rpcholesky(K, n, 0.3, r.uniform(size=6), 6)
    w, _ = O.wildcat_weights(K, n, 0.3, S)
    A = O.wildcat_kernel(K, n, 0.3)

    def J(x):
        quad = sum(x[a] * x[b] * A[S[a]][S[b]] for a in range(len(S)) for b in range(len(S)))
        lin = sum(x[a] * sum(A[S[a]][i] for i in range(n)) for a in range(len(S)))
        return quad - 2.0 * lin

    base = J(list(w))
    for a in range(len(S)):
        for eps in (1e-3, -1e-3):
            x = list(w)
            x[a] += eps
            assert J(x) > base, (a, eps)



def _rotation(r, D):
    Q, _ = np.linalg.qr(r.normal(size=(D, D)))
    return Q


def pin_query_basis_closed_form(seed=29):
    """Calibration queries built along the columns of a random rotation R, one row
    of length sqrt(D lambda_j) per direction, give the second moment R diag(lambda)
    R^T exactly: the eigenvalues come back sorted and each eigenvector is +-R's
    column. In a group of two heads the rows of both heads enter the moment."""
    r = _rng(seed)
    D, Hkv, G = 6, 2, 2
    lam = np.array([5.0, 0.5, 3.0, 1.0, 0.25, 2.0])
    R = _rotation(r, D)
    rows = [math.sqrt(D * lam[j]) * R[:, j] for j in range(D)]
    Qc = np.zeros((D // G, Hkv * G, D))
    for h in range(Hkv):
        for j in range(D):  # direction j: position j // G, head j % G of the group
            Qc[j // G, h * G + j % G] = rows[j] * (1 if (j + h) % 2 == 0 else -1)
    evals, evecs = O.query_basis(Qc, Hkv)
    order = np.argsort(-lam)
    for h in range(Hkv):
        _close(evals[h], lam[order], 1e-12, what="eigenvalues")
        for k, j in enumerate(order):
            c = sum(float(evecs[h][k][d]) * float(R[d][j]) for d in range(D))
            _close(abs(c), 1.0, 1e-10, what="eigenvector direction")


def pin_subspace_rank_by_hand():
    """s: the smallest rank with 90% of the trace per head, the mean over heads
    rounded up; a cumulative sum equal to 90% counts as reaching it."""
    ev = np.array([[5.0, 3.0, 1.0, 1.0],    # 5, 8, 9 >= 9: 3
                   [9.5, 0.3, 0.2, 0.0]])   # 9.5 >= 9: 1
    s, sh = O.subspace_rank(ev, 0.9)
    assert sh == [3, 1] and s == 2, (s, sh)
    ev2 = np.array([[5.0, 3.0, 1.0, 1.0], [4.0, 3.0, 2.0, 1.0], [9.5, 0.5, 0.0, 0.0]])  # 3, 3 (4+3+2=9), 1
    s2, sh2 = O.subspace_rank(ev2, 0.9)
    assert sh2 == [3, 3, 1] and s2 == 3, (s2, sh2)  # mean 7/3 rounds up to 3
    assert O.subspace_rank(np.array([[1.0, 1.0, 1.0, 1.0]]), 0.9)[0] == 4


def _py_cov(X):
    n, D = len(X), len(X[0])
    mu = [sum(X[k][d] for k in range(n)) / n for d in range(D)]
    return [[sum((X[k][a] - mu[a]) * (X[k][b] - mu[b]) for k in range(n)) / n for b in range(D)] for a in range(D)]


def pin_subspace_factors_exact_in_subspace(seed=30):
    """With r = s the subspace factors hold B_b whole, so for a query inside the
    subspace (q = U^T z) the projected quadratic form equals q^T Sigma_b q with the
    covariance written out as Python sums; with U = I they reproduce the full-space
    factors' quadratic forms."""
    r = _rng(seed)
    D, s_dim, L, n = 7, 3, 5, 12
    K = r.normal(size=(n, D))
    U = _rotation(r, D)[:s_dim]  # orthonormal rows
    xi, lam = O.block_cov_factors_ss_one(K, n, L, 3, s_dim, U)
    for b, (st, e) in enumerate(O.blocks_of(n, L)):
        cov = _py_cov(K[st:e].tolist())
        for _ in range(3):
            z = r.normal(size=s_dim)
            q = U.T @ z
            qt = U @ q
            got = sum(float(xi[b, i] @ qt) ** 2 for i in range(s_dim))
            want = sum(q[a] * cov[a][c] * q[c] for a in range(D) for c in range(D))
            _close(got, want, 1e-10, what="projected quadratic form")
    xf, lf = O.block_cov_factors_one(K, n, L, 3, 4)
    xs, ls = O.block_cov_factors_ss_one(K, n, L, 3, 4, np.eye(D))
    _close(ls, lf, 1e-10, what="identity basis eigenvalues")
    for b in range(3):
        for _ in range(3):
            q = r.normal(size=D)
            _close(np.sum((xs[b] @ q) ** 2), np.sum((xf[b] @ q) ** 2), 1e-10, what="identity basis forms")


def pin_fp4_e2m1_grid_and_ties(seed=31):
    """E2M1 codes: the grid points times the scale round-trip exactly; every tie
    between two neighbouring magnitudes goes to the code with mantissa bit 0; the
    largest magnitude is code 7 (6 x scale); zero keeps code 0; a zero vector has
    scale 0; each code is the nearest grid point (checked against every point)."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for sgn in (1.0, -1.0):
        x = [sgn * g for g in grid]
        c, sc = O.fp4_e2m1_quantize(x)
        assert float(sc) == 1.0
        _close(O.fp4_e2m1_decode(c, sc), x, 0.0, what="grid round trip")
        ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
        want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]  # the even neighbour of each midpoint
        c, sc = O.fp4_e2m1_quantize([sgn * t for t in ties] + [sgn * 6.0])
        _close(O.fp4_e2m1_decode(c, sc)[:-1], [sgn * w for w in want], 0.0, what="ties to even")
        assert int(c[-1]) == (7 if sgn > 0 else 15)
    c, sc = O.fp4_e2m1_quantize(np.zeros(5))
    assert float(sc) == 0.0 and not np.any(c)
    r = _rng(seed)
    for _ in range(20):
        x = r.normal(size=33) * math.exp(r.normal())
        c, sc = O.fp4_e2m1_quantize(x)
        scale = float(sc)
        assert abs(scale - float(np.float32(np.max(np.abs(np.float32(x))))) / 6.0) <= 1e-6 * scale
        dec = O.fp4_e2m1_decode(c, sc)
        for j in range(len(x)):
            best = min(abs(abs(float(x[j])) - g * scale) for g in grid)
            assert abs(abs(dec[j]) - abs(float(x[j]))) <= best + 1e-6 * scale, (j, x[j], dec[j])
            assert dec[j] == 0.0 or (dec[j] > 0) == (x[j] > 0)
        assert np.max(np.abs(dec)) == 6.0 * scale


def pin_cobs_subspace_logits(seed=32):
    """The stored-descriptor score: with the full space (U = None), the exact mean
    and the full-space factors it is the second-order score of cobs_logits; with a
    query inside the subspace and r = s it is sigma q.mean + (sigma^2 / 2)
    q^T Sigma_b q + ln n_b written out with Python sums."""
    r = _rng(seed)
    D, L, n, sig = 6, 4, 10, 0.4
    K = r.normal(size=(n, D))
    NB = 3
    ks, _, cnt, _, _ = O.block_summaries_one(K, K, n, L, NB)
    xi, _ = O.block_cov_factors_one(K, n, L, NB, 3)
    qg = r.normal(size=(2, D))
    mean = ks / cnt[:, None]
    _close(O.cobs_subspace_logits(qg, mean, cnt, xi, sig), O.cobs_logits(qg, ks, cnt, xi, sig), 1e-12,
           what="full space")
    U = _rotation(r, D)[:2]
    xs, _ = O.block_cov_factors_ss_one(K, n, L, NB, 2, U)
    z = r.normal(size=(2, 2))
    qs = z @ U  # rows inside the subspace
    got = O.cobs_subspace_logits(qs, mean, cnt, xs, sig, U)
    for b, (st, e) in enumerate(O.blocks_of(n, L)):
        cov = _py_cov(K[st:e].tolist())
        mu = [sum(K[k][d] for k in range(st, e)) / (e - st) for d in range(D)]
        for g in range(2):
            q = qs[g]
            want = (sig * sum(q[d] * mu[d] for d in range(D))
                    + 0.5 * sig * sig * sum(q[a] * cov[a][c] * q[c] for a in range(D) for c in range(D))
                    + math.log(e - st))
            _close(got[g, b], want, 1e-10, what="subspace score")


def pin_qgc_kmeans_lloyd_steps(seed=35):
    """k-means: the start is the tokens ((2c + 1) n) // (2C); one iteration assigns
    every token to its nearest start centroid (distances and argmin written as
    Python loops, ties to the lower cluster) and moves each centroid to its members'
    mean; two iterations assign against those means. Well separated blobs come back
    as the clusters."""
    r = _rng(seed)
    n, C = 23, 4
    Z = r.normal(size=(n, 16)).astype(np.float32)
    Zl = Z.astype(np.float64).tolist()

    def assign(cent):
        lab = []
        for i in range(n):
            best, bd = 0, None
            for c in range(len(cent)):
                dd = sum((Zl[i][j] - cent[c][j]) ** 2 for j in range(16))
                if bd is None or dd < bd:
                    best, bd = c, dd
            lab.append(best)
        return lab

    def update(lab, cent):
        out = []
        for c in range(len(cent)):
            mem = [i for i in range(n) if lab[i] == c]
            out.append([sum(Zl[i][j] for i in mem) / len(mem) for j in range(16)] if mem else cent[c])
        return out

    start = [Zl[((2 * c + 1) * n) // (2 * C)] for c in range(C)]
    lab1 = assign(start)
    cent1 = update(lab1, start)
    l1, c1 = O.qgc_kmeans(Z, C, 1)
    assert list(l1) == lab1
    _close(c1, cent1, 1e-12, what="centroids after one step")
    lab2 = assign(cent1)
    assert lab2 != lab1  # (this case still moves at the second step)
    l2, c2 = O.qgc_kmeans(Z, C, 2)
    assert list(l2) == lab2
    _close(c2, update(lab2, cent1), 1e-12, what="centroids after two steps")
    # blobs 40 apart with unit spread: recovered as the clusters
    centers = r.normal(size=(3, 16)) * 40.0
    B = np.concatenate([centers[k] + r.normal(size=(20, 16)) for k in range(3)]).astype(np.float32)
    lab, _ = O.qgc_kmeans(B, 3, 6)
    for k in range(3):
        assert len(set(int(x) for x in lab[20 * k:20 * (k + 1)])) == 1
    assert len(set(int(x) for x in lab)) == 3


def pin_qgc_project_identity(seed=34):
    """With the identity as the basis (16-dim keys) the coordinates are the keys in fp32."""
    r = _rng(seed)
    K = r.normal(size=(9, 16))
    _close(O.qgc_project(K, 7, np.eye(16)), K[:7].astype(np.float32), 0.0, what="identity projection")


def pin_errorgate_closed_form(seed=35):
    """A cluster of two keys m +- delta e_0: var_0 = delta^2, so for one head
    s2 = sigma^2 q_0^2 delta^2 and E = 2 e^mu (e^(s2/2) - 1) / (2 e^(mu + s2/2))
    = 1 - e^(-s2/2); a cluster of identical keys leaves no error; two heads add their
    normalised errors."""
    r = _rng(seed)
    D, sig, dl = 5, 0.7, 0.9
    m = r.normal(size=D)
    K = np.stack([m + dl * np.eye(D)[0], m - dl * np.eye(D)[0]])
    qg = r.normal(size=(2, D))
    cnt, ks, vs, kq = O.qgc_cluster_stats(K, K, 2, np.array([0, 0]), 1)
    E = O.errorgate_errors(qg, cnt, ks, kq, sig)
    want = sum(1.0 - math.exp(-0.5 * (sig * qg[g][0] * dl) ** 2) for g in range(2))
    _close(E[0], want, 1e-12, what="two-point cluster")
    K2 = np.concatenate([K, np.tile(m + 3.0, (3, 1))])
    cnt, ks, vs, kq = O.qgc_cluster_stats(K2, K2, 5, np.array([0, 0, 1, 1, 1]), 2)
    E2 = O.errorgate_errors(qg[:1], cnt, ks, kq, sig)
    assert abs(E2[1]) <= 1e-15 and E2[0] > 0


def pin_errorgate_split_by_hand():
    """r_c = min(n_c, floor(R E_c / sum E))."""
    r, _ = O.errorgate_split(np.array([1.0, 2.0, 3.5]), [50, 50, 50], 10)  # 1.54, 3.08, 5.38
    assert list(r) == [1, 3, 5]
    r, _ = O.errorgate_split(np.array([1.0, 2.0, 3.5]), [50, 2, 50], 10)   # the second is capped
    assert list(r) == [1, 2, 5]
    r, _ = O.errorgate_split(np.zeros(3), [5, 5, 5], 10)
    assert list(r) == [0, 0, 0]


def pin_qgs_scores(seed=36):
    """Token scores: each head contributes a softmax over the tokens (so the scores
    add up to G), written here with Python loops."""
    r = _rng(seed)
    n, D, G, sig = 11, 20, 3, 0.3
    P = _rotation(r, D)[:16]
    qg = r.normal(size=(G, D))
    Z = r.normal(size=(n, 16))
    t = O.qgs_token_scores(qg, Z, P, sig)
    _close(np.sum(t), float(G), 1e-12, what="scores add up to G")
    qt = [[sum(P[j][d] * qg[g][d] for d in range(D)) for j in range(16)] for g in range(G)]
    for i in range(n):
        want = 0.0
        for g in range(G):
            lg = [sig * sum(qt[g][j] * Z[k][j] for j in range(16)) for k in range(n)]
            mx = max(lg)
            want += math.exp(lg[i] - mx) / sum(math.exp(x - mx) for x in lg)
        _close(t[i], want, 1e-12, what="token score")


def pin_qgc_single_cluster_no_reads(seed=37):
    """One cluster and nothing read: the output is the count-aware proxy of all tokens
    (the value mean, lse = sigma q . mean key + ln n), as the tail proxy of A4."""
    r = _rng(seed)
    n, D = 30, 6
    K, V = r.normal(size=(n, D)), r.normal(size=(n, D))
    qg = r.normal(size=(2, D))
    o, l = O.qgc_attend_one(qg, K, V, n, np.zeros(n, dtype=np.int64), [], 1, 0.4)
    for g in range(2):
        _close(o[g], V.mean(axis=0), 1e-12, what="proxy value")
        _close(l[g], 0.4 * float(qg[g] @ K.mean(axis=0)) + math.log(n), 1e-12, what="proxy lse")
    ot, lt, _ = O.sparse_attend_one(qg, K, V, n, 10, [], 0.4, True)
    _close(o, ot, 1e-12, what="same as the tail proxy")


def pin_qgc_equal_logits_exact(seed=38):
    """Clusters of identical keys: every proxy hides equal logits, ErrorGate's errors
    vanish (up to the rounding of sum-of-squares minus squared mean), and whatever
    it reads, the output is exact dense attention (the proxy is exact when all the
    weights it hides are equal)."""
    r = _rng(seed)
    D, per, C = 16, 12, 3
    keys = r.normal(size=(C, D)) * 8.0
    K = np.concatenate([np.tile(keys[c], (per, 1)) for c in range(C)])
    V = r.normal(size=(C * per, D))
    n = C * per
    qg = r.normal(size=(2, D))
    res = O.qgc_decode_one(qg, K, V, n, np.eye(D), C, 5, 0.25, 0.3)
    assert np.max(np.abs(res["E"])) <= 1e-12
    od, ld = O.dense_attend_one(qg, K, V, n, 0.3)
    _close(res["out"], od, 1e-12, what="equal logits: dense")
    _close(res["lse"], ld, 1e-12, what="equal logits: lse")


def pin_qgc_select_and_budget(seed=39):
    """In-cluster choice by brute force: in every cluster the r_c tokens of largest
    score, ties to the lower index (written as a sort over (score, index) pairs per
    cluster), ascending; the near-tie flag on a constructed tie; the read budget by
    hand (1% of 32768 less 1.5 rows for each of 32 clusters: 327 - 48 = 279)."""
    r = _rng(seed)
    n, C = 40, 4
    t = r.uniform(size=n)
    labels = r.integers(0, C, size=n)
    rc = [3, 0, 5, 100]
    got, near = O.qgc_select(t, labels, rc)
    want = []
    for c in range(C):
        mem = [(-float(t[i]), i) for i in range(n) if labels[i] == c]
        mem.sort()
        want += [i for _, i in mem[:rc[c]]]
    assert got == sorted(want) and not near
    t2 = np.array([0.5, 0.5, 0.1, 0.9])
    got2, near2 = O.qgc_select(t2, np.zeros(4, dtype=np.int64), [2])
    assert got2 == [0, 3] and near2  # 0.5 at index 0 wins the tie; flagged
    assert O.qgc_read_budget(32768, 0.01, 32) == 279
    assert O.qgc_read_budget(100, 0.01, 4) == 0

ALL_PINS = [
    pin_dense_bruteforce, pin_summaries_closed_form, pin_exact_mass_bruteforce,
    pin_block_decomposition, pin_discard_error_identity, pin_all_kept_equals_dense,
    pin_proxy_exact_equal_tail, pin_proxy_logit_is_mean_plus_log_count, pin_jensen,
    pin_integer_weights_duplication, pin_zero_weight_excluded, pin_group_score_invariants,
    pin_topk_bruteforce, pin_near_tie_flag, pin_worked_example, pin_empty_inputs,
    pin_summary_equals_exact_for_constant_blocks, pin_quest_box_corners, pin_quest_upper_bound,
    pin_cobs_full_rank_is_exact_quadratic, pin_cobs_rank_one_block, pin_cobs_two_point_closed_form,
    pin_cobs_error_order, pin_cobs_eigen_structure, pin_round_bf16_nearest_even, pin_mean16_score,
    pin_wildcat_kernel_bruteforce, pin_rpcholesky_pivot_rule, pin_rpcholesky_interpolates,
    pin_wildcat_all_points_is_exact, pin_wildcat_identical_tokens, pin_wildcat_weights_optimal,
    pin_query_basis_closed_form, pin_subspace_rank_by_hand, pin_subspace_factors_exact_in_subspace,
    pin_fp4_e2m1_grid_and_ties, pin_cobs_subspace_logits,
    pin_qgc_kmeans_lloyd_steps, pin_qgc_project_identity, pin_errorgate_closed_form, pin_errorgate_split_by_hand,
    pin_qgs_scores, pin_qgc_single_cluster_no_reads, pin_qgc_equal_logits_exact, pin_qgc_select_and_budget,
]
