"""Second-order (COBS) block scoring on the GPU against the float64 oracle ("COBS:
Cumulant Order Block Sparse Attention", the second-order estimator after Equation
(8), the low-rank covariance form (13), Equation (5)): the per-block covariance
factors (eigenvalues and projected quadratic forms, which do not depend on the
eigenvectors' signs), the kept blocks bit-exact up to flagged near ties, the group
scores, and attention over the chosen blocks."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W
from oracle import oracle as O
from gpu_helpers import OUT_TOL, all_pairs, oracle_inputs, row_rel_err, run_pipeline, selection_matches, to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _check_factors(xi_gpu, K64, seq_lens, L, r, pairs, gen, what):
    xg = xi_gpu.cpu().numpy().astype(np.float64)
    NB = xg.shape[2]
    D = xg.shape[-1]
    for (b, h) in pairs:
        xo, lam = O.block_cov_factors_one(K64[b, h], int(seq_lens[b]), L, NB, r)
        _, lam_all = O.block_cov_factors_one(K64[b, h], int(seq_lens[b]), L, NB, min(D, r + 1))
        for blk in range(NB):
            top = max(float(lam[blk, 0]), 1e-30)
            lg = np.sum(xg[b, h, blk] ** 2, axis=1)  # |xi_i|^2 = lambda_i
            assert np.all(np.abs(lg - lam[blk]) <= 1e-5 * top + 1e-12), f"{what}: eigenvalues at {(b, h, blk)}"
            # the rank-r quadratic form is well defined where lambda_r clears lambda_{r+1}
            gap = (lam_all[blk, r - 1] - lam_all[blk, r]) / top if lam_all.shape[1] > r else 1.0
            if gap < 1e-6:
                continue
            for _ in range(3):
                qv = gen.normal(size=D)
                fg = float(np.sum((xg[b, h, blk] @ qv) ** 2))
                fo = float(np.sum((xo[blk] @ qv) ** 2))
                assert abs(fg - fo) <= 1e-5 * top * float(qv @ qv) + 1e-12, f"{what}: q^T Sigma_r q at {(b, h, blk)}"


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 128)])
def test_cov_factors_random(dtype, D):
    gen = torch.Generator(device=DEV)
    gen.manual_seed(31)
    B, Hkv, Ncap, L = 2, 3, 300, 64  # ragged: 44-key and 1-key blocks below
    K = (torch.randn(B, Hkv, Ncap, D, generator=gen, device=DEV)
         * torch.rand(1, 1, 1, D, generator=gen, device=DEV) * 2).to(dtype)
    lens = [300, 193]
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    for r in (1, 4, 8):
        xi = kv.kv_build_block_cov_factors(K, sl, L, r)
        torch.cuda.synchronize()
        _check_factors(xi, to64(K), lens, L, r, [(b, h) for b in range(B) for h in range(Hkv)],
                       np.random.default_rng(r), f"random D={D} r={r}")


def test_cov_factors_low_rank_blocks():
    # every block's keys span a 3-dimensional affine subspace: rank 4 holds the
    # whole covariance, the fourth factor is zero
    g = np.random.default_rng(5)
    B, Hkv, Ncap, L, D = 1, 2, 256, 32, 128
    K = np.zeros((B, Hkv, Ncap, D))
    for h in range(Hkv):
        for blk in range(Ncap // L):
            base = g.normal(size=D)
            dirs = g.normal(size=(3, D))
            coef = g.normal(size=(L, 3))
            K[0, h, blk * L:(blk + 1) * L] = base + coef @ dirs
    Kt = torch.tensor(K, dtype=torch.float32, device=DEV)
    sl = torch.tensor([Ncap], dtype=torch.int32, device=DEV)
    xi = kv.kv_build_block_cov_factors(Kt, sl, L, 4)
    torch.cuda.synchronize()
    xg = xi.cpu().numpy().astype(np.float64)
    K64 = to64(Kt)
    for h in range(Hkv):
        for blk in range(Ncap // L):
            s, e = blk * L, (blk + 1) * L
            X = K64[0, h, s:e] - K64[0, h, s:e].mean(axis=0)
            cov = X.T @ X / L
            for _ in range(3):
                qv = g.normal(size=D)
                exact = float(qv @ cov @ qv)
                got = float(np.sum((xg[0, h, blk] @ qv) ** 2))
                assert abs(got - exact) <= 1e-5 * max(1.0, exact), f"rank-3 block {(h, blk)}: {got} vs {exact}"
            assert float(np.sum(xg[0, h, blk, 3] ** 2)) <= 1e-6 * float(np.trace(cov))


def test_cov_factors_rejects_large_blocks():
    K = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device=DEV)
    sl = torch.tensor([256], dtype=torch.int32, device=DEV)
    with pytest.raises(Exception):
        kv.kv_build_block_cov_factors(K, sl, 128, 4)


@pytest.mark.parametrize("seq_lens,k", [([3000, 1100], None), ([4096, 65], 3), ([2000, 1], 40)])
def test_cobs_small_pipeline(seq_lens, k):
    wl = W.make("llama_cobs", DEV, B=len(seq_lens), Ncap=max(seq_lens), seq_lens=seq_lens, k_top=k)
    r = run_pipeline(wl)
    q, K, V = oracle_inputs(wl)
    pairs = all_pairs(wl)
    sel = O.select_batch(q, K, wl.seq_lens, wl.block_size, wl.scale, wl.k_top, True, True, "cobs")
    selection_matches(r["idx"], r["nk"], sel, pairs, "cobs select")
    S = r["scores"].cpu().numpy().astype(np.float64)
    for (b, h) in pairs:
        nb = len(sel[(b, h)]["S"])
        assert np.max(np.abs(S[b, h, :nb] - sel[(b, h)]["S"])) < 1e-4, f"group score at {(b, h)}"
    go = r["out"].cpu().numpy().astype(np.float64)
    G = wl.G
    for (b, h) in pairs:
        kept = r["idx"][b, h, :int(r["nk"][b, h])].cpu().tolist()
        o, l, _ = O.sparse_attend_one(q[b, h * G:(h + 1) * G], K[b, h], V[b, h], wl.seq_lens[b],
                                      wl.block_size, kept, wl.scale, True)
        assert row_rel_err(go[b, h * G:(h + 1) * G], o) <= OUT_TOL


def test_cobs_second_order_changes_the_ranking():
    # the second-order term is not a no-op: on this cache it changes some kept set
    # relative to first-order (mean-pool) scoring, and the GPU follows the oracle
    wl = W.make("llama_cobs", DEV, B=4, Ncap=8192, k_top=8)
    r = run_pipeline(wl)
    q, K, _ = oracle_inputs(wl)
    pairs = all_pairs(wl)
    s2 = O.select_batch(q, K, wl.seq_lens, wl.block_size, wl.scale, wl.k_top, True, True, "cobs")
    s1 = O.select_batch(q, K, wl.seq_lens, wl.block_size, wl.scale, wl.k_top, True, True, "summary")
    assert any(s1[p]["kept"] != s2[p]["kept"] for p in pairs), "second-order and first-order rankings agree everywhere"
    selection_matches(r["idx"], r["nk"], s2, pairs, "cobs select B=4")


def test_cobs_full_size_sampled():
    wl = W.make("llama_cobs", DEV)
    r = run_pipeline(wl, want_scores=False)
    gen = np.random.default_rng(13)
    pairs = sorted({(int(gen.integers(wl.B)), int(gen.integers(wl.Hkv))) for _ in range(2)} | {(0, 0)})
    q = to64(wl.q)
    res = {}
    for (b, h) in pairs:
        Kb = to64(wl.K[b:b + 1, h:h + 1])
        qb = q[b:b + 1, h * wl.G:(h + 1) * wl.G]
        res[(b, h)] = O.select_batch(qb, Kb, [wl.seq_lens[b]], wl.block_size, wl.scale, wl.k_top, True, True,
                                     "cobs")[(0, 0)]
    selection_matches(r["idx"], r["nk"], res, pairs, "full cobs select")


@pytest.mark.parametrize("name,rank,L", [
    ("llama", 3, 64),       # ring, two blocks a batch (6 of 8 rows)
    ("llama", 8, 64),       # ring, one block a batch
    ("qwen_long", 4, 64),   # G = 7: ring of 4 rows a stage, one block a batch
    ("qwen_long", 6, 32),   # G = 7, rank above the ring's rows: direct loads
    ("tiny", 2, 16),        # D = 64, fp32, G = 1: direct loads
])
def test_cobs_rank_and_shape_paths(name, rank, L):
    kw = dict(tiny=dict(), llama=dict(B=2, Ncap=2000, seq_lens=[2000, 900]),
              qwen_long=dict(B=2, Ncap=2053, seq_lens=[2053, 700]))[name]
    wl = W.make(name, DEV, **kw)
    sl = wl.seq_lens_tensor(DEV)
    k = 4
    summ = kv.kv_build_block_summaries(wl.K, wl.V, sl, L)
    xi = kv.kv_build_block_cov_factors(wl.K, sl, L, rank)
    idx, nk, sc = kv.kv_select_blocks_cobs(wl.q, wl.K, sl, L, wl.scale, summ["k_sum"], summ["counts"], xi, k,
                                           True, True, want_scores=True)
    torch.cuda.synchronize()
    q, K, _ = oracle_inputs(wl)
    pairs = all_pairs(wl)
    sel = O.select_batch(q, K, wl.seq_lens, L, wl.scale, k, True, True, "cobs", rank=rank)
    selection_matches(idx, nk, sel, pairs, f"cobs {name} rank={rank} L={L}")
    S = sc.cpu().numpy().astype(np.float64)
    for (b, h) in pairs:
        nb = len(sel[(b, h)]["S"])
        assert np.max(np.abs(S[b, h, :nb] - sel[(b, h)]["S"])) < 1e-4, f"group score at {(b, h)}"
