"""The stored second-order descriptor on the GPU against the float64 oracle ("COBS:
Cumulant Order Block Sparse Attention", the subspace and quantisation paragraphs):
the query basis (eigenvalues, eigenvector directions where the spectrum separates
them, the subspace dimension s), the subspace covariance factors (eigenvalues and
quadratic forms, which do not depend on the eigenvectors' signs), the E2M1
quantiser (codes and scales bit-exact on shared inputs: both sides decide in
float32), and the selection it drives, with the GPU chain (basis, s, factors,
codes, scorer) and the oracle chain (its own basis, s, factors and codes, the basis
stored at fp32 like the GPU's) run independently: kept blocks bit-exact up to
flagged near ties, group scores, and attention over the chosen blocks. The
full-space FP4 variant (no basis) is covered the same way."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W
from oracle import oracle as O
from gpu_helpers import OUT_TOL, all_pairs, record_note, row_rel_err, selection_matches, to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
NC = 512  # calibration positions


def _pack(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def test_query_basis_and_rank():
    wl = W.make("llama_cobs_fp4", DEV, B=1, Ncap=256)
    Qc = W.calibration_queries(wl, NC)
    evecs, evals = kv.kv_build_query_basis(Qc, wl.Hkv)
    torch.cuda.synchronize()
    ev_o, vec_o = O.query_basis(to64(Qc), wl.Hkv)
    ge, gv = evals.cpu().double().numpy(), evecs.cpu().double().numpy()
    D = wl.D
    for h in range(wl.Hkv):
        top = float(ev_o[h, 0])
        assert np.max(np.abs(ge[h] - ev_o[h])) <= 1e-5 * top, f"eigenvalues of head {h}"
        checked = 0
        for j in range(D):
            lo = ev_o[h, j] - ev_o[h, j + 1] if j + 1 < D else np.inf
            hi = ev_o[h, j - 1] - ev_o[h, j] if j > 0 else np.inf
            if min(lo, hi) < 1e-3 * top:
                continue  # direction not separated from a neighbour: only the subspace is defined
            assert abs(float(gv[h, j] @ vec_o[h, j])) >= 1.0 - 1e-4, f"eigenvector {j} of head {h}"
            checked += 1
        assert checked >= D // 2
    s_gpu = kv.kv_query_subspace_rank(evals, 0.9)
    s_o, sh = O.subspace_rank(ev_o, 0.9)
    assert s_gpu == s_o, (s_gpu, s_o, sh)
    assert 60 <= s_o <= 100  # the anisotropic query model puts 90% of the energy in ~80 directions


def test_query_basis_fp32_d64_groups():
    # fp32 queries, D = 64, groups of 3 heads: every head of a group enters its moment
    g = torch.Generator(device=DEV).manual_seed(12)
    Hkv, G, D = 2, 3, 64
    A = torch.randn(D, D, generator=g, device=DEV) * torch.exp(-torch.arange(D, device=DEV) / 10.0)
    Qc = torch.randn(200, Hkv * G, D, generator=g, device=DEV) @ A.T
    evecs, evals = kv.kv_build_query_basis(Qc, Hkv)
    torch.cuda.synchronize()
    ev_o, vec_o = O.query_basis(to64(Qc), Hkv)
    ge, gv = evals.cpu().double().numpy(), evecs.cpu().double().numpy()
    for h in range(Hkv):
        assert np.max(np.abs(ge[h] - ev_o[h])) <= 1e-5 * float(ev_o[h, 0])
        for j in range(8):
            assert abs(float(gv[h, j] @ vec_o[h, j])) >= 1.0 - 1e-4
    assert kv.kv_query_subspace_rank(evals, 0.9) == O.subspace_rank(ev_o, 0.9)[0]


@pytest.mark.parametrize("length", [32, 96, 128])
def test_quantize_fp4_bit_exact(length):
    g = torch.Generator(device=DEV).manual_seed(length)
    n = 257
    x = torch.randn(n, length, generator=g, device=DEV) * torch.exp(torch.randn(n, 1, generator=g, device=DEV))
    x[0] = 0.0
    ties = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], device=DEV)
    x[1] = 0.0
    x[1, :8] = ties
    x[2] = -x[1]
    x[3, 1::2] = 0.0
    codes, scales = kv.kv_quantize_fp4(x)
    torch.cuda.synchronize()
    xc, gc, gs = x.cpu().numpy(), codes.cpu().numpy(), scales.cpu().numpy()
    for v in range(n):
        co, so = O.fp4_e2m1_quantize(xc[v])
        assert np.array_equal(gc[v], _pack(co)), f"codes of vector {v}"
        assert gs[v] == np.float32(so), f"scale of vector {v}"
    assert gs[0] == 0.0 and not gc[0].any()


def test_subspace_factors():
    # the model's own leading directions as the basis (a test input, not a GPU output)
    wl = W.make("llama_cobs_fp4", DEV, B=2, Ncap=700, seq_lens=[700, 321])
    R, _ = wl.q_model
    s = 40
    U = R[:, :s].T.contiguous().to(DEV)  # [s][D] rows the basis
    Uh = U.unsqueeze(0).expand(wl.Hkv, s, wl.D).contiguous()
    sl = wl.seq_lens_tensor(DEV)
    r = 4
    xi = kv.kv_build_block_cov_factors_ss(wl.K, sl, wl.block_size, Uh, r)
    torch.cuda.synchronize()
    assert xi.shape[-1] == 64 and float(xi[..., s:].abs().max()) == 0.0
    xg = xi.cpu().double().numpy()
    K64 = to64(wl.K)
    U64 = U.cpu().double().numpy()
    gen = np.random.default_rng(4)
    NB = xg.shape[2]
    for b in range(wl.B):
        for h in range(wl.Hkv):
            xo, lam = O.block_cov_factors_ss_one(K64[b, h], wl.seq_lens[b], wl.block_size, NB, r, U64)
            _, lam_all = O.block_cov_factors_ss_one(K64[b, h], wl.seq_lens[b], wl.block_size, NB, r + 1, U64)
            for blk in range(NB):
                top = max(float(lam[blk, 0]), 1e-30)
                lg = np.sum(xg[b, h, blk, :, :s] ** 2, axis=1)
                assert np.all(np.abs(lg - lam[blk]) <= 1e-5 * top + 1e-12), f"eigenvalues at {(b, h, blk)}"
                if (lam_all[blk, r - 1] - lam_all[blk, r]) / top < 1e-6:
                    continue
                for _ in range(2):
                    qv = gen.normal(size=s)
                    fg = float(np.sum((xg[b, h, blk, :, :s] @ qv) ** 2))
                    fo = float(np.sum((xo[blk] @ qv) ** 2))
                    assert abs(fg - fo) <= 1e-5 * top * float(qv @ qv) + 1e-12, f"quadratic form at {(b, h, blk)}"


def _gpu_chain(wl, r, subspace=True, Qc=None):
    sl = wl.seq_lens_tensor(DEV)
    L = wl.block_size
    summ = kv.kv_build_block_summaries(wl.K, wl.V, sl, L)
    k_mean = kv.kv_build_block_key_means(wl.K, sl, L, summ["k_sum"], summ["counts"])
    U, s = None, wl.D
    if subspace:
        evecs, evals = kv.kv_build_query_basis(Qc, wl.Hkv)
        s = kv.kv_query_subspace_rank(evals, 0.9)
        U = evecs[:, :s, :].contiguous()
        xi = kv.kv_build_block_cov_factors_ss(wl.K, sl, L, U, r)
    else:
        xi = kv.kv_build_block_cov_factors(wl.K, sl, L, r)
    codes, scl = kv.kv_quantize_fp4(xi)
    idx, nk, scores = kv.kv_select_blocks_cobs_fp4(wl.q, wl.K, sl, L, wl.scale, k_mean, summ["counts"], U, codes, scl,
                                                   r, wl.k_top, True, True, wl.kmax, want_scores=True)
    torch.cuda.synchronize()
    return dict(s=s, U=U, xi=xi, codes=codes, scl=scl, idx=idx, nk=nk, scores=scores, summ=summ, sl=sl)


def _oracle_chain(wl, K64, pairs, r, subspace=True, Qc=None):
    """The oracle's own descriptor: basis and s from the calibration queries, the basis
    stored at fp32, factors in float64 rounded to fp32, E2M1 codes (float32 decisions)."""
    D, L, NB = wl.D, wl.block_size, wl.NBcap
    U_pad, s = None, D
    if subspace:
        ev, vec = O.query_basis(to64(Qc), wl.Hkv)
        s, _ = O.subspace_rank(ev, 0.9)
        U32 = vec[:, :s, :].astype(np.float32).astype(np.float64)
    SP = (s + 31) // 32 * 32
    if subspace:
        U_pad = np.zeros((wl.Hkv, SP, D))
        U_pad[:, :s] = U32
    stored, mags = {}, {}
    for (b, h) in pairs:
        n = wl.seq_lens[b]
        if subspace:
            xo, _ = O.block_cov_factors_ss_one(K64[b, h], n, L, NB, r, U32[h])
        else:
            xo, _ = O.block_cov_factors_one(K64[b, h], n, L, NB, r)
        x32 = np.zeros((NB, r, SP), dtype=np.float32)
        x32[:, :, :xo.shape[-1]] = xo.astype(np.float32)
        dec = np.zeros((NB, r, SP))
        mg = np.zeros((NB, r, SP), dtype=np.uint8)
        for blk in range(NB):
            for i in range(r):
                c, sc = O.fp4_e2m1_quantize(x32[blk, i])
                dec[blk, i] = O.fp4_e2m1_decode(c, sc)
                mg[blk, i] = c & 7
        stored[(b, h)] = dec
        mags[(b, h)] = mg
    return s, U_pad, stored, mags


def _compare(wl, g, pairs, subspace, Qc, what, r=4):
    q64, K64, V64 = to64(wl.q), to64(wl.K), to64(wl.V)
    s_o, U_pad, stored, mags = _oracle_chain(wl, K64, pairs, r, subspace, Qc)
    assert g["s"] == s_o, (what, g["s"], s_o)
    # E2M1 magnitudes of the factors: the same wherever the two chains' fp32 factors
    # agree (signs are arbitrary per eigenvector)
    gc = g["codes"].cpu().numpy()
    flips = total = 0
    for (b, h) in pairs:
        lo = gc[b, h] & 0x0F
        hi = gc[b, h] >> 4
        gm = np.stack([lo, hi], axis=-1).reshape(mags[(b, h)].shape) & 7
        flips += int(np.sum(gm != mags[(b, h)]))
        total += gm.size
    assert flips <= max(2, total // 10000), f"{what}: {flips} of {total} E2M1 magnitudes differ"
    record_note(f"{what}: s = {s_o}; {flips} of {total} E2M1 magnitudes differ between the GPU and oracle chains")
    sel = O.select_batch(q64, K64, wl.seq_lens, wl.block_size, wl.scale, wl.k_top, True, True, "cobs_stored",
                         bh=pairs, rank=r, stored_xi=stored, stored_U=U_pad)
    selection_matches(g["idx"], g["nk"], sel, pairs, what)
    S = g["scores"].cpu().numpy().astype(np.float64)
    for (b, h) in pairs:
        nb = len(sel[(b, h)]["S"])
        assert np.max(np.abs(S[b, h, :nb] - sel[(b, h)]["S"])) < 1e-4, f"{what}: group score at {(b, h)}"
    # attention over the GPU's kept blocks
    ws = kv.Workspace(kv.make_shape(wl.q, wl.K, g["sl"], wl.block_size), DEV)
    out, _ = kv.kv_sparse_decode_attn(wl.q, wl.K, wl.V, g["sl"], wl.block_size, wl.scale, ws, block_idx=g["idx"],
                                      n_kept=g["nk"], summaries=g["summ"])
    go = out.cpu().numpy().astype(np.float64)
    G = wl.G
    for (b, h) in pairs:
        kept = [int(x) for x in g["idx"][b, h, :int(g["nk"][b, h])].cpu().tolist()]
        o, _, _ = O.sparse_attend_one(q64[b, h * G:(h + 1) * G], K64[b, h], V64[b, h], wl.seq_lens[b],
                                      wl.block_size, kept, wl.scale, True)
        assert row_rel_err(go[b, h * G:(h + 1) * G], o) <= OUT_TOL, (what, b, h)


@pytest.mark.parametrize("subspace", [True, False])
def test_cobs_fp4_pipeline_small(subspace):
    wl = W.make("llama_cobs_fp4", DEV, B=2, Ncap=4096, seq_lens=[4096, 1999], k_top=6)
    Qc = W.calibration_queries(wl, NC)
    g = _gpu_chain(wl, 4, subspace, Qc)
    _compare(wl, g, all_pairs(wl), subspace, Qc, f"cobs fp4 small subspace={subspace}")


def test_cobs_fp4_rank_paths():
    # rank 1 and rank 6 (the kernel's 8-factor path), groups of 4
    wl = W.make("llama_cobs_fp4", DEV, B=1, Ncap=2048, k_top=5)
    Qc = W.calibration_queries(wl, NC)
    for r in (1, 6):
        g = _gpu_chain(wl, r, True, Qc)
        _compare(wl, g, all_pairs(wl), True, Qc, f"cobs fp4 rank {r}", r=r)


def test_cobs_fp4_full_size_sampled():
    # the full Llama-shaped batch (32 x 32K, 1% read): sampled pairs; the descriptor
    # bytes a launch reads against the full-space fp32 descriptor's
    wl = W.make("llama_cobs_fp4", DEV)
    Qc = W.calibration_queries(wl, NC)
    g = _gpu_chain(wl, 4, True, Qc)
    pairs = [(0, 0), (7, 3), (19, 6), (31, 7)]
    _compare(wl, g, pairs, True, Qc, "cobs fp4 full size")
    NBt = wl.B * wl.Hkv * wl.NBcap
    stored = NBt * (wl.D * 2 + 4 * g["codes"].shape[-1] + 4 * 4)
    full = NBt * (wl.D * 4 + 4 * wl.D * 4)
    record_note(f"stored descriptor {stored / 1e6:.1f} MB vs full-space fp32 {full / 1e6:.1f} MB per launch")
    assert stored <= 0.3 * full
