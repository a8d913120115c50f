"""The WildCat coreset producer on the GPU against the float64 oracle.

The pivots are random draws whose inverse-CDF decisions depend on fp32 sums, so
they are checked step by step against the oracle replaying the GPU's own earlier
pivots: each pivot must be the oracle's draw for the same uniform over the
float64 residual diagonal, unless the uniform's target lies within a 1e-4
relative band of a cumulative-sum boundary (a near tie, counted and reported).
What is unique given the pivots is checked directly: the weights (the oracle's
kernel-distance solve for the GPU's pivots) and the coreset attention they give
(kv_sparse_decode_attn in weighted mode against the oracle's weighted attention).
Cluster sizes 1 to 8 CTAs per pair are covered, including clusters with CTAs
that own no tokens, and the full-size Llama-shaped cache on sampled pairs."""
import math

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from oracle import oracle as O

from gpu_helpers import OUT_TOL, record_near_ties, row_rel_err, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
BAND = 1e-4


def _inputs(B, Hkv, G, D, N, lens, dtype, seed, scale_keys=1.0):
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randn(B, Hkv * G, D, generator=g, device=DEV).to(dtype)
    K = (torch.randn(B, Hkv, N, D, generator=g, device=DEV) * scale_keys).to(dtype)
    V = torch.randn(B, Hkv, N, D, generator=g, device=DEV).to(dtype)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    return q, K, V, sl


def _check(q, K, V, sl, lens, m, sigma, seed, what, C=0, pairs=None):
    B, Hkv, N, D = K.shape
    G = q.shape[1] // Hkv
    gu = torch.Generator(device=DEV).manual_seed(seed + 1)
    u = torch.rand(B, Hkv, m, generator=gu, device=DEV).clamp_(1e-6, 1 - 1e-6)
    idx, w, nsel = kv.kv_build_wildcat_coreset(K, sl, sigma, m, u, ctas_per_pair=C)
    torch.cuda.synchronize()
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    q64 = to64(q)
    gi, gw, gn, gu_ = idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), nsel.cpu().numpy(), \
        u.cpu().numpy().astype(np.float64)
    ws = kv.Workspace(kv.make_shape(q, K, sl, 64), DEV)
    out, lse = kv.kv_sparse_decode_attn(q, K, V, sl, 64, sigma, ws, tok_idx=idx, w=w)
    torch.cuda.synchronize()
    assert kv.kv_workspace_status(ws.tensor) == 0
    go, gl = out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    steps = ties = 0
    for b, h in pairs:
        n = lens[b]
        Kp, Vp = to64(K[b, h]), to64(V[b, h])
        t_n = int(gn[b, h])
        S = [int(x) for x in gi[b, h, :t_n]]
        assert t_n == min(m, n) or (n > 0 and t_n > 0), (what, b, h, t_n)
        assert len(set(S)) == len(S) and all(0 <= s < n for s in S), (what, b, h)
        assert np.all(gw[b, h, t_n:] == 0)
        # each pivot: the oracle's draw over the float64 residual given the GPU's earlier pivots
        _, _, resid = O.rpcholesky_steps(Kp, n, sigma, gu_[b, h], t_n, pivots=S)
        for t, s in enumerate(S):
            d = resid[t]
            c = np.cumsum(d)
            tot = c[-1]
            target = gu_[b, h, t] * tot
            want = min(int(np.searchsorted(c, target, side="left")), n - 1)
            steps += 1
            if s != want:
                lo_s = c[s - 1] if s > 0 else 0.0
                near = min(abs(lo_s - target), abs(c[s] - target), abs(c[want] - target),
                           abs((c[want - 1] if want > 0 else 0.0) - target)) <= BAND * tot
                assert near and d[s] > 0, (what, b, h, t, s, want)
                ties += 1
        if not S:
            continue
        # the weights of the GPU's pivots, and the coreset attention
        wo, woc = O.wildcat_weights(Kp, n, sigma, S)
        scale_w = max(1.0, float(np.max(np.abs(woc))))
        assert np.max(np.abs(gw[b, h, :t_n] - woc)) <= 1e-2 * scale_w, (what, b, h)
        rows = slice(h * G, (h + 1) * G)
        o_gpu_w, l_gpu_w = O.weighted_attend_one(q64[b, rows], Kp, Vp, n, S, gw[b, h, :t_n], sigma)
        assert row_rel_err(go[b, rows], o_gpu_w) <= OUT_TOL, (what, "attention over the GPU coreset")
        o_orc, _ = O.weighted_attend_one(q64[b, rows], Kp, Vp, n, S, woc, sigma)
        assert row_rel_err(go[b, rows], o_orc) <= OUT_TOL, (what, "attention with the oracle's weights")
    record_near_ties(what + " (pivot draws)", steps, ties, ties)


@pytest.mark.parametrize("C", [0, 1, 3])
@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (64, torch.float32), (64, torch.bfloat16),
                                     (128, torch.float32)])
def test_wildcat_coreset(D, dtype, C):
    q, K, V, sl = _inputs(2, 2, 4, D, 1500, [1500, 700], dtype, seed=D)
    _check(q, K, V, sl, [1500, 700], 48, 1 / math.sqrt(D), seed=D, what=f"wildcat D={D} {dtype} C={C}", C=C)


def test_wildcat_clusters_with_idle_ctas():
    # 8 CTAs per pair over 100 and 33 tokens (4 and 2 groups of 32): CTAs that own
    # no group still take part in every exchange; m above n for the short one
    q, K, V, sl = _inputs(2, 1, 2, 128, 128, [100, 33], torch.bfloat16, seed=3)
    _check(q, K, V, sl, [100, 33], 40, 1 / math.sqrt(128), seed=3, what="wildcat 8 CTAs, short", C=8)


def test_wildcat_full_size_sampled():
    # the Llama-shaped cache at full size (8 x 32K, 8 KV heads, D = 128, bf16) with the
    # automatic cluster size; pivots, weights and attention of sampled pairs
    from weighted_coreset_softmax_b200 import workloads as W
    wl = W.make("llama", DEV)
    sl = wl.seq_lens_tensor(DEV)
    pairs = [(0, 0), (3, 5), (wl.B - 1, wl.Hkv - 1)]
    _check(wl.q, wl.K, wl.V, sl, wl.seq_lens, 64, wl.scale, seed=11, what="wildcat llama full size", pairs=pairs)


def test_wildcat_planted_keys():
    # Llama-shaped keys with planted heavy hitters: the producer must handle
    # kernel entries spread over many orders of magnitude
    from weighted_coreset_softmax_b200 import workloads as W
    wl = W.make("llama", DEV, B=2, Ncap=2048, seq_lens=[2048, 1500])
    sl = wl.seq_lens_tensor(DEV)
    _check(wl.q, wl.K, wl.V, sl, wl.seq_lens, 32, wl.scale, seed=5, what="wildcat llama-shaped")


def test_wildcat_degenerate():
    # identical keys: one pivot of weight n; an empty sequence: no pivot
    D, n = 64, 300
    k = torch.randn(D, device=DEV)
    K = k.repeat(1, 1, n, 1).to(torch.float32)
    K = torch.cat([K, K], dim=0)
    sl = torch.tensor([n, 0], dtype=torch.int32, device=DEV)
    u = torch.full((2, 1, 8), 0.5, device=DEV)
    idx, w, nsel = kv.kv_build_wildcat_coreset(K, sl, 0.125, 8, u)
    torch.cuda.synchronize()
    assert int(nsel[0, 0]) == 1 and int(nsel[1, 0]) == 0
    assert abs(float(w[0, 0, 0]) - n) <= 1e-3 * n
    assert float(w[0, 0, 1:].abs().sum()) == 0 and float(w[1].abs().sum()) == 0


def test_wildcat_rejects_bad_arguments():
    K = torch.zeros(1, 1, 64, 64, device=DEV)
    sl = torch.tensor([64], dtype=torch.int32, device=DEV)
    for m in (0, 65):
        with pytest.raises(kv.KVError):
            kv.kv_build_wildcat_coreset(K, sl, 0.1, m, torch.rand(1, 1, max(m, 1), device=DEV))
    for C in (-1, 9):
        with pytest.raises(kv.KVError):
            kv.kv_build_wildcat_coreset(K, sl, 0.1, 4, torch.rand(1, 1, 4, device=DEV), ctas_per_pair=C)
