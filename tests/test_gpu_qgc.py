"""Query-guided clusters with an error-gated read budget on the GPU against the
float64 oracle ("OpenAttention reads 1% of the KV cache", sections "Three helpers that
make the proxy accurate" and "Skipping reviews without losing the verdict"): the
projection (bf16 coordinates bit-exact), the k-means clusters (labels equal, or a
token equidistant within rounding of two centroids), the member lists and the cached
mean and variance tokens; then a decode step -- the errors' split of the read budget,
the tokens read in every cluster (bit-exact unless the oracle flags a near tie) and the
output (the read tokens plus one count-aware proxy per cluster) against the oracle's
own chain. The projection rows are a test input (the query model's leading
directions), not a GPU output."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W
from oracle import oracle as O
from gpu_helpers import OUT_TOL, record_near_ties, record_note, row_rel_err, to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _proj(wl):
    R, _ = wl.q_model
    P = R[:, :16].T.contiguous().to(DEV)  # [16][D]
    return P.unsqueeze(0).expand(wl.Hkv, 16, wl.D).contiguous()


def _check_build(wl, g, P, pairs, C, iters, what):
    K64, V64 = to64(wl.K), to64(wl.V)
    P64 = P[0].cpu().double().numpy()
    z16 = g["z16"].cpu().float().numpy()
    lab = g["labels"].cpu().numpy()
    perm, offs, cnt = g["perm"].cpu().numpy(), g["offs"].cpu().numpy(), g["counts"].cpu().numpy()
    ks, vs, kq = (g[k].cpu().double().numpy() for k in ("k_sum", "v_sum", "k_sq"))
    res = {}
    for (b, h) in pairs:
        n = wl.seq_lens[b]
        Z32 = O.qgc_project(K64[b, h], n, P64)
        zo = O.round_bf16(Z32.astype(np.float64))
        # z16 is in member order: entry m is token perm[m]'s projection
        bad = int(np.sum(z16[b, h, :n] != zo[perm[b, h, :n]]))
        assert bad <= max(1, n * 16 // 10000), f"{what}: {bad} bf16 coordinates differ at {(b, h)}"
        assert not np.any(z16[b, h, n:])
        lo, cent = O.qgc_kmeans(Z32, C, iters)
        Ce = min(C, n)
        diff = np.nonzero(lab[b, h, :n] != lo)[0]
        for i in diff:  # a token may only change sides where it is equidistant within rounding
            z = Z32[i].astype(np.float64)
            d = [float(np.sum((z - cent[c]) ** 2)) for c in range(Ce)]
            assert abs(d[int(lab[b, h, i])] - d[int(lo[i])]) <= 1e-9 * max(d), f"{what}: label of token {i}"
        assert len(diff) <= max(1, n // 1000), f"{what}: {len(diff)} labels differ at {(b, h)}"
        assert np.all(lab[b, h, n:] == -1)
        # member lists: every cluster's tokens, ascending, in its range
        assert offs[b, h, 0] == 0 and offs[b, h, C] == n
        for c in range(C):
            mem = perm[b, h, offs[b, h, c]:offs[b, h, c + 1]]
            assert cnt[b, h, c] == len(mem)
            assert np.all(np.diff(mem) > 0) and np.all(lab[b, h, mem] == c)
        # the cached tokens of the GPU's clusters
        co, kso, vso, kqo = O.qgc_cluster_stats(K64[b, h], V64[b, h], n, lab[b, h, :n], C)
        assert np.array_equal(co, cnt[b, h])
        for name, a, o in (("k_sum", ks, kso), ("v_sum", vs, vso), ("k_sq", kq, kqo)):
            sc = max(1.0, float(np.max(np.abs(o))))
            assert np.max(np.abs(a[b, h] - o)) <= 1e-5 * sc, f"{what}: {name} at {(b, h)}"
        res[(b, h)] = lo
    return res


def _decode_check(wl, P, qgc, budget, pairs, what):
    ws = kv.Workspace(kv.make_shape(wl.q, wl.K, wl.seq_lens_tensor(DEV), 64), DEV)
    sl = wl.seq_lens_tensor(DEV)
    out, lse, sel = kv.qgc_decode(wl.q, wl.K, wl.V, sl, wl.scale, P, qgc, budget, ws)
    torch.cuda.synchronize()
    assert kv.kv_workspace_status(ws.tensor) == 0
    tok, w, nr, pk, pv, pn = (x.cpu().numpy() for x in sel)
    go, gl = out.cpu().double().numpy(), lse.cpu().double().numpy()
    q64, K64, V64 = to64(wl.q), to64(wl.K), to64(wl.V)
    P64 = P[0].cpu().double().numpy()
    lab = qgc["labels"].cpu().numpy()
    C = qgc["C"]
    G = wl.G
    ties = flagged = 0
    for (b, h) in pairs:
        n = wl.seq_lens[b]
        rows = slice(h * G, (h + 1) * G)
        r = O.qgc_decode_one(q64[b, rows], K64[b, h], V64[b, h], n, P64, C, 8, budget, wl.scale)
        flagged += int(r["near_tie"])
        got = sorted(int(x) for x in tok[b, h, :nr[b, h]])
        assert np.all(w[b, h, :nr[b, h]] == 1.0) and np.all(w[b, h, nr[b, h]:] == 0.0)
        same_labels = np.array_equal(lab[b, h, :n], r["labels"])
        if got != r["read"]:
            assert r["near_tie"] or not same_labels, f"{what}: read set differs at {(b, h)} without a near tie"
            ties += 1
        # the output over the GPU's own read set and clusters, against the oracle
        o_own, l_own = O.qgc_attend_one(q64[b, rows], K64[b, h], V64[b, h], n, lab[b, h, :n], got, C, wl.scale)
        assert row_rel_err(go[b, rows], o_own) <= OUT_TOL, (what, b, h)
        fin = np.isfinite(l_own)
        assert np.all(np.abs(gl[b, rows][fin] - l_own[fin]) <= 1e-3 * np.maximum(1.0, np.abs(l_own[fin])))
        if got == r["read"] and same_labels:
            assert row_rel_err(go[b, rows], r["out"]) <= OUT_TOL, (what, b, h)
        # proxies: counts of unread tokens
        rc = np.bincount(lab[b, h, got], minlength=C) if got else np.zeros(C, dtype=np.int64)
        assert np.array_equal(pn[b, h], qgc["counts"][b, h].cpu().numpy() - rc)
    record_near_ties(what, len(pairs), flagged, ties)
    return out, lse, sel


@pytest.mark.parametrize("D,dtype,G", [(128, torch.bfloat16, 4), (64, torch.float32, 2), (64, torch.bfloat16, 2),
                                       (128, torch.bfloat16, 7)])
def test_qgc_small(D, dtype, G):
    if D == 128 and G == 4:
        wl = W.make("llama_cobs_fp4", DEV, B=2, Ncap=3000, seq_lens=[3000, 1234])
        P = _proj(wl)
    elif D == 128:
        # G = 7 (the Qwen-shaped group) on a bf16 cache from the same recipe: the
        # selection's two-product path for G > 4
        wl = W.make("llama_cobs_fp4", DEV, B=2, Ncap=2500, seq_lens=[2500, 777])
        gq = torch.Generator(device=DEV).manual_seed(4)
        wl.Hkv, wl.Hq = 2, 14
        wl.K = wl.K[:, :2].contiguous()
        wl.V = wl.V[:, :2].contiguous()
        wl.q = (torch.randn(2, 14, 128, generator=gq, device=DEV) * 1.5).to(torch.bfloat16)
        P = _proj(wl)
    else:
        gq = torch.Generator(device=DEV).manual_seed(2)
        wl = W.make("llama_cobs_fp4", DEV, B=2, Ncap=2000, seq_lens=[2000, 333])
        # a D = 64 cache (fp32 or bf16) with G = 2 from the same recipe's shapes
        wl.D, wl.Hq, wl.Hkv = 64, 4, 2
        wl.K = (torch.randn(2, 2, 2000, 64, generator=gq, device=DEV) * torch.exp(
            0.5 * torch.randn(2, 2, 1, 64, generator=gq, device=DEV))).to(dtype)
        wl.V = torch.randn(2, 2, 2000, 64, generator=gq, device=DEV).to(dtype)
        wl.q = torch.randn(2, 4, 64, generator=gq, device=DEV).to(dtype)
        wl.scale = 1 / math.sqrt(64)
        Rm = torch.linalg.qr(torch.randn(64, 64, generator=torch.Generator().manual_seed(3), dtype=torch.float64))[0]
        P = Rm[:, :16].T.contiguous().float().to(DEV).unsqueeze(0).expand(2, 16, 64).contiguous()
    C, iters = 16, 8
    sl = wl.seq_lens_tensor(DEV)
    qgc = kv.kv_build_qgc(wl.K, wl.V, sl, P, C, iters)
    torch.cuda.synchronize()
    pairs = [(b, h) for b in range(wl.B) for h in range(wl.Hkv)]
    _check_build(wl, qgc, P, pairs, C, iters, f"qgc build D={D}")
    _decode_check(wl, P, qgc, 0.05, pairs, f"qgc decode D={D}")


def test_qgc_large_clusters():
    # two clusters over 9,000 tokens: clusters above the 3,072 scores a warp's idle
    # ring holds, so the selection reads their scores from the scratch; a ragged
    # length below a whole 128-token chunk and a 16-token step
    wl = W.make("llama_cobs_fp4", DEV, B=1, Ncap=9000, seq_lens=[8999])
    P = _proj(wl)
    C, iters = 2, 8
    sl = wl.seq_lens_tensor(DEV)
    qgc = kv.kv_build_qgc(wl.K, wl.V, sl, P, C, iters)
    torch.cuda.synchronize()
    pairs = [(0, h) for h in range(wl.Hkv)]
    cnt = qgc["counts"].cpu().numpy()
    assert cnt.max() > 3072
    _check_build(wl, qgc, P, pairs, C, iters, "qgc build large clusters")
    _decode_check(wl, P, qgc, 0.05, pairs, "qgc decode large clusters")


def test_qgc_edges():
    # an empty sequence, one shorter than the cluster count, a zero budget (proxies
    # only) and one cluster
    wl = W.make("llama_cobs_fp4", DEV, B=3, Ncap=512, seq_lens=[0, 9, 512])
    P = _proj(wl)
    sl = wl.seq_lens_tensor(DEV)
    for C, budget in ((16, 0.05), (1, 0.0), (16, 0.0)):
        qgc = kv.kv_build_qgc(wl.K, wl.V, sl, P, C, 4)
        torch.cuda.synchronize()
        pairs = [(b, h) for b in (1, 2) for h in range(wl.Hkv)]
        _check_build(wl, qgc, P, pairs, C, 4, f"qgc edges C={C}")
        out, lse, sel = _decode_check(wl, P, qgc, budget, pairs, f"qgc edges C={C} budget={budget}")
        assert int(sel[2][0].sum()) == 0 and int(sel[5][0].sum()) == 0  # the empty sequence reads nothing
        if budget == 0.0:
            assert int(sel[2].sum()) == 0


def test_qgc_equal_logits_is_dense():
    # clusters of identical keys: every proxy is exact, so the step equals dense attention
    B, Hkv, G, D, per, C = 1, 2, 4, 128, 64, 8
    g = torch.Generator(device=DEV).manual_seed(5)
    keys = torch.randn(Hkv, C, D, generator=g, device=DEV) * 3.0
    K = keys.repeat_interleave(per, dim=1).unsqueeze(0).to(torch.bfloat16).contiguous()
    V = torch.randn(B, Hkv, C * per, D, generator=g, device=DEV).to(torch.bfloat16)
    q = torch.randn(B, Hkv * G, D, generator=g, device=DEV).to(torch.bfloat16)
    sl = torch.tensor([C * per], dtype=torch.int32, device=DEV)
    # projection rows spanning the cluster keys (8 directions) and 8 more: the
    # clusters are separated in the projection
    Pk = torch.linalg.qr(keys[0].T.double().cpu(), mode="complete")[0][:, :16].T.float().to(DEV)
    P = Pk.unsqueeze(0).expand(Hkv, 16, D).contiguous()
    qgc = kv.kv_build_qgc(K, V, sl, P, C, 6)
    ws = kv.Workspace(kv.make_shape(q, K, sl, 64), DEV)
    out, lse, sel = kv.qgc_decode(q, K, V, sl, 1 / math.sqrt(D), P, qgc, 0.05, ws)
    torch.cuda.synchronize()
    q64, K64, V64 = to64(q), to64(K), to64(V)
    for h in range(Hkv):
        od, ld = O.dense_attend_one(q64[0, h * G:(h + 1) * G], K64[0, h], V64[0, h], C * per, 1 / math.sqrt(D))
        assert row_rel_err(out[0, h * G:(h + 1) * G].cpu().double().numpy(), od) <= OUT_TOL


def test_qgc_full_size_sampled():
    # the Llama-shaped batch at full size (32 x 32K), 32 clusters, 1% read: sampled pairs
    wl = W.make("llama_cobs_fp4", DEV)
    P = _proj(wl)
    sl = wl.seq_lens_tensor(DEV)
    qgc = kv.kv_build_qgc(wl.K, wl.V, sl, P, 32, 8)
    torch.cuda.synchronize()
    pairs = [(0, 0), (13, 5), (31, 7)]
    _check_build(wl, qgc, P, pairs, 32, 8, "qgc build full size")
    _, _, sel = _decode_check(wl, P, qgc, 0.01, pairs, "qgc decode full size")
    record_note(f"qgc full size: tokens read per (sequence, KV head): mean {float(sel[2].float().mean()):.1f}")
