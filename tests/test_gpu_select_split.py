"""The few-pairs selector (each pair's blocks over a cluster of 2 to 8 CTAs, chosen
when at least two CTAs per pair fit on the SMs) against the float64 oracle: kept
blocks bit-exact except at flagged near ties, group scores, forced blocks, k from 0
to 16, empty sequences and single blocks, the fp32-sum and bf16-mean scorers, and pair
counts that give every cluster size."""
import math

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from oracle import oracle as O
from gpu_helpers import selection_matches, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(B, Hkv, G, lens, k, ff, fl, mode, seed, L=64, Ncap=None):
    Ncap = Ncap or max(max(lens), 1)
    D = 128
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randn(B, Hkv * G, D, generator=g, device=DEV).to(torch.bfloat16)
    K = (torch.randn(B, Hkv, Ncap, D, generator=g, device=DEV)
         * torch.exp(0.5 * torch.randn(B, Hkv, 1, D, generator=g, device=DEV))).to(torch.bfloat16)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    summ = kv.kv_build_block_summaries(K, K, sl, L)
    NB = (Ncap + L - 1) // L
    kmax = max(1, min(NB, k + int(ff) + int(fl)))
    scale = 1 / math.sqrt(D)
    if mode == "mean16":
        km = kv.kv_build_block_key_means(K, sl, L, summ["k_sum"], summ["counts"])
        idx, nk, sc = kv.kv_select_blocks_mean16(q, K, sl, L, scale, km, summ["counts"], k, ff, fl, kmax=kmax,
                                                 want_scores=True)
        omode = "summary_mean16"
    else:
        idx, nk, sc = kv.kv_select_blocks(q, K, sl, L, scale, summ["counts"], k, ff, fl, k_sum=summ["k_sum"],
                                          kmax=kmax, want_scores=True)
        omode = "summary"
    torch.cuda.synchronize()
    ref = O.select_batch(to64(q), to64(K), lens, L, scale, k, ff, fl, omode)
    pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    selection_matches(idx, nk, ref, pairs, f"split selector {mode} B={B} Hkv={Hkv} k={k}")
    S = sc.cpu().numpy().astype(np.float64)
    for (b, h) in pairs:
        nb = len(ref[(b, h)]["S"])
        if nb:
            assert np.max(np.abs(S[b, h, :nb] - ref[(b, h)]["S"])) < 1e-4, (b, h)
        assert np.all(S[b, h, nb:] == 0.0)


@pytest.mark.parametrize("mode", ["mean16", "sum32"])
@pytest.mark.parametrize("k,ff,fl", [(5, True, True), (0, True, True), (1, False, True), (16, True, False),
                                     (3, False, False)])
def test_split_single_sequence(mode, k, ff, fl):
    # 8 pairs: clusters of 8 CTAs
    _case(1, 8, 4, [9000], k, ff, fl, mode, seed=k + 10 * ff + 100 * fl)


@pytest.mark.parametrize("mode", ["mean16", "sum32"])
def test_split_ragged_and_empty(mode):
    # 4 pairs (clusters of 8): an empty sequence, one block, one token, a long one
    _case(4, 1, 7, [0, 64, 1, 5000], 5, True, True, mode, seed=3)
    _case(4, 1, 7, [0, 64, 1, 5000], 16, False, False, mode, seed=4)


@pytest.mark.parametrize("B,Hkv,G", [(8, 4, 7), (35, 2, 4), (5, 4, 4)])
def test_split_cluster_sizes(B, Hkv, G):
    # 32 pairs (clusters of 4), 70 pairs (2), 20 pairs (7)
    lens = [3000 - 37 * i for i in range(B)]
    _case(B, Hkv, G, lens, 10, True, True, "mean16", seed=B + Hkv)
