"""Both ranking paths of the block selector against the float64 oracle ("COBS:
Cumulant Order Block Sparse Attention", Equation (5)): k up to 16 takes the
per-warp top-k, larger k the radix select, and k at or above the candidate count
keeps every block. Every forcing combination, summary and Quest scoring, and
ragged lengths whose last block is partial."""
from __future__ import annotations

import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W
from oracle import oracle as O
from gpu_helpers import all_pairs, oracle_inputs, selection_matches

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

LENS = [8192, 5000, 1100, 129]  # 128, 79, 18 and 3 valid blocks of 64


@pytest.mark.parametrize("k", [1, 5, 16, 17, 40, 200])
@pytest.mark.parametrize("ff,fl", [(False, False), (True, False), (False, True), (True, True)])
@pytest.mark.parametrize("mode", ["summary", "quest"])
def test_select_paths(k, ff, fl, mode):
    name = "llama_quest" if mode == "quest" else "llama"
    wl = W.make(name, DEV, B=len(LENS), Ncap=max(LENS), seq_lens=LENS, k_top=k, seed=21)
    sl = wl.seq_lens_tensor(DEV)
    L = wl.block_size
    if mode == "quest":
        kb = kv.kv_build_block_bounds(wl.K, sl, L)
        idx, nk, _ = kv.kv_select_blocks_quest(wl.q, wl.K, sl, L, wl.scale, kb, k, ff, fl)
    else:
        summ = kv.kv_build_block_summaries(wl.K, wl.V, sl, L)
        idx, nk, _ = kv.kv_select_blocks(wl.q, wl.K, sl, L, wl.scale, summ["counts"], k, ff, fl,
                                         k_sum=summ["k_sum"])
    torch.cuda.synchronize()
    q, K, _ = oracle_inputs(wl)
    sel = O.select_batch(q, K, wl.seq_lens, L, wl.scale, k, ff, fl, mode)
    selection_matches(idx, nk, sel, all_pairs(wl), f"{mode} k={k} ff={ff} fl={fl}")
    for (b, h) in all_pairs(wl):
        nbv = (wl.seq_lens[b] + L - 1) // L
        forced = len({i for i, f in ((0, ff), (nbv - 1, fl)) if f and nbv > 0})
        assert int(nk[b, h]) == min(nbv, k + forced), f"n_kept at {(b, h)}"
