"""Quest key-box scoring on the GPU against the float64 oracle ("COBS: Cumulant
Order Block Sparse Attention", the Quest paragraph, scored through Equation (5)):
the per-block key bounds bit-exact, the kept blocks bit-exact up to flagged near
ties, the group scores within fp32 rounding, and the attention over the chosen
blocks within the output tolerance."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W
from oracle import oracle as O
from gpu_helpers import OUT_TOL, all_pairs, check_out, oracle_inputs, row_rel_err, run_pipeline, \
    selection_matches, to64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _bounds_match(kb, K64, seq_lens, L, pairs):
    got = kb.to(torch.float32).cpu().numpy().astype(np.float64)
    NB = got.shape[2]
    for (b, h) in pairs:
        kmin, kmax = O.block_bounds_one(K64[b, h], int(seq_lens[b]), L, NB)
        assert np.array_equal(got[b, h, :, :, 0], kmin), f"min bounds differ at {(b, h)}"
        assert np.array_equal(got[b, h, :, :, 1], kmax), f"max bounds differ at {(b, h)}"


@pytest.mark.parametrize("D", [64, 128])
def test_block_bounds_exact(D):
    # ragged lengths: a partial last block, an empty sequence, one token
    gen = torch.Generator(device=DEV)
    gen.manual_seed(11)
    B, Hkv, Ncap, L = 4, 3, 1000, 64
    K = torch.randn(B, Hkv, Ncap, D, generator=gen, device=DEV).to(torch.bfloat16)
    lens = [1000, 999, 0, 1]
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    kb = kv.kv_build_block_bounds(K, sl, L)
    torch.cuda.synchronize()
    _bounds_match(kb, to64(K), lens, L, [(b, h) for b in range(B) for h in range(Hkv)])


def test_block_bounds_rejects_fp32():
    K = torch.zeros(1, 1, 64, 64, dtype=torch.float32, device=DEV)
    sl = torch.tensor([64], dtype=torch.int32, device=DEV)
    with pytest.raises(Exception):
        kv.kv_build_block_bounds(K, sl, 64)


@pytest.mark.parametrize("seq_lens", [[3000, 1100], [4096, 65]])
@pytest.mark.parametrize("use_proxy", [True, False])
def test_quest_small_pipeline(seq_lens, use_proxy):
    wl = W.make("llama_quest", DEV, B=len(seq_lens), Ncap=max(seq_lens), seq_lens=seq_lens)
    r = run_pipeline(wl, use_proxy=use_proxy)
    q, K, V = oracle_inputs(wl)
    pairs = all_pairs(wl)
    _bounds_match(r["summ"]["k_bounds"], K, wl.seq_lens, wl.block_size, pairs)
    sel = O.select_batch(q, K, wl.seq_lens, wl.block_size, wl.scale, wl.k_top, True, True, "quest")
    selection_matches(r["idx"], r["nk"], sel, pairs, "quest select")
    S = r["scores"].cpu().numpy().astype(np.float64)
    for (b, h) in pairs:
        nb = len(sel[(b, h)]["S"])
        assert np.max(np.abs(S[b, h, :nb] - sel[(b, h)]["S"])) < 1e-4, f"group score at {(b, h)}"
    # attention over the blocks the GPU chose, proxy from the GPU's own sums
    go = r["out"].cpu().numpy().astype(np.float64)
    gl = r["lse"].cpu().numpy().astype(np.float64)
    for (b, h) in pairs:
        kept = r["idx"][b, h, :int(r["nk"][b, h])].cpu().tolist()
        G = wl.G
        o, l, _ = O.sparse_attend_one(q[b, h * G:(h + 1) * G], K[b, h], V[b, h], wl.seq_lens[b],
                                      wl.block_size, kept, wl.scale, use_proxy)
        err = row_rel_err(go[b, h * G:(h + 1) * G], o)
        assert err <= OUT_TOL, f"quest attention {(b, h)}: {err:.3e}"
        assert np.max(np.abs(gl[b, h * G:(h + 1) * G] - l)) <= OUT_TOL * max(1.0, float(np.max(np.abs(l))))


def test_quest_k_covers_everything():
    # k_top >= valid blocks: every block kept, the tail is empty and the output is dense
    wl = W.make("llama_quest", DEV, B=2, Ncap=1500, seq_lens=[1500, 700], k_top=64)
    r = run_pipeline(wl)
    q, K, V = oracle_inputs(wl)
    for (b, h) in all_pairs(wl):
        nb = (wl.seq_lens[b] + wl.block_size - 1) // wl.block_size
        assert int(r["nk"][b, h]) == nb
        assert r["idx"][b, h, :nb].cpu().tolist() == list(range(nb))
    ref_o, ref_l = O.dense_batch(q, K, V, wl.seq_lens, wl.scale)
    check_out(r["out"], r["lse"], ref_o, ref_l, what="quest all kept = dense")


def test_quest_full_size_sampled():
    wl = W.make("llama_quest", DEV)
    r = run_pipeline(wl)
    gen = np.random.default_rng(9)
    pairs = sorted({(int(gen.integers(wl.B)), int(gen.integers(wl.Hkv))) for _ in range(3)}
                   | {(0, 0), (wl.B - 1, wl.Hkv - 1)})
    q = to64(wl.q)
    kb = r["summ"]["k_bounds"]
    res_sel = {}
    for (b, h) in pairs:
        Kb = to64(wl.K[b:b + 1, h:h + 1])
        qb = q[b:b + 1, h * wl.G:(h + 1) * wl.G]
        sel = O.select_batch(qb, Kb, [wl.seq_lens[b]], wl.block_size, wl.scale, wl.k_top, True, True, "quest")
        res_sel[(b, h)] = sel[(0, 0)]
        kmin, kmax = O.block_bounds_one(Kb[0, 0], wl.seq_lens[b], wl.block_size, kb.shape[2])
        got = kb[b, h].to(torch.float32).cpu().numpy().astype(np.float64)
        assert np.array_equal(got[..., 0], kmin) and np.array_equal(got[..., 1], kmax)
    selection_matches(r["idx"], r["nk"], res_sel, pairs, "full quest select")
