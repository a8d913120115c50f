"""GPU parity of kv_decode_step: selection (summary mode) and attention in one
call, in both forms -- the two kernels back to back, and the single fused kernel
(bf16 caches where the per-CTA layout fits; it falls back to two kernels
otherwise). The kept sets must match the float64 oracle's (up to flagged near
ties) and the outputs must match the oracle's attention over the kept sets, with
and without the tail proxy, for ragged lengths, and at full size on sampled
(sequence, KV head) pairs."""

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W
from oracle import oracle as O
from gpu_helpers import OUT_TOL, all_pairs, check_out, oracle_inputs, row_rel_err, selection_matches, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


HOWS = [kv.KV_STEP_FUSED, kv.KV_STEP_TWO_KERNELS]


def decode_step(wl, use_proxy=True, want_scores=False, how=kv.KV_STEP_FUSED):
    sl = wl.seq_lens_tensor(DEV)
    summ = kv.kv_build_block_summaries(wl.K, wl.V, sl, wl.block_size)
    ws = kv.Workspace(kv.make_shape(wl.q, wl.K, sl, wl.block_size), DEV)
    NB = (wl.Ncap + wl.block_size - 1) // wl.block_size
    scores = torch.full((wl.B, wl.Hkv, NB), -1.0, device=DEV) if want_scores else None
    out, lse, idx, nk = kv.kv_decode_step(wl.q, wl.K, wl.V, sl, wl.block_size, wl.scale, ws, summ, wl.k_top,
                                          wl.force_first, wl.force_last, use_tail_proxy=use_proxy, scores=scores,
                                          how=how)
    torch.cuda.synchronize()
    assert kv.kv_workspace_status(ws.tensor) == 0
    return out, lse, idx, nk, scores


CASES = [
    ("llama", dict(B=32, Ncap=1024, k_top=2)),                                   # 256 pairs, one kernel
    ("llama", dict(B=3, Ncap=4160, seq_lens=[4160, 3001, 70], budget=0.05)),     # ragged, 5 %
    ("llama", dict(B=2, Ncap=2048, seq_lens=[2048, 1], k_top=3)),                # a 1-token sequence
    ("llama", dict(B=4, Ncap=640, seq_lens=[0, 1, 640, 200], k_top=0)),          # empty sequence, k = 0
    ("qwen_long", dict(B=2, Ncap=4096 + 128 + 5, seq_lens=[4229, 2000], k_top=4)),  # G = 7: two kernels
]


@pytest.mark.parametrize("name,kw", CASES)
@pytest.mark.parametrize("use_proxy", [True, False])
@pytest.mark.parametrize("how", HOWS)
def test_decode_step_matches_oracle(name, kw, use_proxy, how):
    wl = W.make(name, DEV, **kw)
    out, lse, idx, nk, _ = decode_step(wl, use_proxy, how=how)
    q, K, V = oracle_inputs(wl)
    sel = O.select_batch(q, K, wl.seq_lens, wl.block_size, wl.scale, wl.k_top, True, True, "summary")
    selection_matches(idx, nk, sel, all_pairs(wl), f"{name} decode-step select")
    gi, gn = idx.cpu().numpy(), nk.cpu().numpy()
    kept = {(b, h): [int(x) for x in gi[b, h, :gn[b, h]]] for (b, h) in all_pairs(wl)}
    ro, rl = O.sparse_batch(q, K, V, wl.seq_lens, wl.block_size, wl.scale, kept, use_proxy)
    check_out(out, lse, ro, rl, what=f"{name} decode step proxy={use_proxy}")


def test_decode_step_scores_match_selector():
    """The optional scores output equals the separate selector's (same Eq. 5 group
    scores, different summation order: fp32 rounding only)."""
    wl = W.make("llama", DEV, B=32, Ncap=1024 + 37, seq_lens=[1061 - 13 * i for i in range(32)], k_top=3)
    _, _, _, _, scores = decode_step(wl, want_scores=True)
    sl = wl.seq_lens_tensor(DEV)
    summ = kv.kv_build_block_summaries(wl.K, wl.V, sl, wl.block_size)
    _, _, ref = kv.kv_select_blocks(wl.q, wl.K, sl, wl.block_size, wl.scale, summ["counts"], wl.k_top, True, True,
                                    k_sum=summ["k_sum"], want_scores=True)
    torch.cuda.synchronize()
    assert torch.allclose(scores, ref, rtol=1e-4, atol=1e-7)


def test_decode_step_forms_agree():
    """Both forms give the same kept sets and outputs within the tolerance."""
    wl = W.make("llama", DEV, B=32, Ncap=1024, k_top=2)
    r = {how: decode_step(wl, how=how) for how in HOWS}
    a, b = r[kv.KV_STEP_FUSED], r[kv.KV_STEP_TWO_KERNELS]
    assert torch.equal(a[3], b[3]) and torch.equal(a[2], b[2])
    err = row_rel_err(a[0].cpu().numpy().astype(np.float64), b[0].cpu().numpy().astype(np.float64))
    assert err <= OUT_TOL, err


@pytest.mark.parametrize("how", HOWS)
def test_decode_step_full_size_sampled(how):
    wl = W.make("llama", DEV, budget=0.01)
    out, lse, idx, nk, _ = decode_step(wl, how=how)
    gen = np.random.default_rng(11)
    pairs = sorted({(int(gen.integers(wl.B)), int(gen.integers(wl.Hkv))) for _ in range(3)}
                   | {(0, 0), (wl.B - 1, wl.Hkv - 1)})
    q = to64(wl.q)
    res_sel = {}
    go = out.cpu().numpy().astype(np.float64)
    for (b, h) in pairs:
        Kb = to64(wl.K[b:b + 1, h:h + 1])
        Vb = to64(wl.V[b:b + 1, h:h + 1])
        qb = q[b:b + 1, h * wl.G:(h + 1) * wl.G]
        sel = O.select_batch(qb, Kb, [wl.seq_lens[b]], wl.block_size, wl.scale, wl.k_top, True, True, "summary")
        res_sel[(b, h)] = sel[(0, 0)]
        gi = idx[b, h, :int(nk[b, h])].cpu().tolist()
        o, l, _ = O.sparse_attend_one(qb[0], Kb[0, 0], Vb[0, 0], wl.seq_lens[b], wl.block_size, gi, wl.scale, True)
        err = row_rel_err(go[b, h * wl.G:(h + 1) * wl.G], o)
        assert err <= OUT_TOL, f"full decode step {(b, h)}: {err:.3e}"
    selection_matches(idx, nk, res_sel, pairs, "full decode step select")
