"""The bf16 block-mean summary and the selector that scores from it.

The means must be bit-exact: the GPU rounds the correctly rounded fp32 quotient
k_sum / n_b to the nearest bf16, so the check takes the GPU's own fp32 sums,
forms that quotient in float32 and rounds it with the oracle's round_bf16 (the
decision is taken in the kernel's precision on both sides). The kept blocks must
match the oracle's bf16-mean ranking except at flagged near ties, over ragged
lengths and both top-k paths (k <= 16 per-warp, larger k radix select)."""
import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from oracle import oracle as O
from weighted_coreset_softmax_b200 import workloads as W

from gpu_helpers import OUT_TOL, check_out, oracle_inputs, run_pipeline, selection_matches, all_pairs

DEV = "cuda"


def _means_reference(k_sum_gpu, counts_gpu):
    ks = k_sum_gpu.cpu().numpy().astype(np.float32)          # [B][Hkv][NB][D]
    cn = counts_gpu.cpu().numpy()                             # [B][NB]
    n = cn[:, None, :, None].astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        quo = np.where(n > 0, ks / np.maximum(n, np.float32(1)), np.float32(0))   # float32 division
    return O.round_bf16(quo.astype(np.float64))


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", [
    ("llama", dict(B=3, Ncap=4096 + 64, seq_lens=[4160, 1000, 0])),
    ("llama", dict(B=2, Ncap=2048, seq_lens=[2048, 33])),
    ("qwen_long", dict(B=1, Ncap=8192, seq_lens=[8000])),
])
def test_key_means_bit_exact(name, kw):
    wl = W.make(name, DEV, **kw)
    sl = wl.seq_lens_tensor(DEV)
    su = kv.kv_build_block_summaries(wl.K, wl.V, sl, wl.block_size)
    km = kv.kv_build_block_key_means(wl.K, sl, wl.block_size, su["k_sum"], su["counts"])
    torch.cuda.synchronize()
    got = km.to(torch.float64).cpu().numpy()
    want = _means_reference(su["k_sum"], su["counts"])
    assert np.array_equal(got, want), f"{int(np.sum(got != want))} bf16 means differ"


@pytest.mark.gpu
@pytest.mark.parametrize("k_top", [1, 5, 16, 17, 40])
@pytest.mark.parametrize("ff,fl", [(True, True), (False, False), (True, False)])
def test_mean16_selection_and_attention(k_top, ff, fl):
    wl = W.make("llama", DEV, B=3, Ncap=6000, seq_lens=[6000, 2500, 97], k_top=k_top,
                score_mode="summary_mean16")
    wl.force_first, wl.force_last = int(ff), int(fl)
    r = run_pipeline(wl, want_scores=True)
    q, K, V = oracle_inputs(wl)
    sel = O.select_batch(q, K, wl.seq_lens, wl.block_size, wl.scale, wl.k_top, ff, fl, "summary_mean16")
    selection_matches(r["idx"], r["nk"], sel, all_pairs(wl), f"mean16 k={k_top} ff={ff} fl={fl}")
    # group scores: the oracle's bf16-mean scores, within fp32 rounding
    gs = r["scores"].cpu().numpy()
    for (b, h), s in sel.items():
        nb = len(s["S"])
        assert np.max(np.abs(gs[b, h, :nb] - s["S"])) <= 1e-4 * max(1.0, float(np.max(s["S"])))
    # attention over the GPU's kept blocks against the oracle on the same blocks
    gi, gn = r["idx"].cpu().numpy(), r["nk"].cpu().numpy()
    kept = {(b, h): [int(x) for x in gi[b, h, :gn[b, h]]] for (b, h) in all_pairs(wl)}
    ro, rl = O.sparse_batch(q, K, V, wl.seq_lens, wl.block_size, wl.scale, kept, True)
    check_out(r["out"], r["lse"], ro, rl, tol=OUT_TOL, what="mean16 attention")


@pytest.mark.gpu
def test_mean16_rejects_fp32_cache():
    wl = W.make("tiny", DEV)
    sl = wl.seq_lens_tensor(DEV)
    su = kv.kv_build_block_summaries(wl.K, wl.V, sl, wl.block_size)
    fake = torch.zeros(wl.B, wl.Hkv, wl.NBcap, wl.D, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(kv.KVError):
        kv.kv_select_blocks_mean16(wl.q.to(torch.bfloat16), wl.K, sl, wl.block_size, wl.scale, fake, su["counts"],
                                   wl.k_top)
