"""The warp-specialised block-mode attention kernel against the float64 oracle on
the paths of its own design: chunks of 32 rows (block size 32) and 64 rows
(block sizes 64 and 128: a block of 128 is two chunks), D = 64 (one 2-D box a
tile) and D = 128 (one 3-D box), group sizes 1..8, ranges of whole pairs
(at least as many pairs as CTAs) and ranges that share pairs between CTAs (fewer
pairs: partial records merged by the last arriving CTA), ragged and empty
sequences (chunks with fewer valid rows, empty chunks), kept lists shorter than
kmax, the tail proxy on and off, and repeated launches on one workspace (the
shared-pair counters must come back to zero)."""
import math

import numpy as np
import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from oracle import oracle as O

from gpu_helpers import check_out, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(B, Hkv, G, D, N, L, lens, k_top, seed, use_proxy=True, kmax_extra=0, reps=1):
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randn(B, Hkv * G, D, generator=g, device=DEV).to(torch.bfloat16)
    K = torch.randn(B, Hkv, N, D, generator=g, device=DEV).to(torch.bfloat16)
    V = torch.randn(B, Hkv, N, D, generator=g, device=DEV).to(torch.bfloat16)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    scale = 1 / math.sqrt(D)
    summ = kv.kv_build_block_summaries(K, V, sl, L)
    NB = (N + L - 1) // L
    kmax = min(NB, min(NB, k_top + 2) + kmax_extra)
    idx, nk, _ = kv.kv_select_blocks(q, K, sl, L, scale, summ["counts"], k_top, True, True, k_sum=summ["k_sum"],
                                     kmax=kmax)
    ws = kv.Workspace(kv.make_shape(q, K, sl, L), DEV)
    for _ in range(reps):
        out, lse = kv.kv_sparse_decode_attn(q, K, V, sl, L, scale, ws, block_idx=idx, n_kept=nk, summaries=summ,
                                            use_tail_proxy=use_proxy)
    torch.cuda.synchronize()
    assert kv.kv_workspace_status(ws.tensor) == 0
    q64, K64, V64 = to64(q), to64(K), to64(V)
    gi, gn = idx.cpu().numpy(), nk.cpu().numpy()
    pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    kept = {p: [int(x) for x in gi[p[0], p[1], :gn[p]]] for p in pairs}
    ro, rl = O.sparse_batch(q64, K64, V64, lens, L, scale, kept, use_proxy)
    check_out(out, lse, ro, rl, what=f"gather B={B} Hkv={Hkv} G={G} D={D} L={L} k={k_top} proxy={use_proxy}")
    # the counters the shared pairs use are back at zero after every launch
    ctr = ws.tensor[256:256 + 4 * B * Hkv].view(torch.int32)
    assert int(ctr.abs().sum()) == 0


@pytest.mark.parametrize("L", [32, 64, 128])
@pytest.mark.parametrize("G,D", [(1, 128), (4, 128), (7, 128), (8, 128), (2, 64), (5, 64), (8, 64)])
def test_block_sizes_and_groups(L, G, D):
    # 12 pairs on 148 SMs: ranges share pairs between CTAs
    _case(B=3, Hkv=4, G=G, D=D, N=3000, L=L, lens=[3000, 1777, 45], k_top=6, seed=L * 10 + G * 100 + D)


@pytest.mark.parametrize("L", [32, 64, 128])
def test_whole_pair_ranges(L):
    # 160 pairs >= 148 SMs: every CTA holds whole pairs (one or two)
    _case(B=40, Hkv=4, G=4, D=128, N=1300, L=L, lens=[1300 - 17 * i for i in range(40)], k_top=3,
          seed=7 + L)


def test_long_kept_lists_many_ctas_per_pair():
    # few pairs, long kept lists: each pair spans several CTAs
    _case(B=1, Hkv=2, G=4, D=128, N=16384, L=64, lens=[16000], k_top=120, seed=3)


def test_empty_sequences_and_short_lists():
    # seq_len 0 and 1, and kept lists shorter than kmax (empty chunks)
    _case(B=4, Hkv=2, G=4, D=128, N=2048, L=64, lens=[0, 1, 2048, 300], k_top=5, seed=11, kmax_extra=4)


@pytest.mark.parametrize("use_proxy", [True, False])
def test_proxy_on_off_repeated(use_proxy):
    _case(B=2, Hkv=8, G=4, D=128, N=4096, L=64, lens=[4096, 2500], k_top=5, seed=21, use_proxy=use_proxy, reps=3)
