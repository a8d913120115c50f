"""The CUDA-core attention consumer on bf16 caches (selected by KVSPARSE_ATTN=fma,
read once per process) against the float64 oracle in block, dense and weighted
modes, run in a child process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import numpy as np, torch
import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W
from oracle import oracle as O
from gpu_helpers import all_pairs, check_out, oracle_inputs, run_pipeline, selection_matches
for name, kw in (("llama", dict(B=2, Ncap=3100, seq_lens=[3100, 777], budget=0.05)),
                 ("qwen_long", dict(B=1, Ncap=2100, k_top=3))):
    wl = W.make(name, "cuda", **kw)
    r = run_pipeline(wl)
    q, K, V = oracle_inputs(wl)
    gi, gn = r["idx"].cpu().numpy(), r["nk"].cpu().numpy()
    kept = {{(b, h): [int(x) for x in gi[b, h, :gn[b, h]]] for (b, h) in all_pairs(wl)}}
    ro, rl = O.sparse_batch(q, K, V, wl.seq_lens, wl.block_size, wl.scale, kept, True)
    check_out(r["out"], r["lse"], ro, rl, what=name + " cuda-core consumer")
    sl = wl.seq_lens_tensor("cuda")
    out, lse = kv.kv_dense_decode_attn(wl.q, wl.K, wl.V, sl, wl.block_size, wl.scale, r["ws"])
    do, dl = O.dense_batch(q, K, V, wl.seq_lens, wl.scale)
    check_out(out, lse, do, dl, what=name + " cuda-core dense")
# weighted coreset rows, one copy per gathered row
wc = W.make("llama_coreset", "cuda", B=2, Ncap=2500, seq_lens=[2500, 900], m=300)
slc = wc.seq_lens_tensor("cuda")
wsc = kv.Workspace(kv.make_shape(wc.q, wc.K, slc, wc.block_size), "cuda")
out, lse = kv.kv_sparse_decode_attn(wc.q, wc.K, wc.V, slc, wc.block_size, wc.scale, wsc, tok_idx=wc.tok_idx, w=wc.w)
torch.cuda.synchronize()
assert kv.kv_workspace_status(wsc.tensor) == 0
qc, Kc, Vc = oracle_inputs(wc)
ro, rl = O.weighted_batch(qc, Kc, Vc, wc.seq_lens, wc.tok_idx.cpu().numpy(), wc.w.cpu().numpy().astype(np.float64),
                          wc.scale)
check_out(out, lse, ro, rl, what="cuda-core weighted")
print("ok")
"""


def test_cuda_core_consumer_on_bf16():
    env = dict(os.environ, KVSPARSE_ATTN="fma")
    code = SCRIPT.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
