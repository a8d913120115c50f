"""The per-worker-ring tensor-core attention kernel in block mode (selected by
KVSPARSE_ATTN=v1, read once per process; the warp-specialised kernel is the
default there) against the float64 oracle, in a child process: the headline
shapes with every (sequence, KV head) pair merged in its CTA, few pairs split
over many workers, ragged lengths, and block sizes 32, 64 and 128."""
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
from gpu_helpers import all_pairs, check_out, oracle_inputs, run_pipeline
cases = (("llama", dict(B=32, Ncap=2048)),
         ("llama", dict(B=2, Ncap=3100, seq_lens=[3100, 777], budget=0.05)),
         ("qwen_long", dict(B=1, Ncap=4100, k_top=5)))
for name, kw in cases:
    wl = W.make(name, "cuda", **kw)
    r = run_pipeline(wl)
    q, K, V = oracle_inputs(wl)
    gi, gn = r["idx"].cpu().numpy(), r["nk"].cpu().numpy()
    kept = {{(b, h): [int(x) for x in gi[b, h, :gn[b, h]]] for (b, h) in all_pairs(wl)}}
    ro, rl = O.sparse_batch(q, K, V, wl.seq_lens, wl.block_size, wl.scale, kept, True)
    check_out(r["out"], r["lse"], ro, rl, what=name + " per-worker-ring kernel")
print("ok")
"""


def test_per_worker_ring_kernel_block_mode():
    env = dict(os.environ, KVSPARSE_ATTN="v1")
    code = SCRIPT.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
