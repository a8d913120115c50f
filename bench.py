#!/usr/bin/env python
"""Decode-step benchmark of reduced-KV softmax attention on B200.

One step = one decode step of one layer for the whole batch: block selection per
KV head (kv_select_blocks, summary mode) and attention over the kept blocks plus
the tail proxy (kv_sparse_decode_attn). The block summaries are built once before
timing (they belong to prefill). Default workload: Llama-3.1-8B-shaped GQA decode
(32 query heads, 8 KV heads, head dim 128), batch 32, 32K context, block 64, 1%
read budget (top-5 + first + last block + proxy), synthetic bf16 cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch with torch.distributed.run: every rank runs its own batch on its
GPU (weak scaling, no collective on the data path); value = queries of all ranks /
max-over-ranks time. `--impl reference` times the float64 CPU oracle on the host
cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse decode queries/s and achieved HBM GB/s (% of 8 TB/s) at B=32, 32K ctx"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama", choices=["llama", "llama_b1", "qwen_long", "llama_osa", "llama_quest",
                                                           "llama_cobs", "llama_cobs_fp4", "llama_qgc",
                                                           "llama_coreset"])
    ap.add_argument("--scorer", choices=["mean16", "sum32"], default="mean16",
                    help="summary-mode selection: bf16 block means (default) or fp32 block sums")
    ap.add_argument("--attn", choices=["v1", "v2"], default=None,
                    help="attention kernel for block mode (default: the library's choice)")
    ap.add_argument("--no-secondary", action="store_true", help="skip the 5%% budget line and the read floor")
    ap.add_argument("--no-selection-check", action="store_true", help="skip the oracle check of the kept blocks")
    ap.add_argument("--budget", type=float, default=0.01)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU-baseline work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--rot", type=int, default=None,
                    help="independent batches rotated through the steps (default: enough to pass twice "
                         "the L2 capacity between two uses of a batch; 1 for small profiling captures)")
    ap.add_argument("--wildcat-m", type=int, default=64,
                    help="coreset size of the timed WildCat build after prefill (0: skip it)")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per GPU (default: the workload's own batch; smaller for profiler captures)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- distributed
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        import torch.distributed as dist
        if self.world > 1 and not dist.is_initialized():
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
            self.pg = True

    def barrier(self, device=None):
        if self.pg:
            import torch.distributed as dist
            if device is not None and device.type == "cuda":
                dist.barrier(device_ids=[device.index])
            else:
                dist.barrier()

    def max(self, x: float, device) -> float:
        if not self.pg:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def shard_seed_offset(rank: int) -> int:
    """Each rank draws its own batch: seeds shift by 1000 per rank."""
    return 1000 * rank


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.idx = gpu_index
        self.period = period_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.period)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(2 * self.period / 1000.0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[5], parts[6:10]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
        use = inside if inside else sorted(rows, key=lambda r: abs(r[0] - (t0 + t1) / 2))[:3]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[4]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "samples_in_window": len(inside)}


# DRAM bytes per launch of the dominant kernel from an ncu capture of the same
# kernel build, keyed by (kernel, attention variant, workload, budget, B): the
# capture ran at B = 8 and is scaled x4 by sequences to the B = 32 launch. An entry
# is removed whenever its kernel changes, and the line then reports null.
NCU_TRAFFIC = {
    # warp-specialised kernel, B = 8 capture (15,382,272 B read, 0 written) x 4
    ("kv_sparse_decode_attn", "default", "llama", 0.01, 32): 4 * 15_382_272,
}


CALIB_POSITIONS = 512  # calibration query positions for the stored descriptor's basis


def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- byte model
def attention_bytes(wl, n_kept, seq_lens):
    """Algorithmic bytes of one kv_sparse_decode_attn launch (block mode + proxy):
    the kept blocks' K and V rows, the kept blocks' key/value sums and counts, the
    totals, the index lists, q in and out/lse out."""
    import numpy as np
    L, D, G = wl.block_size, wl.D, wl.G
    es = 2 if str(wl.dtype).endswith("bfloat16") else 4
    nk = n_kept.cpu().numpy()
    total = 0
    for b in range(wl.B):
        n = seq_lens[b]
        for h in range(wl.Hkv):
            k = int(nk[b, h])
            # all kept blocks are full except possibly the last block of the sequence
            toks = min(k * L, n) if k else 0
            total += toks * D * es * 2                  # K and V rows
            total += k * (D * 4 * 2 + 4 + 4)            # kept k_sum, v_sum rows, counts, indices
            total += 2 * D * 4 + 4 + 4                  # totals, n_kept, seq_len
            total += G * D * es + G * D * 4 + G * 4     # q in, out and lse out
    return total


def select_bytes(wl, seq_lens, kmax=None):
    """Algorithmic bytes of one summary-mode selection launch: every valid block's
    key summary row (fp32 sum, or bf16 mean with the bf16-mean scorer) and count,
    q, and the kept indices written."""
    L, D, G = wl.block_size, wl.D, wl.G
    es = 2 if str(wl.dtype).endswith("bfloat16") else 4
    row = D * 2 if wl.score_mode == "summary_mean16" else D * 4
    kmax = wl.kmax if kmax is None else kmax
    total = 0
    for b in range(wl.B):
        nbv = (seq_lens[b] + L - 1) // L
        total += wl.Hkv * (nbv * (row + 4) + G * D * es + kmax * 4 + 4)
    return total


def quest_select_bytes(wl, seq_lens):
    """Algorithmic bytes of one kv_select_blocks_quest launch: every valid block's
    bf16 (min, max) key bounds, q, and the kept indices written."""
    L, D, G = wl.block_size, wl.D, wl.G
    total = 0
    for b in range(wl.B):
        nbv = (seq_lens[b] + L - 1) // L
        total += wl.Hkv * (nbv * D * 4 + G * D * 2 + wl.kmax * 4 + 4)
    return total


def cobs_select_bytes(wl, seq_lens, rank=4):
    """Algorithmic bytes of one kv_select_blocks_cobs launch: every valid block's
    fp32 key sum, count and rank fp32 covariance factors, q, and the kept indices."""
    L, D, G = wl.block_size, wl.D, wl.G
    total = 0
    for b in range(wl.B):
        nbv = (seq_lens[b] + L - 1) // L
        total += wl.Hkv * (nbv * (D * 4 + 4 + rank * D * 4) + G * D * 2 + wl.kmax * 4 + 4)
    return total


def cobs_fp4_select_bytes(wl, seq_lens, s_dim, rank=4):
    """Algorithmic bytes of one kv_select_blocks_cobs_fp4 launch: every valid block's
    bf16 mean, count, rank E2M1 factors of SP / 2 bytes and rank fp32 scales, q, the
    kept indices, and the query basis (Hkv x s x D fp32, counted once: every
    sequence's CTA of a KV head reads the same rows)."""
    L, D, G = wl.block_size, wl.D, wl.G
    SP = (s_dim + 31) // 32 * 32
    total = wl.Hkv * s_dim * D * 4
    for b in range(wl.B):
        nbv = (seq_lens[b] + L - 1) // L
        total += wl.Hkv * (nbv * (D * 2 + 4 + rank * (SP // 2) + rank * 4) + G * D * 2 + wl.kmax * 4 + 4)
    return total


QGC_C, QGC_ITERS = 32, 8  # clusters per (sequence, KV head), Lloyd iterations


def qgc_step_bytes(wl, n_read, budget):
    """Algorithmic bytes of one QGC decode step, (selection, attention + merge): the
    selection scans every token's bf16 projection (32 B) and member index, writes and
    reads back its score, reads the cluster mean and variance tokens and the read rows
    (keys and values, for the proxies), and writes the read list and the proxies; the
    attention reads the read rows, q, and writes out / lse; the merge reads the proxies
    and q and rewrites out / lse."""
    D, G, C = wl.D, wl.G, QGC_C
    es = 2 if str(wl.dtype).endswith("bfloat16") else 4
    nr = n_read.cpu().tolist()
    max_read = max(1, int(math.floor(budget * wl.Ncap)))
    sel = att = 0
    for b in range(wl.B):
        n = wl.seq_lens[b]
        for h in range(wl.Hkv):
            r = int(nr[b][h])
            sel += n * (32 + 4 + 8) + C * (3 * D * 4 + 8) + r * D * es * 2 + C * (2 * D * 4 + 4) + max_read * 8 \
                + G * D * es + 4
            att += r * (D * es * 2 + 8) + G * D * es + G * (D + 1) * 4 \
                + C * (2 * D * 4 + 4) + G * D * es + 2 * G * (D + 1) * 4
    return sel, att


def osa_select_bytes(wl, seq_lens):
    es = 2 if str(wl.dtype).endswith("bfloat16") else 4
    return sum(wl.Hkv * (seq_lens[b] * wl.D * es + wl.G * wl.D * es) for b in range(wl.B))


def wildcat_bytes(wl, seq_lens, n_sel):
    """Algorithmic bytes of kv_build_wildcat_coreset: per (sequence, KV head) with n
    tokens and T pivots, one read of the keys for the shift, then per step t the n
    keys, t factor rows read and one written (n fp32 each) and the residual diagonal
    read and written."""
    kb = wl.K.element_size()
    total = 0
    ns = n_sel.cpu().tolist()
    for b, n in enumerate(seq_lens):
        for h in range(wl.Hkv):
            T = int(ns[b][h])
            total += n * wl.D * kb + T * n * (wl.D * kb + 12) + 4 * n * T * (T - 1) // 2
    return total


def weighted_bytes(wl):
    es = 2 if str(wl.dtype).endswith("bfloat16") else 4
    return wl.B * wl.Hkv * (wl.m * (wl.D * es * 2 + 8) + wl.G * wl.D * (es + 4) + wl.G * 4)


# ----------------------------------------------------------------- CPU oracle
def _oracle_task(args):
    """One (sequence, KV head) decode step with the float64 oracle. Returns the
    kept blocks and near-tie flag (block modes), plus the kept set at the other
    budgets asked for and, for bf16-mean scoring, the exact-mean kept set."""
    import numpy as np
    from oracle import oracle as O
    kind, q16, K16, V16, n, L, scale, k_top, ff, fl, extra = args[:11]
    more_k = args[11] if len(args) > 11 else ()

    def f64(a):
        if a.dtype == np.uint16:
            return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        return a.astype(np.float64)

    q, K, V = f64(q16)[None], f64(K16)[None, None], f64(V16)[None, None]
    if kind == "weighted":
        O.weighted_batch(q, K, V, [n], extra[0][None, None], extra[1][None, None], scale)
        return None
    if kind == "dense":
        O.dense_batch(q, K, V, [n], scale)
        return None
    if kind == "qgc":
        P_o, C_o, it_o, budget_o = extra
        r = O.qgc_decode_one(q[0], K[0, 0], V[0, 0], n, P_o, C_o, it_o, budget_o, scale)
        return {"kept": r["read"], "near_tie": r["near_tie"], "more": {}}
    if kind == "cobs_fp4":
        # the oracle's own stored descriptor of this pair: factors within its basis
        # (stored at fp32), rounded to fp32 and E2M1-coded with float32 decisions
        U_pad, s_dim, rank = extra
        SP = U_pad.shape[0]
        NBc = (K.shape[2] + L - 1) // L
        xo, _ = O.block_cov_factors_ss_one(K[0, 0], n, L, NBc, rank, U_pad[:s_dim])
        dec = np.zeros((NBc, rank, SP))
        x32 = np.zeros((NBc, rank, SP), dtype=np.float32)
        x32[:, :, :s_dim] = xo.astype(np.float32)
        for blk in range(NBc):
            for i in range(rank):
                c, sc = O.fp4_e2m1_quantize(x32[blk, i])
                dec[blk, i] = O.fp4_e2m1_decode(c, sc)
        sel = O.select_batch(q, K, [n], L, scale, k_top, ff, fl, "cobs_stored", rank=rank, stored_xi={(0, 0): dec},
                             stored_U=U_pad[None])
        s = sel[(0, 0)]
        O.sparse_batch(q, K, V, [n], L, scale, {(0, 0): s["kept"]}, True)
        nb = (n + L - 1) // L
        return {"kept": s["kept"], "near_tie": s["near_tie"],
                "more": {k: O.select_blocks(s["S"], nb, k, ff, fl) for k in more_k}}
    sel, _, _ = O.decode_step(q, K, V, [n], L, scale, k_top, ff, fl, score_mode=kind, use_proxy=True)
    s = sel[(0, 0)]
    nb = (n + L - 1) // L
    res = {"kept": s["kept"], "near_tie": s["near_tie"],
           "more": {k: O.select_blocks(s["S"], nb, k, ff, fl) for k in more_k}}
    res["more"] = {k: {"kept": v["kept"], "near_tie": v["near_tie"]} for k, v in res["more"].items()}
    if kind == "summary_mean16":
        ex = O.select_batch(q, K, [n], L, scale, k_top, ff, fl, "summary")[(0, 0)]
        res["exact_mean_kept"] = ex["kept"]
    return res


def _pool_init():
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
    os.environ.setdefault("MKL_NUM_THREADS", "1")


def oracle_tasks(wl, pairs, more_k=()):
    import numpy as np
    import torch
    from weighted_coreset_softmax_b200 import workloads as W
    tasks = []
    kind = {"summary": "summary", "summary_mean16": "summary_mean16", "exact_mass": "exact_mass", "quest": "quest",
            "cobs": "cobs", "cobs_fp4": "cobs_fp4", "qgc": "qgc"}[wl.score_mode]
    if kind == "qgc" and not hasattr(wl, "oracle_qgc_basis"):
        # the oracle's projection rows: its own top-16 query eigenvectors, stored at fp32
        from oracle import oracle as O
        Qc = W.calibration_queries(wl, CALIB_POSITIONS).to(torch.float64).cpu().numpy()
        _, vec = O.query_basis(Qc, wl.Hkv)
        wl.oracle_qgc_basis = vec[:, :16, :].astype(np.float32).astype(np.float64)
    if kind == "cobs_fp4" and not hasattr(wl, "oracle_basis"):
        # the oracle's basis and s from the calibration queries, stored at fp32
        from oracle import oracle as O
        Qc = W.calibration_queries(wl, CALIB_POSITIONS).to(torch.float64).cpu().numpy()
        ev, vec = O.query_basis(Qc, wl.Hkv)
        s_o, _ = O.subspace_rank(ev, 0.9)
        SP = (s_o + 31) // 32 * 32
        U_pad = np.zeros((wl.Hkv, SP, wl.D))
        U_pad[:, :s_o] = vec[:, :s_o, :].astype(np.float32).astype(np.float64)
        wl.oracle_basis = (U_pad, s_o)
    if wl.attn_mode == "weighted":
        kind = "weighted"
    for (b, h) in pairs:
        def raw(t):
            t = t.detach().cpu()
            return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()
        q = raw(wl.q[b, h * wl.G:(h + 1) * wl.G])
        K = raw(wl.K[b, h])
        V = raw(wl.V[b, h])
        extra = None
        if kind == "weighted":
            extra = (wl.tok_idx[b, h].cpu().numpy(), wl.w[b, h].cpu().numpy().astype(np.float64))
        if kind == "cobs_fp4":
            extra = (wl.oracle_basis[0][h], wl.oracle_basis[1], 4)
        if kind == "qgc":
            extra = (wl.oracle_qgc_basis[h], QGC_C, QGC_ITERS, wl.qgc_budget)
        tasks.append((kind, q, K, V, wl.seq_lens[b], wl.block_size, wl.scale, wl.k_top,
                      bool(wl.force_first), bool(wl.force_last), extra, tuple(more_k)))
    return tasks


def time_oracle(wl, n_pairs_target, workers, warm_pairs=1, more_k=()):
    """Wall time of the oracle over n pairs (sequence, KV head) on a spawn pool;
    also returns each distinct pair's oracle result."""
    pairs_all = [(b, h) for b in range(wl.B) for h in range(wl.Hkv)]
    n = max(1, n_pairs_target)
    pairs = [pairs_all[i % len(pairs_all)] for i in range(n)]
    uniq = sorted(set(pairs))
    tmap = dict(zip(uniq, oracle_tasks(wl, uniq, more_k)))
    tasks = [tmap[p] for p in pairs]
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers, initializer=_pool_init) as pool:
        pool.map(_oracle_task, tasks[:max(1, min(warm_pairs, len(tasks)))] * 1)
        t0 = time.perf_counter()
        outs = pool.map(_oracle_task, tasks, chunksize=1)
        dt = time.perf_counter() - t0
    results = {}
    for pr, o in zip(pairs, outs):
        results.setdefault(pr, o)
    return dt, n, results


def cpu_baseline(wl, seconds, label_sample, more_k=()):
    """Oracle throughput on the host cores over a bounded sample of the workload;
    also returns the oracle's per-pair results (kept blocks) for the sample."""
    workers = max(1, min(os.cpu_count() or 1, 32))
    # calibrate with one pair in-process, single-threaded BLAS
    _pool_init()
    t0 = time.perf_counter()
    _oracle_task(oracle_tasks(wl, [(0, 0)])[0])
    t1 = time.perf_counter() - t0
    n = int(max(1, min(wl.B * wl.Hkv * 4, seconds * workers / max(t1, 1e-3))))
    n = max(workers, n) if n >= workers else n
    dt, n, results = time_oracle(wl, n, workers, more_k=more_k)
    queries = n / wl.Hkv
    return {"value": queries / dt, "unit": "queries/s", "cores": workers, "kind": "oracle",
            "sample": f"{n} (sequence, KV head) decode steps = {queries:g} queries of {label_sample}; "
                      f"float64 NumPy oracle (select + attend), {workers} spawn workers, 1 BLAS thread each",
            "seconds": dt}, results


def selection_check(wl, oracle_res, idx, nk, idx5=None, nk5=None, more_k=()):
    """Kept blocks of batch 0 on the GPU against the oracle's on the pairs the CPU
    baseline sample covered: exact matches, mismatches at flagged near ties
    (allowed, reported) and any other mismatch; for the bf16-mean scorer also how
    many kept sets differ from the exact-mean (float64) ranking."""
    gi, gn = idx.cpu().numpy(), nk.cpu().numpy()
    out = {"pairs": 0, "exact": 0, "near_tie_flagged": 0, "near_tie_mismatch": 0, "other_mismatch": 0}
    if wl.score_mode == "summary_mean16":
        out["differ_from_exact_mean_ranking"] = 0
    out5 = None
    if idx5 is not None and more_k:
        g5i, g5n = idx5.cpu().numpy(), nk5.cpu().numpy()
        out5 = {"pairs": 0, "exact": 0, "near_tie_flagged": 0, "near_tie_mismatch": 0, "other_mismatch": 0}
    for (b, h), r in sorted(oracle_res.items()):
        if r is None:
            continue
        got = [int(x) for x in gi[b, h, :gn[b, h]]]
        out["pairs"] += 1
        out["near_tie_flagged"] += int(r["near_tie"])
        if got == r["kept"]:
            out["exact"] += 1
        elif r["near_tie"]:
            out["near_tie_mismatch"] += 1
        else:
            out["other_mismatch"] += 1
        if "exact_mean_kept" in r and "differ_from_exact_mean_ranking" in out:
            out["differ_from_exact_mean_ranking"] += int(got != r["exact_mean_kept"])
        if out5 is not None and more_k[0] in r["more"]:
            r5 = r["more"][more_k[0]]
            got5 = [int(x) for x in g5i[b, h, :g5n[b, h]]]
            out5["pairs"] += 1
            out5["near_tie_flagged"] += int(r5["near_tie"])
            if got5 == r5["kept"]:
                out5["exact"] += 1
            elif r5["near_tie"]:
                out5["near_tie_mismatch"] += 1
            else:
                out5["other_mismatch"] += 1
    ranking = {"summary_mean16": "bf16-mean ranking",
               "cobs_fp4": "stored-descriptor ranking (the oracle's own basis, factors and E2M1 codes)",
               "qgc": "read tokens of the oracle's own clusters, error split and in-cluster scores"}
    out["reference"] = ("float64 oracle, " + ranking.get(wl.score_mode, "exact-mean ranking")
                        + ", pairs of the CPU baseline sample")
    if out5 is not None:
        out["budget_5pct"] = out5
    return out


# ----------------------------------------------------------------- our arm
def workload_label(wl, budget):
    names = {
        "llama": "Llama-3.1-8B-shaped GQA decode",
        "llama_b1": "Llama-3.1-8B-shaped GQA decode, batch 1 (latency)",
        "qwen_long": "Qwen2.5-7B-shaped long-context GQA decode",
        "llama_osa": "Llama-3.1-8B-shaped GQA decode, OSA exact-mass selection",
        "llama_quest": "Llama-3.1-8B-shaped GQA decode, Quest key-box selection",
        "llama_cobs": "Llama-3.1-8B-shaped GQA decode, COBS second-order selection (rank-4 factors)",
        "llama_cobs_fp4": "Llama-3.1-8B-shaped GQA decode, COBS stored descriptor (bf16 means, rank-4 E2M1 "
                          "factors in the 90%-energy query subspace)",
        "llama_coreset": "Llama-3.1-8B-shaped GQA decode, weighted coreset m=2048",
        "llama_qgc": f"Llama-3.1-8B-shaped GQA decode, query-guided clusters (C={QGC_C}) with error-gated reads",
    }
    if wl.attn_mode == "qgc":
        return (f"{names[wl.name]}: B={wl.B}, {wl.Hq} q heads / {wl.Hkv} KV heads, d={wl.D}, ctx={wl.Ncap}, "
                f"read budget {budget:g} (exact tokens plus 1.5 rows a cluster, one proxy a cluster)")
    return (f"{names[wl.name]}: B={wl.B}, {wl.Hq} q heads / {wl.Hkv} KV heads, d={wl.D}, "
            f"ctx={wl.Ncap}, block={wl.block_size}, read budget {budget:g} "
            f"(top-{wl.k_top} + first + last + tail proxy)" if wl.attn_mode != "weighted" else
            f"{names[wl.name]}: B={wl.B}, ctx={wl.Ncap}, m={wl.m} weighted tokens per KV head")


def run_ours(args, dist):
    if args.attn:
        os.environ["KVSPARSE_ATTN"] = args.attn  # read once, when the library first runs attention
    import torch
    import weighted_coreset_softmax_b200 as kv
    from weighted_coreset_softmax_b200 import workloads as W

    dev = torch.device("cuda", dist.local_rank if torch.cuda.device_count() > dist.local_rank else 0)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    kv.lib()

    name = args.workload
    base_seed = {"llama": 100, "llama_b1": 1, "qwen_long": 2}.get(name, 3) + shard_seed_offset(dist.rank)
    score_override = "summary_mean16" if args.scorer == "mean16" else None
    L2_BYTES = 126 << 20

    shared_basis = {}

    def make_set(j):
        seed = (None if dist.rank == 0 else base_seed) if j == 0 else base_seed + 50000 * j
        w_ = W.make(name, dev, budget=args.budget, B=args.batch, seed=seed)
        if score_override and w_.score_mode == "summary":
            w_.score_mode = score_override
        sl_ = w_.seq_lens_tensor(dev)
        su_ = kv.kv_build_block_summaries(w_.K, w_.V, sl_, w_.block_size)
        if w_.score_mode == "summary_mean16":
            su_["k_mean"] = kv.kv_build_block_key_means(w_.K, sl_, w_.block_size, su_["k_sum"], su_["counts"])
        if w_.score_mode == "quest":
            su_["k_bounds"] = kv.kv_build_block_bounds(w_.K, sl_, w_.block_size)
        if w_.score_mode == "cobs":
            su_["k_xi"] = kv.kv_build_block_cov_factors(w_.K, sl_, w_.block_size, 4)
        if w_.score_mode == "qgc":
            if "P" not in shared_basis:  # the model's projection rows, from calibration queries
                Qc = W.calibration_queries(w_, CALIB_POSITIONS)
                evecs, _ = kv.kv_build_query_basis(Qc, w_.Hkv)
                shared_basis.update(P=evecs[:, :16, :].contiguous(), Qc=Qc)
            su_["qgc"] = kv.kv_build_qgc(w_.K, w_.V, sl_, shared_basis["P"], QGC_C, QGC_ITERS)
            mr = max(1, int(math.floor(args.budget * w_.Ncap)))
            su_["qsel"] = (torch.zeros(w_.B, w_.Hkv, mr, dtype=torch.int32, device=dev),
                           torch.zeros(w_.B, w_.Hkv, mr, dtype=torch.float32, device=dev),
                           torch.zeros(w_.B, w_.Hkv, dtype=torch.int32, device=dev),
                           torch.zeros(w_.B, w_.Hkv, QGC_C, w_.D, dtype=torch.float32, device=dev),
                           torch.zeros(w_.B, w_.Hkv, QGC_C, w_.D, dtype=torch.float32, device=dev),
                           torch.zeros(w_.B, w_.Hkv, QGC_C, dtype=torch.int32, device=dev))
            su_["qws"] = torch.empty(w_.B * w_.Hkv * w_.Ncap * 4, dtype=torch.uint8, device=dev)
            w_.qgc_budget = args.budget
        if w_.score_mode == "cobs_fp4":
            if "U" not in shared_basis:  # one basis for the model: every batch draws queries from it
                Qc = W.calibration_queries(w_, CALIB_POSITIONS)
                evecs, evals = kv.kv_build_query_basis(Qc, w_.Hkv)
                s_q = kv.kv_query_subspace_rank(evals, 0.9)
                shared_basis.update(U=evecs[:, :s_q, :].contiguous(), s=s_q, Qc=Qc)
            su_["k_mean"] = kv.kv_build_block_key_means(w_.K, sl_, w_.block_size, su_["k_sum"], su_["counts"])
            xi_ss = kv.kv_build_block_cov_factors_ss(w_.K, sl_, w_.block_size, shared_basis["U"], 4)
            su_["codes"], su_["code_scales"] = kv.kv_quantize_fp4(xi_ss)
            del xi_ss
        return dict(wl=w_, sl=sl_, summ=su_,
                    idx=torch.zeros(w_.B, w_.Hkv, w_.kmax, dtype=torch.int32, device=dev),
                    nk=torch.zeros(w_.B, w_.Hkv, dtype=torch.int32, device=dev),
                    out=torch.empty(w_.B, w_.Hq, w_.D, dtype=torch.float32, device=dev),
                    lse=torch.empty(w_.B, w_.Hq, dtype=torch.float32, device=dev),
                    ws=kv.Workspace(kv.make_shape(w_.q, w_.K, sl_, w_.block_size), dev))

    # independent batches (own caches, summaries, queries) rotated through the timed
    # steps: enough that twice the L2 capacity of other data passes between two uses
    # of a batch
    sets = [make_set(0)]
    w0_ = sets[0]["wl"]
    es = 2 if str(w0_.dtype).endswith("bfloat16") else 4
    if w0_.attn_mode == "weighted":
        step_est = weighted_bytes(w0_)
    else:
        step_est = (osa_select_bytes(w0_, w0_.seq_lens) if w0_.score_mode == "exact_mass" else
                    select_bytes(w0_, w0_.seq_lens))
        step_est += w0_.B * w0_.Hkv * w0_.kmax * w0_.block_size * w0_.D * es * 2
    ROT = int(min(16, max(8, 1 + -(-2 * L2_BYTES // step_est)))) if args.rot is None else max(1, args.rot)
    sets += [make_set(j) for j in range(1, ROT)]
    s0 = sets[0]
    wl, sl, summ, idx, nk, out, lse, ws = (s0[k] for k in ("wl", "sl", "summ", "idx", "nk", "out", "lse", "ws"))
    B = wl.B
    quest = wl.score_mode == "quest"
    mode = kv.KV_SCORE_SUMMARY if wl.score_mode in ("summary", "summary_mean16") else kv.KV_SCORE_EXACT_MASS
    kmax = wl.kmax
    weighted = wl.attn_mode == "weighted"
    qgc = wl.attn_mode == "qgc"

    def su0_qsel():
        return s0["summ"]["qsel"]

    def select_on(st_, q_=None, k_top=None, kmax_=None, idx_=None, nk_=None):
        if weighted:
            return
        w_, sl_, su_ = st_["wl"], st_["sl"], st_["summ"]
        q_ = w_.q if q_ is None else q_
        if qgc:
            kv.kv_select_qgc(q_, w_.K, w_.V, sl_, w_.scale, shared_basis["P"], su_["qgc"], args.budget,
                             workspace=su_["qws"], out=su_["qsel"])
            return
        if k_top is not None:
            kv.kv_select_blocks_mean16(q_, w_.K, sl_, w_.block_size, w_.scale, su_["k_mean"], su_["counts"], k_top,
                                       w_.force_first, w_.force_last, kmax=kmax_, block_idx=idx_, n_kept=nk_) \
                if wl.score_mode == "summary_mean16" else \
                kv.kv_select_blocks(q_, w_.K, sl_, w_.block_size, w_.scale, su_["counts"], k_top, w_.force_first,
                                    w_.force_last, k_sum=su_["k_sum"], kmax=kmax_, block_idx=idx_, n_kept=nk_)
            return
        if wl.score_mode == "summary_mean16":
            kv.kv_select_blocks_mean16(q_, w_.K, sl_, w_.block_size, w_.scale, su_["k_mean"], su_["counts"], w_.k_top,
                                       w_.force_first, w_.force_last, kmax=kmax, block_idx=st_["idx"],
                                       n_kept=st_["nk"])
        elif wl.score_mode == "cobs_fp4":
            kv.kv_select_blocks_cobs_fp4(q_, w_.K, sl_, w_.block_size, w_.scale, su_["k_mean"], su_["counts"],
                                         shared_basis["U"], su_["codes"], su_["code_scales"], 4, w_.k_top,
                                         w_.force_first, w_.force_last, kmax=kmax, block_idx=st_["idx"],
                                         n_kept=st_["nk"])
        elif wl.score_mode == "cobs":
            kv.kv_select_blocks_cobs(q_, w_.K, sl_, w_.block_size, w_.scale, su_["k_sum"], su_["counts"], su_["k_xi"],
                                     w_.k_top, w_.force_first, w_.force_last, kmax=kmax, block_idx=st_["idx"],
                                     n_kept=st_["nk"])
        elif quest:
            kv.kv_select_blocks_quest(q_, w_.K, sl_, w_.block_size, w_.scale, su_["k_bounds"], w_.k_top,
                                      w_.force_first, w_.force_last, kmax=kmax, block_idx=st_["idx"],
                                      n_kept=st_["nk"])
        else:
            kv.kv_select_blocks(q_, w_.K, sl_, w_.block_size, w_.scale, su_["counts"], w_.k_top,
                                w_.force_first, w_.force_last, mode=mode, k_sum=su_["k_sum"], kmax=kmax,
                                block_idx=st_["idx"], n_kept=st_["nk"])

    def attend_on(st_, q_=None, idx_=None, nk_=None):
        w_, sl_, su_ = st_["wl"], st_["sl"], st_["summ"]
        q_ = w_.q if q_ is None else q_
        if idx_ is not None:
            kv.kv_sparse_decode_attn(q_, w_.K, w_.V, sl_, w_.block_size, w_.scale, st_["ws"], block_idx=idx_,
                                     n_kept=nk_, summaries=su_, use_tail_proxy=True, out=st_["out"], lse=st_["lse"])
            return
        if qgc:
            qs = su_["qsel"]
            kv.kv_sparse_decode_attn(q_, w_.K, w_.V, sl_, w_.block_size, w_.scale, st_["ws"],
                                     tok_idx=qs[0], w=qs[1], out=st_["out"], lse=st_["lse"])
            kv.kv_merge_qgc_proxies(q_, w_.K, sl_, w_.scale, QGC_C, qs[3], qs[4], qs[5], st_["out"], st_["lse"])
        elif weighted:
            kv.kv_sparse_decode_attn(q_, w_.K, w_.V, sl_, w_.block_size, w_.scale, st_["ws"],
                                     tok_idx=w_.tok_idx, w=w_.w, out=st_["out"], lse=st_["lse"])
        else:
            kv.kv_sparse_decode_attn(q_, w_.K, w_.V, sl_, w_.block_size, w_.scale, st_["ws"],
                                     block_idx=st_["idx"], n_kept=st_["nk"], summaries=su_,
                                     use_tail_proxy=True, out=st_["out"], lse=st_["lse"])

    def step_full(st_, q_=None):
        select_on(st_, q_)
        attend_on(st_, q_)

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # the once-after-prefill builds, timed on batch 0 (not part of the step)
    def time_build(fn, reps=3):
        fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    stream = torch.cuda.current_stream(dev)
    builds = {"kv_build_block_summaries_ms": time_build(
        lambda: kv.kv_build_block_summaries(wl.K, wl.V, sl, wl.block_size, out=summ))}
    if quest:
        builds["kv_build_block_bounds_ms"] = time_build(
            lambda: kv.kv_build_block_bounds(wl.K, sl, wl.block_size, out=summ["k_bounds"]))
    if wl.score_mode == "cobs":
        builds["kv_build_block_cov_factors_ms"] = time_build(
            lambda: kv.kv_build_block_cov_factors(wl.K, sl, wl.block_size, 4, out=summ["k_xi"]), reps=1)
    if qgc:
        builds["kv_build_qgc_ms"] = time_build(
            lambda: kv.kv_build_qgc(wl.K, wl.V, sl, shared_basis["P"], QGC_C, QGC_ITERS), reps=1)
        builds["qgc"] = {"clusters": QGC_C, "lloyd_iterations": QGC_ITERS}
    if wl.score_mode == "cobs_fp4":
        builds["kv_build_query_basis_ms"] = time_build(
            lambda: kv.kv_build_query_basis(shared_basis["Qc"], wl.Hkv), reps=1)
        xi_t = {}

        def ss_build():
            xi_t["x"] = kv.kv_build_block_cov_factors_ss(wl.K, sl, wl.block_size, shared_basis["U"], 4)
        builds["kv_build_block_cov_factors_ss_ms"] = time_build(ss_build, reps=1)
        builds["kv_quantize_fp4_ms"] = time_build(lambda: kv.kv_quantize_fp4(xi_t["x"]), reps=1)
        builds["subspace_s"] = shared_basis["s"]
        del xi_t

    if args.wildcat_m > 0:
        # the WildCat coreset producer on the same cache (randomly pivoted Cholesky
        # with kernel-distance weights, m pivots per (sequence, KV head))
        m_wc = min(args.wildcat_m, wl.Ncap)
        g_wc = torch.Generator(device=dev).manual_seed(4242 + shard_seed_offset(dist.rank))
        u_wc = torch.rand(wl.B, wl.Hkv, m_wc, generator=g_wc, device=dev).clamp_(1e-6, 1 - 1e-6)
        shp_wc = kv.KVShape(wl.B, wl.Hkv, wl.Hkv, wl.D, wl.Ncap, wl.block_size, kv._dtype_code(wl.K.dtype), sl.data_ptr())
        ws_wc = torch.empty(int(kv.lib().kv_wildcat_workspace_bytes(ctypes.byref(shp_wc), m_wc)),
                            dtype=torch.uint8, device=dev)
        out_wc = {}

        def wc_build():
            out_wc["r"] = kv.kv_build_wildcat_coreset(wl.K, sl, wl.scale, m_wc, u_wc, workspace=ws_wc)
        wc_ms = time_build(wc_build, reps=1)
        wc_b = wildcat_bytes(wl, wl.seq_lens, out_wc["r"][2])
        pk, pk_kind = measured_peak_hbm()
        builds["kv_build_wildcat_coreset"] = {
            "m": m_wc, "ms": wc_ms, "bytes": wc_b, "GB_s": wc_b / (wc_ms * 1e-3) / 1e9,
            "frac": wc_b / (wc_ms * 1e-3) / 1e9 / pk, "peak_kind": pk_kind,
            "pivots_min": int(out_wc["r"][2].min()) if out_wc["r"][2].numel() else 0}
        del ws_wc, out_wc

    def check_status(what):
        for st_ in sets:
            if kv.kv_workspace_status(st_["ws"].tensor) != 0:
                raise RuntimeError(f"device checks failed {what}")

    for i in range(max(3, args.warmup, ROT)):
        step_full(sets[i % ROT])
    torch.cuda.synchronize(dev)
    check_status("during warm-up")

    K_steps = args.steps
    # The timed region: K steps back to back on one stream, captured once in a
    # CUDA graph (so the host's per-call cost cannot stretch the device time) and
    # replayed between one event pair. A step is select + attention (each kernel
    # may be scheduled while the one before it finishes, and waits for it before
    # touching memory). Step i works on batch i mod ROT: a batch's inputs were last
    # touched ROT - 1 steps (at least twice the L2 capacity of other data) earlier,
    # as in a decode loop over distinct layers.
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    timed_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(timed_graph, stream=cap):
        for i in range(K_steps):
            step_full(sets[i % ROT])
    stream.wait_stream(cap)
    timed_graph.replay()  # warm the graph
    torch.cuda.synchronize(dev)
    check_status("in the captured steps")
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.1)
    dist.barrier(dev)
    torch.cuda.synchronize(dev)
    w0 = time.time()
    torch.cuda.nvtx.range_push("timed")  # lets a profiler restrict itself to the timed steps
    t_start.record(stream)
    timed_graph.replay()
    t_end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    del timed_graph

    # The secondary loops are issued eagerly behind a GPU sleep long enough for the
    # host to queue them all, so their events time the device, not the host.
    def host_ahead(n_launch):
        torch.cuda._sleep(int(min(4e9, 2.5e5 * n_launch)))  # about 125 us of SM clock per launch

    # each step alone: an event pair around every step, so steps do not overlap
    k_steps = min(K_steps, 100)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(k_steps)]
    host_ahead(2 * k_steps)
    for i in range(k_steps):
        ev[i][0].record(stream)
        step_full(sets[i % ROT])
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    # each kernel alone (an event pair around each launch, batches rotating): the
    # per-kernel durations of the roofline
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(k_steps)]
    host_ahead(2 * k_steps)
    for i in range(k_steps):
        st_ = sets[i % ROT]
        kev[i][0].record(stream)
        select_on(st_)
        kev[i][1].record(stream)
        kev[i][2].record(stream)
        attend_on(st_)
        kev[i][3].record(stream)
    torch.cuda.synchronize(dev)
    # the same step on one batch with a 512 MiB write flushing L2 before each step
    # (a stricter bound: it also evicts the kernels' code from L2)
    fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(k_steps)]
    host_ahead(3 * k_steps)
    for i in range(k_steps):
        flush.zero_()
        fev[i][0].record(stream)
        step_full(s0)
        fev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    w1 = time.time()
    dist.barrier(dev)
    clk = clocks.stop(w0, w1)
    step_ms_local = t_start.elapsed_time(t_end) / K_steps
    step_ms = dist.max(step_ms_local, dev)
    isolated_ms = dist.max(statistics.fmean(e[0].elapsed_time(e[1]) for e in ev), dev)
    flushed_ms = dist.max(statistics.fmean(e[0].elapsed_time(e[1]) for e in fev), dev)
    sel_avg = statistics.fmean(e[0].elapsed_time(e[1]) for e in kev) if not weighted else 0.0
    att_avg = statistics.fmean(e[2].elapsed_time(e[3]) for e in kev)

    # End to end through the public API: every step's q comes in from pinned host
    # memory and its out/lse go back, inside the timed region. The step's copies
    # run on two copy streams and overlap the neighbouring steps' kernels, as a
    # serving loop would; the ROT independent batches rotate, so a step never
    # finds its inputs in L2 (no flush needed).
    e2e_ms = None
    h2d_bytes = wl.q.numel() * wl.q.element_size()
    d2h_bytes = out.numel() * 4 + lse.numel() * 4
    if not args.no_e2e:
        for st_ in sets:
            st_["q_dev"] = torch.empty_like(st_["wl"].q)
            st_["q_host"] = st_["wl"].q.detach().cpu().pin_memory()
            st_["out_host"] = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
            st_["lse_host"] = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
            for e in ("ev_in", "ev_comp", "ev_out"):
                st_[e] = torch.cuda.Event()

        def step_on(st_):
            step_full(st_, st_["q_dev"])

        s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def enqueue(n):
            # n steps over the rotating batches; a wait only on events recorded here
            seen = set()
            for i in range(n):
                st_ = sets[i % ROT]
                key = i % ROT
                with torch.cuda.stream(s_in):
                    if (key, "comp") in seen:
                        s_in.wait_event(st_["ev_comp"])  # the step before on this batch has read q_dev
                    st_["q_dev"].copy_(st_["q_host"], non_blocking=True)
                    st_["ev_in"].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(st_["ev_in"])
                    if (key, "out") in seen:
                        s_comp.wait_event(st_["ev_out"])  # out of the step before on this batch is back
                    step_on(st_)
                    st_["ev_comp"].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(st_["ev_comp"])
                    st_["out_host"].copy_(st_["out"], non_blocking=True)
                    st_["lse_host"].copy_(st_["lse"], non_blocking=True)
                    st_["ev_out"].record(s_out)
                seen.update({(key, "comp"), (key, "out")})

        # the steps are captured once in a CUDA graph (24 steps, three streams forked
        # from the capture stream and joined at its end) and replayed: the host
        # issues one launch per 24 steps instead of a dozen calls per step
        NG = 24
        cap = torch.cuda.Stream(dev)
        for _ in range(2):  # eager warm-up on the same streams
            cap.wait_stream(torch.cuda.current_stream(dev))
            for s_ in (s_in, s_comp, s_out):
                s_.wait_stream(cap)
            enqueue(ROT)
            for s_ in (s_in, s_comp, s_out):
                cap.wait_stream(s_)
            torch.cuda.current_stream(dev).wait_stream(cap)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            for s_ in (s_in, s_comp, s_out):
                s_.wait_stream(cap)
            enqueue(NG)
            for s_ in (s_in, s_comp, s_out):
                cap.wait_stream(s_)
        torch.cuda.synchronize(dev)
        reps = max(1, -(-K_steps // NG))
        graph.replay()
        torch.cuda.synchronize(dev)
        dist.barrier(dev)
        torch.cuda.synchronize(dev)
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        rs = torch.cuda.current_stream(dev)
        e_start.record(rs)
        for _ in range(reps):
            graph.replay()
        e_end.record(rs)
        torch.cuda.synchronize(dev)
        dist.barrier(dev)
        e2e_ms = dist.max(e_start.elapsed_time(e_end) / (reps * NG), dev)
        del graph
        check_status("in the end-to-end steps")

    # the dense baseline on the identical cache
    dense = None
    if not args.no_dense and not weighted:
        dws = ws
        dout = torch.empty_like(out)
        dl = torch.empty_like(lse)
        for _ in range(2):
            kv.kv_dense_decode_attn(wl.q, wl.K, wl.V, sl, wl.block_size, wl.scale, dws, out=dout, lse=dl)
        dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(10)]
        for i in range(10):
            flush.zero_()
            dev_ev[i][0].record(stream)
            kv.kv_dense_decode_attn(wl.q, wl.K, wl.V, sl, wl.block_size, wl.scale, dws, out=dout, lse=dl)
            dev_ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        d_ms = statistics.fmean(e[0].elapsed_time(e[1]) for e in dev_ev)
        dbytes = sum(wl.Hkv * wl.seq_lens[b] * wl.D * 2 * 2 for b in range(B))
        dense = {"ms": d_ms, "GB_s": dbytes / (d_ms * 1e-3) / 1e9, "bytes": dbytes,
                 "speedup_attn_kernel": d_ms / att_avg, "speedup_step": d_ms / step_ms_local}

    # secondary figures on the same batches: each kernel back to back (a graph of
    # launches over the rotating batches: a decode loop's steady state), the 5%
    # read budget, and a plain streaming read of the same byte counts (the time one
    # launch needs just to move those bytes, launch and ramp included)
    def graph_avg_ms(fn, n):
        capst = torch.cuda.Stream(dev)
        capst.wait_stream(stream)
        g_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_, stream=capst):
            for i in range(n):
                fn(i)
        stream.wait_stream(capst)
        g_.replay()
        torch.cuda.synchronize(dev)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        g_.replay()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        del g_
        return a_.elapsed_time(b_) / n

    def alone_avg_ms(fn, n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        host_ahead(n)
        for i in range(n):
            evs[i][0].record(stream)
            fn(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        return statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)

    secondary = {}
    if not args.no_secondary:
        secondary["kernels_ms_back_to_back"] = {
            "kv_sparse_decode_attn": graph_avg_ms(lambda i: attend_on(sets[i % ROT]), k_steps)}
        if not weighted:
            secondary["kernels_ms_back_to_back"]["kv_select_blocks"] = graph_avg_ms(
                lambda i: select_on(sets[i % ROT]), k_steps)
        sink = torch.zeros(1, dtype=torch.int32, device=dev)
        a_b = (qgc_step_bytes(wl, su0_qsel()[2], args.budget)[1] if qgc else
               attention_bytes(wl, nk, wl.seq_lens) if not weighted else weighted_bytes(wl))
        floor = {"attn_bytes_alone_ms": alone_avg_ms(
            lambda i: kv.kv_stream_read(sets[i % ROT]["wl"].K, a_b & ~15, sink), k_steps),
                 "attn_bytes_back_to_back_ms": graph_avg_ms(
            lambda i: kv.kv_stream_read(sets[i % ROT]["wl"].K, a_b & ~15, sink), k_steps)}
        if not weighted:
            s_b = select_bytes(wl, wl.seq_lens) if wl.score_mode in ("summary", "summary_mean16") else None
            if s_b:
                floor["select_bytes_alone_ms"] = alone_avg_ms(
                    lambda i: kv.kv_stream_read(sets[i % ROT]["wl"].K, s_b & ~15, sink), k_steps)
        secondary["read_floor"] = floor
        if not weighted and wl.score_mode in ("summary", "summary_mean16") and abs(args.budget - 0.01) < 1e-9:
            NBv = wl.NBcap
            k5 = max(1, int(math.floor(0.05 * NBv)))
            kmax5 = min(NBv, k5 + int(bool(wl.force_first)) + int(bool(wl.force_last)))
            for st_ in sets:
                st_["idx5"] = torch.zeros(st_["wl"].B, st_["wl"].Hkv, kmax5, dtype=torch.int32, device=dev)
                st_["nk5"] = torch.zeros(st_["wl"].B, st_["wl"].Hkv, dtype=torch.int32, device=dev)

            def step5(i):
                st_ = sets[i % ROT]
                select_on(st_, k_top=k5, kmax_=kmax5, idx_=st_["idx5"], nk_=st_["nk5"])
                attend_on(st_, idx_=st_["idx5"], nk_=st_["nk5"])
            for i in range(ROT):
                step5(i)
            torch.cuda.synchronize(dev)
            step5_ms = graph_avg_ms(step5, k_steps)
            att5 = alone_avg_ms(lambda i: attend_on(sets[i % ROT], idx_=sets[i % ROT]["idx5"],
                                                    nk_=sets[i % ROT]["nk5"]), k_steps)
            sel5 = alone_avg_ms(lambda i: select_on(sets[i % ROT], k_top=k5, kmax_=kmax5, idx_=sets[i % ROT]["idx5"],
                                                    nk_=sets[i % ROT]["nk5"]), k_steps)
            a5 = attention_bytes(wl, s0["nk5"], wl.seq_lens)
            secondary["budget_5pct"] = {
                "k_top": k5, "kmax": kmax5, "ms_per_step": step5_ms, "queries_per_s": B / (step5_ms * 1e-3),
                "kernels_ms": {"kv_select_blocks": sel5, "kv_sparse_decode_attn": att5},
                "attn_bytes_per_launch": a5, "attn_GB_s": a5 / (att5 * 1e-3) / 1e9,
                "dense_over_sparse_attn_kernel": (dense["ms"] / att5) if dense else None,
                "dense_over_sparse_step": (dense["ms"] / step5_ms) if dense else None}
        check_status("in the secondary measurements")

    torch.cuda.synchronize(dev)
    check_status("during timing")

    # algorithmic bytes and the roofline of the dominant kernel
    if weighted:
        a_bytes, s_bytes = weighted_bytes(wl), 0
    elif qgc:
        s_bytes, a_bytes = qgc_step_bytes(wl, su0_qsel()[2], args.budget)
    else:
        a_bytes = attention_bytes(wl, nk, wl.seq_lens)
        s_bytes = (quest_select_bytes(wl, wl.seq_lens) if quest else
                   cobs_select_bytes(wl, wl.seq_lens) if wl.score_mode == "cobs" else
                   cobs_fp4_select_bytes(wl, wl.seq_lens, shared_basis["s"]) if wl.score_mode == "cobs_fp4" else
                   select_bytes(wl, wl.seq_lens) if mode == kv.KV_SCORE_SUMMARY else osa_select_bytes(wl, wl.seq_lens))
    peak, peak_kind = measured_peak_hbm()
    # the roofline line is the attention kernel's (the kernel the target names);
    # the selector's figures sit beside it
    dom, dom_bytes, dom_ms = "kv_sparse_decode_attn", a_bytes, att_avg
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    sel_roof = None
    if not weighted and sel_avg > 0:
        sel_ach = s_bytes / (sel_avg * 1e-3) / 1e9
        sel_roof = {"kernel": "kv_select_blocks", "achieved": sel_ach, "peak": peak, "unit": "GB/s",
                    "frac": sel_ach / peak, "pct_of_8TBs": 100.0 * sel_ach / NOMINAL_HBM_GBS}
    step_gbs = (a_bytes + s_bytes) / (step_ms_local * 1e-3) / 1e9

    queries = B * dist.world
    res = {
        "metric": METRIC,
        "value": queries / (step_ms * 1e-3),
        "unit": "queries/s",
        "n_gpus": dist.world,
        "steps": K_steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "ms_per_step_isolated": isolated_ms,
        "ms_per_step_l2_flushed": flushed_ms,
        "value_l2_flushed": queries / (flushed_ms * 1e-3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded bf16 caches shaped like the pages' workloads)",
        "config": {
            "workload": workload_label(wl, args.budget),
            "B_per_gpu": B, "Hq": wl.Hq, "Hkv": wl.Hkv, "D": wl.D, "ctx": wl.Ncap,
            "block": wl.block_size, "k_top": wl.k_top, "kmax": kmax, "kv_dtype": "bf16", "accumulate": "fp32",
            "selection": {"summary_mean16": "bf16 block means (kv_select_blocks_mean16)",
                          "summary": "fp32 block sums (kv_select_blocks)"}.get(wl.score_mode, wl.score_mode),
            "attention_kernel": os.environ.get("KVSPARSE_ATTN", "library default"),
            "parallelism": f"replicas: batch-sharded, {dist.world} rank(s), no collective",
            "l2": "one batch and no flush (--rot 1, a profiling run: the timed steps may hit L2)" if ROT == 1 else
                  f"inputs larger than L2: {ROT} independent batches (own caches, summaries, queries) rotate, "
                  f"so {ROT - 1} steps' data (about {(ROT - 1) * step_est / 1e6:.0f} MB) pass between two uses of "
                  f"a batch; no flush. "
                  f"ms_per_step: K steps back to back (one CUDA graph) in one event pair; ms_per_step_isolated: an event "
                  f"pair around each step; ms_per_step_l2_flushed: the step on one batch after a 512 MiB "
                  f"L2-flushing write",
            "step": ("kv_select_qgc + kv_sparse_decode_attn (weighted, the read tokens) + kv_merge_qgc_proxies "
                     "(kernels_ms.kv_sparse_decode_attn covers the last two)") if qgc else
                    "kv_select_blocks + kv_sparse_decode_attn" if not weighted else "kv_sparse_decode_attn",
        },
        "achieved_step_GB_s": step_gbs,
        "achieved_step_pct_of_8TBs": 100.0 * step_gbs / NOMINAL_HBM_GBS,
        "kernels_ms": {"kv_select_blocks": sel_avg, "kv_sparse_decode_attn": att_avg},
        "bytes_per_launch": {"kv_select_blocks": s_bytes, "kv_sparse_decode_attn": a_bytes},
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": NCU_TRAFFIC.get((dom, os.environ.get("KVSPARSE_ATTN", "default"), args.workload,
                                                 args.budget, B)),
                     "traffic_how": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the current "
                                    "kernel on a B = 8 capture of this workload, scaled x4 by the pairs processed "
                                    "(null for shapes without a capture)",
                     "timing": "event pair around each launch, batches rotating (the kernel alone)",
                     "pct_of_8TBs": 100.0 * achieved / NOMINAL_HBM_GBS},
        "roofline_select": sel_roof,
        "e2e": None if e2e_ms is None else {
            "value": queries / (e2e_ms * 1e-3), "unit": "queries/s", "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes, "ms_per_step": e2e_ms,
            "how": "q in from pinned host memory and out/lse back every step, on two copy streams "
                   f"overlapping the neighbouring steps' kernels; {ROT} independent batches rotate "
                   "(inputs never L2-resident); 24 steps per CUDA graph replay"},
        "gpu_launches": (1 if weighted else 3 if qgc else 2) * K_steps,  # our kernels in the timed steps
        "clocks": clk,
        "dense": dense,
        "builds_once_after_prefill": builds,
        **secondary,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        more_k = (secondary["budget_5pct"]["k_top"],) if "budget_5pct" in secondary else ()
        res["cpu_baseline"], oracle_res = cpu_baseline(wl, args.cpu_seconds, workload_label(wl, args.budget), more_k)
        if qgc and not args.no_selection_check:
            qs = su0_qsel()
            big = torch.iinfo(torch.int32).max
            srt = torch.sort(torch.where(qs[1] > 0, qs[0], torch.full_like(qs[0], big)), dim=-1).values
            res["selection_check"] = selection_check(wl, oracle_res, srt, qs[2])
        elif not weighted and not args.no_selection_check:
            res["selection_check"] = selection_check(wl, oracle_res, idx, nk,
                                                     s0.get("idx5"), s0.get("nk5"), more_k)
    dist.close()
    return res


# ----------------------------------------------------------------- reference arm
def run_reference(args, dist):
    """The float64 oracle on the host cores, rank 0 only; same metric and config."""
    if dist.rank != 0:
        return None
    import torch
    from weighted_coreset_softmax_b200 import workloads as W
    _pool_init()
    name = args.workload
    # a bounded sample of the same workload: the first sequences of the batch
    nseq = 4
    wl = W.make(name, "cpu", budget=args.budget, B=min(nseq, W.make(name, "cpu", materialize=False).B))
    if args.scorer == "mean16" and wl.score_mode == "summary":
        wl.score_mode = "summary_mean16"
    nseq = wl.B
    workers = max(1, min(os.cpu_count() or 1, 32))
    steps = args.steps
    # one step = one (sequence, KV head) decode step; capped so the run stays short
    t_one = time.perf_counter()
    _oracle_task(oracle_tasks(wl, [(0, 0)])[0])
    t_one = time.perf_counter() - t_one
    cap = int(max(workers, 90.0 * workers / max(t_one, 1e-3)))
    n = min(steps, cap)
    if args.warmup:
        time_oracle(wl, min(args.warmup, workers), workers)
    dt, n, _ = time_oracle(wl, n, workers)
    queries = n / wl.Hkv
    value = queries / dt
    sample = (f"{n} (sequence, KV head) decode steps = {queries:g} queries from the first {nseq} sequences "
              f"of the workload; float64 NumPy oracle, {workers} spawn workers, 1 BLAS thread each")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": dist.world,
        "steps": n, "warmup": args.warmup, "ms_per_step": dt / n * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(wl, args.budget) + f" (sample of {nseq} sequences)",
                   "parallelism": "host CPU pool"},
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": workers, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    args = parse_args(argv)
    dist = Dist()
    if args.impl == "reference":
        res = run_reference(args, dist)
    else:
        res = run_ours(args, dist)
    if res is not None and dist.rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
