"""Shared helpers for the GPU parity tests: run the library on a workload and
compare with the float64 oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import weighted_coreset_softmax_b200 as kv
from oracle import oracle as O

# Max relative error of an output row (max_j |o_j - o*_j| / max_j |o*_j|), the
# tolerance the target states for fp32 accumulation over bf16 inputs.
OUT_TOL = 2e-3


def to64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 / fp32 device tensor."""
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def row_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    got = got.reshape(-1, got.shape[-1])
    ref = ref.reshape(-1, ref.shape[-1])
    worst = 0.0
    for g, r in zip(got, ref):
        denom = float(np.max(np.abs(r)))
        err = float(np.max(np.abs(g - r)))
        worst = max(worst, err / denom if denom > 0 else err)
    return worst


def check_out(got_out, got_lse, ref_out, ref_lse, rows=None, tol=OUT_TOL, what=""):
    go = got_out.detach().cpu().numpy().astype(np.float64)
    gl = got_lse.detach().cpu().numpy().astype(np.float64) if got_lse is not None else None
    if rows is not None:
        go = np.stack([go[b, hq] for (b, hq) in rows])
        ref_out = np.stack([ref_out[b, hq] for (b, hq) in rows])
        if gl is not None:
            gl = np.array([gl[b, hq] for (b, hq) in rows])
            ref_lse = np.array([ref_lse[b, hq] for (b, hq) in rows])
    err = row_rel_err(go, ref_out)
    assert err <= tol, f"{what}: output row rel err {err:.3e} > {tol:.1e}"
    if gl is not None:
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(gl), fin), f"{what}: lse finiteness differs"
        if fin.any():
            lerr = float(np.max(np.abs(gl[fin] - ref_lse[fin]) / np.maximum(1.0, np.abs(ref_lse[fin]))))
            assert lerr <= tol, f"{what}: lse err {lerr:.3e}"
    return err


# Near ties seen by the selection checks of this session: (label, pairs checked,
# pairs the oracle flags as a near tie, pairs whose kept set differs there). The
# session summary (tests/conftest.py) prints them.
NEAR_TIES = []


def record_near_ties(what, n_pairs, n_flagged, n_mismatch):
    NEAR_TIES.append((what, int(n_pairs), int(n_flagged), int(n_mismatch)))


# Other figures a test reports rather than asserts (printed in the session summary).
NOTES = []


def record_note(text):
    NOTES.append(str(text))


def selection_matches(gpu_idx, gpu_nk, sel_ref, pairs, what=""):
    """Kept sets must be bit-exact unless the oracle flags a near tie at the k / k+1
    boundary; returns the number of near-tie pairs where they differ (also
    recorded for the session's near-tie report)."""
    gi = gpu_idx.cpu().numpy()
    gn = gpu_nk.cpu().numpy()
    ties = 0
    for (b, h) in pairs:
        ref = sel_ref[(b, h)]
        got = [int(x) for x in gi[b, h, :gn[b, h]]]
        assert got == sorted(got), f"{what}: indices not ascending at {(b, h)}: {got}"
        if got != ref["kept"]:
            assert ref["near_tie"], f"{what}: kept {got} != oracle {ref['kept']} at {(b, h)} (no near tie)"
            ties += 1
    record_near_ties(what, len(pairs), sum(1 for p in pairs if sel_ref[p]["near_tie"]), ties)
    return ties


def oracle_inputs(wl):
    q = to64(wl.q)
    K = to64(wl.K)
    V = to64(wl.V)
    return q, K, V


def run_pipeline(wl, *, want_scores=True, use_proxy=True, kmax=None):
    """GPU: summaries, selection and sparse attention for a workload."""
    dev = wl.q.device
    sl = wl.seq_lens_tensor(dev)
    summ = kv.kv_build_block_summaries(wl.K, wl.V, sl, wl.block_size)
    if wl.score_mode == "cobs":
        summ["k_xi"] = kv.kv_build_block_cov_factors(wl.K, sl, wl.block_size, 4)
        idx, nk, scores = kv.kv_select_blocks_cobs(wl.q, wl.K, sl, wl.block_size, wl.scale, summ["k_sum"],
                                                   summ["counts"], summ["k_xi"], wl.k_top, wl.force_first,
                                                   wl.force_last, kmax=kmax, want_scores=want_scores)
    elif wl.score_mode == "summary_mean16":
        summ["k_mean"] = kv.kv_build_block_key_means(wl.K, sl, wl.block_size, summ["k_sum"], summ["counts"])
        idx, nk, scores = kv.kv_select_blocks_mean16(wl.q, wl.K, sl, wl.block_size, wl.scale, summ["k_mean"],
                                                     summ["counts"], wl.k_top, wl.force_first, wl.force_last,
                                                     kmax=kmax, want_scores=want_scores)
    elif wl.score_mode == "quest":
        summ["k_bounds"] = kv.kv_build_block_bounds(wl.K, sl, wl.block_size)
        idx, nk, scores = kv.kv_select_blocks_quest(wl.q, wl.K, sl, wl.block_size, wl.scale, summ["k_bounds"],
                                                    wl.k_top, wl.force_first, wl.force_last, kmax=kmax,
                                                    want_scores=want_scores)
    else:
        mode = kv.KV_SCORE_SUMMARY if wl.score_mode == "summary" else kv.KV_SCORE_EXACT_MASS
        idx, nk, scores = kv.kv_select_blocks(wl.q, wl.K, sl, wl.block_size, wl.scale, summ["counts"],
                                              wl.k_top, wl.force_first, wl.force_last, mode=mode,
                                              k_sum=summ["k_sum"], kmax=kmax, want_scores=want_scores)
    shape = kv.make_shape(wl.q, wl.K, sl, wl.block_size)
    ws = kv.Workspace(shape, dev)
    out, lse = kv.kv_sparse_decode_attn(wl.q, wl.K, wl.V, sl, wl.block_size, wl.scale, ws,
                                        block_idx=idx, n_kept=nk, summaries=summ,
                                        use_tail_proxy=use_proxy)
    torch.cuda.synchronize()
    status = kv.kv_workspace_status(ws.tensor)
    assert status == 0, f"device status 0x{status:x}"
    return dict(summ=summ, idx=idx, nk=nk, scores=scores, out=out, lse=lse, ws=ws, sl=sl)


def kept_tensor(sel, B, Hkv, kmax, device):
    idx = torch.zeros(B, Hkv, kmax, dtype=torch.int32)
    nk = torch.zeros(B, Hkv, dtype=torch.int32)
    for (b, h), s in sel.items():
        k = s["kept"]
        nk[b, h] = len(k)
        idx[b, h, :len(k)] = torch.tensor(k, dtype=torch.int32)
    return idx.to(device), nk.to(device)


def all_pairs(wl):
    return [(b, h) for b in range(wl.B) for h in range(wl.Hkv)]


def rows_of(wl, pairs):
    G = wl.G
    return [(b, h * G + g) for (b, h) in pairs for g in range(G)]


def finite_or_neg_inf(x):
    return x if math.isfinite(x) else -math.inf
