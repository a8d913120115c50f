"""Seeded synthetic decode workloads.

This module only draws inputs: queries, KV caches, coreset indices and weights.
It holds none of the method's arithmetic (no scores, no selection, no softmax),
so the CUDA path and the float64 oracle can both be fed from it.

The shapes follow the workloads on the pages:
  * Llama-3.1-8B-shaped GQA decode (32 query heads, 8 KV heads, head dim 128),
    32K context, block size 64 -- "OpenAttention reads 1% of the KV cache",
    section "The news" (batch 32, 32K context).
  * Qwen2.5-7B-shaped long context (28 query heads, 4 KV heads, head dim 128),
    128K context, block size 128.
  * A tiny single-head fp32 check.
They stand in for the RULER-32K long-context suite the pages evaluate on; no item
of that suite is reproduced.

Key distribution: k = s_c * z with z ~ N(0, 1) and a per-(sequence, KV head,
channel) scale s_c ~ lognormal(0, 0.5); a number of planted heavy-hitter tokens per
KV head have keys hh_gain * unit(sum of the group's queries) + N(0, 0.1^2).
Values ~ N(0, 1). Queries ~ N(0, 1), except in the stored-descriptor workload
(llama_cobs_fp4), whose queries are anisotropic: q = R (sigma * z) with z ~ N(0, I),
a seeded rotation R and sigma_j^2 proportional to exp(-j / 45) (normalised to
E|q|^2 = D), so that about 85 of 128 directions carry 90% of the query energy --
the subspace size the COBS page reports at D = 128 (340 = 4 x 85 floats per block).
Its calibration queries (calibration_queries) come from the same model.

Draw order per generator: q, channel scales, K, V, planted positions, planted
noise, then (weighted workloads) coreset indices and weights.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    Ncap: int
    block_size: int
    dtype: torch.dtype
    seq_lens: List[int]
    scale: float                 # softmax scale sigma applied to q.k
    k_top: int                   # blocks chosen by score, forced blocks not counted
    force_first: int
    force_last: int
    score_mode: str              # "summary", "exact_mass", "quest" or "cobs"
    attn_mode: str               # "proxy", "discard", "weighted" or "dense"
    m: int = 0                   # coreset size per (sequence, KV head), weighted mode
    q: Optional[torch.Tensor] = None        # [B][Hq][D]
    K: Optional[torch.Tensor] = None        # [B][Hkv][Ncap][D]
    V: Optional[torch.Tensor] = None        # [B][Hkv][Ncap][D]
    tok_idx: Optional[torch.Tensor] = None  # [B][Hkv][m] int32
    w: Optional[torch.Tensor] = None        # [B][Hkv][m] fp32
    q_model: Optional[tuple] = None         # (R [D][D], sigma [D]) of anisotropic queries

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def NBcap(self) -> int:
        return (self.Ncap + self.block_size - 1) // self.block_size

    @property
    def kmax(self) -> int:
        nb = self.NBcap
        forced = (1 if self.force_first else 0) + (1 if self.force_last else 0)
        return min(nb, self.k_top + forced)

    def seq_lens_tensor(self, device) -> torch.Tensor:
        return torch.tensor(self.seq_lens, dtype=torch.int32, device=device)


def query_model(D: int, tau: float = 45.0, seed: int = 77):
    """The anisotropic query distribution: (R, sigma) with R a seeded rotation (QR of
    a Gaussian matrix, drawn on the CPU so every device sees the same one) and
    sigma_j = sqrt(lambda_j), lambda_j proportional to exp(-j / tau), sum lambda = D."""
    g = torch.Generator().manual_seed(seed)
    R, _ = torch.linalg.qr(torch.randn(D, D, generator=g, dtype=torch.float64))
    lam = torch.exp(-torch.arange(D, dtype=torch.float64) / tau)
    lam = lam * (D / lam.sum())
    return R.to(torch.float32), lam.sqrt().to(torch.float32)


def _draw_sequence(gen, device, Hq, Hkv, D, N, n_planted, hh_gain, dtype,
                   q_scale=1.0, channel_sigma=0.5, plain=False, q_model=None):
    """Draws one sequence's query and cache. Returns q [Hq][D], K, V [Hkv][N][D]."""
    G = Hq // Hkv
    q = torch.randn(Hq, D, generator=gen, device=device, dtype=torch.float32) * q_scale
    if q_model is not None:
        R, sig = q_model
        q = (q * sig.to(device)) @ R.to(device).T
    if plain:
        K = torch.randn(Hkv, N, D, generator=gen, device=device, dtype=torch.float32)
        V = torch.randn(Hkv, N, D, generator=gen, device=device, dtype=torch.float32)
        return q.to(dtype), K.to(dtype), V.to(dtype)
    scales = torch.exp(channel_sigma * torch.randn(Hkv, 1, D, generator=gen, device=device))
    K = torch.randn(Hkv, N, D, generator=gen, device=device, dtype=torch.float32)
    K.mul_(scales)
    V = torch.randn(Hkv, N, D, generator=gen, device=device, dtype=torch.float32)
    if n_planted > 0:
        pos = torch.stack([torch.randperm(N, generator=gen, device=device)[:n_planted]
                           for _ in range(Hkv)])
        noise = 0.1 * torch.randn(Hkv, n_planted, D, generator=gen, device=device)
        qg = q.view(Hkv, G, D).sum(dim=1)
        qhat = qg / qg.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        planted = hh_gain * qhat[:, None, :] + noise
        for h in range(Hkv):
            K[h, pos[h]] = planted[h]
    return q.to(dtype), K.to(dtype), V.to(dtype)


def _draw_coreset(gen, device, B, Hkv, N, m):
    idx = torch.empty(B, Hkv, m, dtype=torch.int32, device=device)
    for b in range(B):
        for h in range(Hkv):
            perm = torch.randperm(N, generator=gen, device=device)[:m]
            idx[b, h] = perm.to(torch.int32)
    w = torch.exp(torch.randn(B, Hkv, m, generator=gen, device=device, dtype=torch.float32))
    w = w * (float(N) / w.sum(dim=-1, keepdim=True))
    return idx, w


def make(name: str, device="cpu", *, B=None, Ncap=None, seq_lens=None, budget=0.01,
         hh_gain=4.0, seed=None, attn_mode=None, score_mode=None, k_top=None,
         m=None, materialize=True) -> Workload:
    """Builds one named workload.

    name: "tiny" (1 head, d=64, n=1024, L=16, fp32), "llama_b1" (batch 1, 32K),
    "llama" (batch 32, 32K, seeds 100..131), "qwen_long" (batch 8, 128K, G=7),
    "llama_osa" (exact-mass scoring), "llama_quest" (key-box bound scoring),
    "llama_cobs" (second-order scoring, rank-4 covariance factors),
    "llama_cobs_fp4" (the stored descriptor: bf16 means, query-subspace E2M1
    factors; anisotropic queries), "llama_qgc" (query-guided clusters with an
    error-gated read; anisotropic queries), "llama_coreset" (weighted coreset, m=2048).
    Keyword overrides shrink a workload for fast tests while keeping its head
    shapes and distributions.
    """
    dev = torch.device(device)
    if name == "tiny":
        spec = dict(B=1, Hq=1, Hkv=1, D=64, Ncap=1024, L=16, dtype=torch.float32,
                    k_top=8, ff=0, fl=0, smode="summary", amode="proxy", planted=0,
                    seeds=[0], per_seq=True, plain=True)
    elif name == "llama_b1":
        spec = dict(B=1, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=None, ff=1, fl=1, smode="summary", amode="proxy", planted=32,
                    seeds=[1], per_seq=True, plain=False)
    elif name == "llama":
        spec = dict(B=32, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=None, ff=1, fl=1, smode="summary", amode="proxy", planted=32,
                    seeds=list(range(100, 132)), per_seq=True, plain=False)
    elif name == "qwen_long":
        spec = dict(B=8, Hq=28, Hkv=4, D=128, Ncap=131072, L=128, dtype=torch.bfloat16,
                    k_top=None, ff=1, fl=1, smode="summary", amode="proxy", planted=128,
                    seeds=[2], per_seq=False, plain=False)
    elif name == "llama_osa":
        spec = dict(B=32, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=None, ff=1, fl=1, smode="exact_mass", amode="proxy", planted=32,
                    seeds=[3], per_seq=False, plain=False)
    elif name == "llama_quest":
        spec = dict(B=32, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=None, ff=1, fl=1, smode="quest", amode="proxy", planted=32,
                    seeds=[4], per_seq=False, plain=False)
    elif name == "llama_cobs":
        spec = dict(B=32, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=None, ff=1, fl=1, smode="cobs", amode="proxy", planted=32,
                    seeds=[5], per_seq=False, plain=False)
    elif name == "llama_cobs_fp4":
        spec = dict(B=32, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=None, ff=1, fl=1, smode="cobs_fp4", amode="proxy", planted=32,
                    seeds=[6], per_seq=False, plain=False, aniso=True)
    elif name == "llama_qgc":
        spec = dict(B=32, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=0, ff=0, fl=0, smode="qgc", amode="qgc", planted=32,
                    seeds=[7], per_seq=False, plain=False, aniso=True)
    elif name == "llama_coreset":
        spec = dict(B=32, Hq=32, Hkv=8, D=128, Ncap=32768, L=64, dtype=torch.bfloat16,
                    k_top=0, ff=0, fl=0, smode="summary", amode="weighted", planted=32,
                    seeds=[3], per_seq=False, plain=False, m=2048)
    else:
        raise ValueError(f"unknown workload {name!r}")

    Bv = B if B is not None else spec["B"]
    N = Ncap if Ncap is not None else spec["Ncap"]
    L = spec["L"]
    nb = (N + L - 1) // L
    if seq_lens is None:
        seq_lens = [N] * Bv
    assert len(seq_lens) == Bv and all(0 <= s <= N for s in seq_lens)
    kt = k_top if k_top is not None else spec["k_top"]
    if kt is None:
        kt = max(1, int(math.floor(budget * nb)))
    mm = m if m is not None else spec.get("m", 0)
    scale = 1.0 if name == "tiny" else 1.0 / math.sqrt(spec["D"])
    wl = Workload(name=name, B=Bv, Hq=spec["Hq"], Hkv=spec["Hkv"], D=spec["D"], Ncap=N,
                  block_size=L, dtype=spec["dtype"], seq_lens=list(seq_lens), scale=scale,
                  k_top=kt, force_first=spec["ff"], force_last=spec["fl"],
                  score_mode=score_mode or spec["smode"], attn_mode=attn_mode or spec["amode"],
                  m=mm)
    if not materialize:
        return wl

    n_planted = spec["planted"]
    if N < 4 * n_planted:
        n_planted = max(1, N // 64) if n_planted else 0
    q_scale = 1.0 / math.sqrt(spec["D"]) if name == "tiny" else 1.0
    q = torch.empty(Bv, wl.Hq, wl.D, dtype=wl.dtype, device=dev)
    K = torch.empty(Bv, wl.Hkv, N, wl.D, dtype=wl.dtype, device=dev)
    V = torch.empty_like(K)
    seeds = spec["seeds"]
    if seed is not None:
        seeds = [seed + i for i in range(len(seeds))]
    qm = query_model(spec["D"]) if spec.get("aniso") else None
    wl.q_model = qm
    gen = None
    for b in range(Bv):
        if spec["per_seq"] or gen is None:
            s = seeds[b % len(seeds)] + (b // len(seeds)) * 1000 if spec["per_seq"] else seeds[0]
            gen = torch.Generator(device=dev)
            gen.manual_seed(s)
        qb, Kb, Vb = _draw_sequence(gen, dev, wl.Hq, wl.Hkv, wl.D, N, n_planted, hh_gain,
                                    wl.dtype, q_scale=q_scale, plain=spec["plain"], q_model=qm)
        q[b], K[b], V[b] = qb, Kb, Vb
    wl.q, wl.K, wl.V = q, K, V
    if wl.attn_mode == "weighted":
        idx, w = _draw_coreset(gen, dev, Bv, wl.Hkv, min(seq_lens) if seq_lens else N, wl.m)
        wl.tok_idx, wl.w = idx, w
    return wl


def equalize_tail(wl: Workload, kept_blocks) -> None:
    """Rewrites, in place, every key outside the kept blocks of each (sequence,
    KV head) to the mean of those keys, so that all tail logits are equal.

    kept_blocks: nested list [b][h] -> iterable of kept block indices.
    Used for the "proxy is exact when every tail logit is equal" case.
    """
    L = wl.block_size
    for b in range(wl.B):
        n = wl.seq_lens[b]
        for h in range(wl.Hkv):
            mask = torch.ones(n, dtype=torch.bool, device=wl.K.device)
            for blk in kept_blocks[b][h]:
                mask[blk * L:min(n, (blk + 1) * L)] = False
            if mask.any():
                tail = wl.K[b, h, :n][mask].to(torch.float64)
                mean = tail.mean(dim=0).to(wl.dtype)
                wl.K[b, h, :n][mask] = mean


def calibration_queries(wl: Workload, Nc: int, seed: int = 9001) -> torch.Tensor:
    """Nc calibration positions of queries [Nc][Hq][D] (the workload's dtype) from the
    workload's query distribution (its anisotropic model when it has one)."""
    dev = wl.q.device if wl.q is not None else torch.device("cpu")
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    z = torch.randn(Nc, wl.Hq, wl.D, generator=gen, device=dev, dtype=torch.float32)
    if wl.q_model is not None:
        R, sig = wl.q_model
        z = (z * sig.to(dev)) @ R.to(dev).T
    return z.to(wl.dtype)
