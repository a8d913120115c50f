"""Reduced-KV softmax decode attention for B200 (sm_100a).

Thin Python binding of libkvsparse.so (C ABI declared in include/kvsparse.h).
The functions keep the C names; they only marshal torch tensors into pointers,
sizes and the current CUDA stream. Every step of the computation runs in the
library's CUDA kernels; there is no fallback: if the library is missing or no GPU
is present the calls raise.

Method (see include/kvsparse.h for the per-call sources):
  kv_build_block_summaries  once after prefill: per-block key/value sums, counts
  kv_select_blocks          per step: GQA-normalised block score, top-k per KV head
  kv_sparse_decode_attn     per step: attention over kept blocks + tail proxy, or
                            over a weighted coreset
  kv_dense_decode_attn      exact attention over every token (baseline)
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from typing import Optional

import torch

__all__ = [
    "KV_OK", "KV_ERR_INVALID_ARG", "KV_ERR_UNSUPPORTED", "KV_ERR_CUDA", "KV_ERR_DEVICE_CHECK",
    "KV_BF16", "KV_F32", "KV_SCORE_SUMMARY", "KV_SCORE_EXACT_MASS", "KV_STEP_AUTO", "KV_STEP_TWO_KERNELS",
    "KV_STEP_FUSED", "KVShape", "KVError",
    "lib", "library_path", "header_path", "make_shape", "kv_build_block_summaries",
    "kv_select_blocks", "kv_build_block_bounds", "kv_select_blocks_quest", "kv_build_block_key_means",
    "kv_select_blocks_mean16",
    "kv_build_block_cov_factors", "kv_select_blocks_cobs", "kv_sparse_decode_attn", "kv_dense_decode_attn", "kv_decode_step", "kv_workspace_bytes",
    "kv_workspace_init", "kv_workspace_status", "kv_last_error", "Workspace", "kv_selftest_wait_timeout",
    "kv_stream_read", "kv_build_wildcat_coreset", "kv_build_query_basis", "kv_query_subspace_rank",
    "kv_build_block_cov_factors_ss", "kv_quantize_fp4", "kv_select_blocks_cobs_fp4", "kv_build_qgc",
    "kv_select_qgc", "kv_merge_qgc_proxies", "qgc_decode",
]

KV_OK, KV_ERR_INVALID_ARG, KV_ERR_UNSUPPORTED, KV_ERR_CUDA, KV_ERR_DEVICE_CHECK = 0, 1, 2, 3, 4
KV_BF16, KV_F32 = 0, 1
KV_SCORE_SUMMARY, KV_SCORE_EXACT_MASS = 0, 1
KV_STEP_AUTO, KV_STEP_TWO_KERNELS, KV_STEP_FUSED = 0, 1, 2

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)


def library_path() -> str:
    return os.path.join(_PKG, "libkvsparse.so")


def header_path() -> str:
    return os.path.join(_ROOT, "include", "kvsparse.h")


class KVShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("Ncap", ctypes.c_int), ("block_size", ctypes.c_int),
                ("dtype", ctypes.c_int), ("seq_lens", ctypes.c_void_p)]


class KVError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"kvsparse status {status}: {message}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t
_SHP = ctypes.POINTER(KVShape)


def lib():
    """Loads libkvsparse.so (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with "
                           "`python -m weighted_coreset_softmax_b200.build`")
    L = ctypes.CDLL(path)
    sigs = {
        "kv_build_block_summaries": [_SHP, _P, _P, _P, _P, _P, _P, _P, _P],
        "kv_select_blocks": [_SHP, _P, _F, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P],
        "kv_build_block_bounds": [_SHP, _P, _P, _P],
        "kv_build_block_key_means": [_SHP, _P, _P, _P, _P],
        "kv_select_blocks_mean16": [_SHP, _P, _F, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P],
        "kv_select_blocks_quest": [_SHP, _P, _F, _P, _I, _I, _I, _I, _P, _P, _P, _P],
        "kv_build_block_cov_factors": [_SHP, _P, _I, _P, _P],
        "kv_select_blocks_cobs": [_SHP, _P, _F, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P],
        "kv_sparse_decode_attn": [_SHP, _P, _F, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _I,
                                  _P, _P, _I, _P, _P, _P, _S, _P],
        "kv_dense_decode_attn": [_SHP, _P, _F, _P, _P, _P, _P, _P, _S, _P],
        "kv_decode_step": [_SHP, _P, _F, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                           _P, _S, _I, _P],
        "kv_workspace_init": [_P, _S, _P],
        "kv_workspace_status": [_P, ctypes.POINTER(ctypes.c_uint32), _P],
        "kv_selftest_wait_timeout": [_P, _P, ctypes.c_uint64, _I, _P],
        "kv_stream_read": [_P, _S, _P, _P],
        "kv_build_wildcat_coreset": [_SHP, _P, _F, _I, _I, _P, _P, _P, _P, _P, _S, _P],
        "kv_build_query_basis": [_P, _I, _I, _I, _I, _I, _P, _P, _P, _S, _P],
        "kv_build_block_cov_factors_ss": [_SHP, _P, _P, _I, _I, _P, _P],
        "kv_quantize_fp4": [_P, ctypes.c_longlong, _I, _P, _P, _P],
        "kv_select_blocks_cobs_fp4": [_SHP, _P, _F, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P],
        "kv_query_subspace_rank": [_P, _I, _I, ctypes.c_double],
        "kv_build_qgc": [_SHP, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P],
        "kv_select_qgc": [_SHP, _P, _F, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _I, _P, _P, _P, _P, _P,
                          _P, _P, _S, _P],
        "kv_merge_qgc_proxies": [_SHP, _P, _F, _I, _P, _P, _P, _P, _P, _P],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = _I
    L.kv_workspace_bytes.argtypes = [_SHP]
    L.kv_workspace_bytes.restype = _S
    L.kv_wildcat_workspace_bytes.argtypes = [_SHP, _I]
    L.kv_wildcat_workspace_bytes.restype = _S
    L.kv_query_basis_workspace_bytes.argtypes = [_I, _I]
    L.kv_query_basis_workspace_bytes.restype = _S
    for fn in ("kv_qgc_workspace_bytes", "kv_qgc_select_workspace_bytes"):
        getattr(L, fn).argtypes = [_SHP]
        getattr(L, fn).restype = _S
    L.kv_last_error.argtypes = []
    L.kv_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def header_functions():
    """Names of the functions include/kvsparse.h declares."""
    with open(header_path()) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kv_[a-z_]+)\s*\(", text)))


def kv_last_error() -> str:
    return lib().kv_last_error().decode()


def _check(status: int):
    if status != KV_OK:
        raise KVError(status, kv_last_error())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return KV_BF16
    if dt == torch.float32:
        return KV_F32
    raise TypeError(f"unsupported cache dtype {dt}")


def _need(t: torch.Tensor, name: str, dtype=None, cuda=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def make_shape(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor, block_size: int) -> KVShape:
    """Shape descriptor from q [B][Hq][D], K [B][Hkv][Ncap][D], seq_lens [B] int32."""
    if q.dim() != 3 or K.dim() != 4:
        raise ValueError("q must be [B][Hq][D] and K [B][Hkv][Ncap][D]")
    B, Hq, D = q.shape
    B2, Hkv, Ncap, D2 = K.shape
    if B != B2 or D != D2:
        raise ValueError(f"q {tuple(q.shape)} and K {tuple(K.shape)} disagree")
    return KVShape(B, Hq, Hkv, D, Ncap, int(block_size), _dtype_code(K.dtype),
                   seq_lens.data_ptr() if seq_lens is not None else None)


def kv_workspace_bytes(shape: KVShape) -> int:
    return int(lib().kv_workspace_bytes(ctypes.byref(shape)))


class Workspace:
    """A zero-initialised device workspace for the attention entry points."""

    def __init__(self, shape: KVShape, device):
        n = kv_workspace_bytes(shape)
        self.tensor = torch.zeros(max(n, 256), dtype=torch.uint8, device=device)

    @property
    def nbytes(self) -> int:
        return self.tensor.numel()

    def ptr(self):
        return ctypes.c_void_p(self.tensor.data_ptr())


def kv_workspace_init(ws: torch.Tensor):
    _check(lib().kv_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(ws.device)))


def kv_workspace_status(ws: torch.Tensor) -> int:
    v = ctypes.c_uint32(0)
    st = lib().kv_workspace_status(_ptr(ws), ctypes.byref(v), _stream(ws.device))
    if st not in (KV_OK, KV_ERR_DEVICE_CHECK):
        _check(st)
    return int(v.value)


def kv_build_block_summaries(K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                             out: Optional[dict] = None) -> dict:
    """Block summaries of the cache; returns dict(k_sum, v_sum, counts, k_tot, v_tot)."""
    _need(K, "K")
    _need(V, "V", K.dtype)
    _need(seq_lens, "seq_lens", torch.int32)
    B, Hkv, Ncap, D = K.shape
    NB = (Ncap + block_size - 1) // block_size
    dev = K.device
    if out is None:
        out = {
            "k_sum": torch.empty(B, Hkv, NB, D, dtype=torch.float32, device=dev),
            "v_sum": torch.empty(B, Hkv, NB, D, dtype=torch.float32, device=dev),
            "counts": torch.empty(B, NB, dtype=torch.int32, device=dev),
            "k_tot": torch.empty(B, Hkv, D, dtype=torch.float32, device=dev),
            "v_tot": torch.empty(B, Hkv, D, dtype=torch.float32, device=dev),
        }
    shape = KVShape(B, Hkv, Hkv, D, Ncap, block_size, _dtype_code(K.dtype), seq_lens.data_ptr())
    _check(lib().kv_build_block_summaries(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(out["k_sum"]),
                                          _ptr(out["v_sum"]), _ptr(out["counts"]), _ptr(out["k_tot"]),
                                          _ptr(out["v_tot"]), _stream(dev)))
    return out


def kv_select_blocks(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                     scale: float, counts: torch.Tensor, k_top: int, force_first: bool = False,
                     force_last: bool = False, mode: int = KV_SCORE_SUMMARY,
                     k_sum: Optional[torch.Tensor] = None, kmax: Optional[int] = None,
                     block_idx: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                     scores: Optional[torch.Tensor] = None, want_scores: bool = False):
    """Kept blocks per KV head. K is read only in exact-mass mode (its shape is
    always used for the descriptor). Returns (block_idx [B][Hkv][kmax], n_kept
    [B][Hkv], scores or None)."""
    _need(q, "q", K.dtype)
    _need(counts, "counts", torch.int32)
    if mode == KV_SCORE_SUMMARY:
        _need(k_sum, "k_sum", torch.float32)
    else:
        _need(K, "K")
    shape = make_shape(q, K, seq_lens, block_size)
    NB = (shape.Ncap + block_size - 1) // block_size
    forced = int(bool(force_first)) + int(bool(force_last))
    if kmax is None:
        kmax = max(1, min(NB, k_top + forced))
    dev = q.device
    if block_idx is None:
        block_idx = torch.zeros(shape.B, shape.Hkv, kmax, dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.zeros(shape.B, shape.Hkv, dtype=torch.int32, device=dev)
    if scores is None and want_scores:
        scores = torch.empty(shape.B, shape.Hkv, NB, dtype=torch.float32, device=dev)
    _check(lib().kv_select_blocks(ctypes.byref(shape), _ptr(q), float(scale), int(mode), _ptr(k_sum),
                                  _ptr(counts), _ptr(K) if mode == KV_SCORE_EXACT_MASS else None,
                                  int(k_top), int(bool(force_first)), int(bool(force_last)), int(kmax),
                                  _ptr(block_idx), _ptr(n_kept), _ptr(scores), _stream(dev)))
    return block_idx, n_kept, scores


def kv_build_block_key_means(K: torch.Tensor, seq_lens: torch.Tensor, block_size: int, k_sum: torch.Tensor,
                             counts: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Block mean keys at bf16 precision [B][Hkv][NB][D] from the fp32 key sums and
    counts of kv_build_block_summaries (K gives the shape only)."""
    _need(K, "K", torch.bfloat16)
    _need(k_sum, "k_sum", torch.float32)
    _need(counts, "counts", torch.int32)
    B, Hkv, Ncap, D = K.shape
    NB = (Ncap + block_size - 1) // block_size
    if out is None:
        out = torch.empty(B, Hkv, NB, D, dtype=torch.bfloat16, device=K.device)
    shape = KVShape(B, Hkv, Hkv, D, Ncap, block_size, KV_BF16, seq_lens.data_ptr())
    _check(lib().kv_build_block_key_means(ctypes.byref(shape), _ptr(k_sum), _ptr(counts), _ptr(out),
                                          _stream(K.device)))
    return out


def kv_select_blocks_mean16(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                            scale: float, k_mean: torch.Tensor, counts: torch.Tensor, k_top: int,
                            force_first: bool = False, force_last: bool = False, kmax: Optional[int] = None,
                            block_idx: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                            scores: Optional[torch.Tensor] = None, want_scores: bool = False):
    """Kept blocks per KV head scored from the bf16 block means (summary score
    with the mean at bf16). K is not read. Returns (block_idx [B][Hkv][kmax],
    n_kept [B][Hkv], scores or None)."""
    _need(q, "q", torch.bfloat16)
    _need(k_mean, "k_mean", torch.bfloat16)
    _need(counts, "counts", torch.int32)
    shape = make_shape(q, K, seq_lens, block_size)
    NB = (shape.Ncap + block_size - 1) // block_size
    forced = int(bool(force_first)) + int(bool(force_last))
    if kmax is None:
        kmax = max(1, min(NB, k_top + forced))
    dev = q.device
    if block_idx is None:
        block_idx = torch.zeros(shape.B, shape.Hkv, kmax, dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.zeros(shape.B, shape.Hkv, dtype=torch.int32, device=dev)
    if scores is None and want_scores:
        scores = torch.empty(shape.B, shape.Hkv, NB, dtype=torch.float32, device=dev)
    _check(lib().kv_select_blocks_mean16(ctypes.byref(shape), _ptr(q), float(scale), _ptr(k_mean), _ptr(counts),
                                         int(k_top), int(bool(force_first)), int(bool(force_last)), int(kmax),
                                         _ptr(block_idx), _ptr(n_kept), _ptr(scores), _stream(dev)))
    return block_idx, n_kept, scores


def kv_build_block_bounds(K: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                          out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per-block key bounding boxes of a bf16 cache: [B][Hkv][NB][D][2] bf16, the
    last axis (min, max)."""
    _need(K, "K", torch.bfloat16)
    _need(seq_lens, "seq_lens", torch.int32)
    B, Hkv, Ncap, D = K.shape
    NB = (Ncap + block_size - 1) // block_size
    if out is None:
        out = torch.empty(B, Hkv, NB, D, 2, dtype=torch.bfloat16, device=K.device)
    shape = KVShape(B, Hkv, Hkv, D, Ncap, block_size, KV_BF16, seq_lens.data_ptr())
    _check(lib().kv_build_block_bounds(ctypes.byref(shape), _ptr(K), _ptr(out), _stream(K.device)))
    return out


def kv_select_blocks_quest(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                           scale: float, k_bounds: torch.Tensor, k_top: int, force_first: bool = False,
                           force_last: bool = False, kmax: Optional[int] = None,
                           block_idx: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                           scores: Optional[torch.Tensor] = None, want_scores: bool = False):
    """Kept blocks per KV head, each query head scoring a block by its key box
    bound. K is not read (its shape gives the descriptor). Returns (block_idx
    [B][Hkv][kmax], n_kept [B][Hkv], scores or None)."""
    _need(q, "q", torch.bfloat16)
    _need(k_bounds, "k_bounds", torch.bfloat16)
    shape = make_shape(q, K, seq_lens, block_size)
    NB = (shape.Ncap + block_size - 1) // block_size
    forced = int(bool(force_first)) + int(bool(force_last))
    if kmax is None:
        kmax = max(1, min(NB, k_top + forced))
    dev = q.device
    if block_idx is None:
        block_idx = torch.zeros(shape.B, shape.Hkv, kmax, dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.zeros(shape.B, shape.Hkv, dtype=torch.int32, device=dev)
    if scores is None and want_scores:
        scores = torch.empty(shape.B, shape.Hkv, NB, dtype=torch.float32, device=dev)
    _check(lib().kv_select_blocks_quest(ctypes.byref(shape), _ptr(q), float(scale), _ptr(k_bounds), int(k_top),
                                        int(bool(force_first)), int(bool(force_last)), int(kmax),
                                        _ptr(block_idx), _ptr(n_kept), _ptr(scores), _stream(dev)))
    return block_idx, n_kept, scores


def kv_build_block_cov_factors(K: torch.Tensor, seq_lens: torch.Tensor, block_size: int, rank: int = 4,
                               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per-block scaled covariance eigenvectors: [B][Hkv][NB][rank][D] fp32."""
    _need(K, "K")
    _need(seq_lens, "seq_lens", torch.int32)
    B, Hkv, Ncap, D = K.shape
    NB = (Ncap + block_size - 1) // block_size
    if out is None:
        out = torch.empty(B, Hkv, NB, rank, D, dtype=torch.float32, device=K.device)
    shape = KVShape(B, Hkv, Hkv, D, Ncap, block_size, _dtype_code(K.dtype), seq_lens.data_ptr())
    _check(lib().kv_build_block_cov_factors(ctypes.byref(shape), _ptr(K), int(rank), _ptr(out), _stream(K.device)))
    return out


def kv_select_blocks_cobs(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                          scale: float, k_sum: torch.Tensor, counts: torch.Tensor, k_xi: torch.Tensor, k_top: int,
                          force_first: bool = False, force_last: bool = False, kmax: Optional[int] = None,
                          block_idx: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                          scores: Optional[torch.Tensor] = None, want_scores: bool = False):
    """Kept blocks per KV head by the second-order block logit. K is not read (its
    shape gives the descriptor); the rank is k_xi's fourth dimension. Returns
    (block_idx [B][Hkv][kmax], n_kept [B][Hkv], scores or None)."""
    _need(q, "q", K.dtype)
    _need(k_sum, "k_sum", torch.float32)
    _need(counts, "counts", torch.int32)
    _need(k_xi, "k_xi", torch.float32)
    shape = make_shape(q, K, seq_lens, block_size)
    NB = (shape.Ncap + block_size - 1) // block_size
    forced = int(bool(force_first)) + int(bool(force_last))
    if kmax is None:
        kmax = max(1, min(NB, k_top + forced))
    dev = q.device
    if block_idx is None:
        block_idx = torch.zeros(shape.B, shape.Hkv, kmax, dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.zeros(shape.B, shape.Hkv, dtype=torch.int32, device=dev)
    if scores is None and want_scores:
        scores = torch.empty(shape.B, shape.Hkv, NB, dtype=torch.float32, device=dev)
    _check(lib().kv_select_blocks_cobs(ctypes.byref(shape), _ptr(q), float(scale), _ptr(k_sum), _ptr(counts),
                                       _ptr(k_xi), int(k_xi.shape[3]), int(k_top), int(bool(force_first)),
                                       int(bool(force_last)), int(kmax), _ptr(block_idx), _ptr(n_kept),
                                       _ptr(scores), _stream(dev)))
    return block_idx, n_kept, scores


def kv_sparse_decode_attn(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor,
                          block_size: int, scale: float, workspace: Workspace, *,
                          block_idx: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                          summaries: Optional[dict] = None, use_tail_proxy: bool = True,
                          tok_idx: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                          want_lse: bool = True):
    """Block mode (block_idx, n_kept, summaries) or weighted-coreset mode
    (tok_idx, w). Returns (out [B][Hq][D] fp32, lse [B][Hq] fp32 or None)."""
    _need(q, "q", K.dtype)
    _need(K, "K")
    _need(V, "V", K.dtype)
    shape = make_shape(q, K, seq_lens, block_size)
    dev = q.device
    if out is None:
        out = torch.empty(shape.B, shape.Hq, shape.D, dtype=torch.float32, device=dev)
    if lse is None and want_lse:
        lse = torch.empty(shape.B, shape.Hq, dtype=torch.float32, device=dev)
    kmax, m = 0, 0
    s = summaries or {}
    if tok_idx is not None:
        _need(tok_idx, "tok_idx", torch.int32)
        _need(w, "w", torch.float32)
        m = tok_idx.shape[-1]
        if m == 0:
            # an empty tensor may have a NULL data pointer, which the C API reads as
            # block mode; with m = 0 nothing is read, so any aligned pointer will do
            tok_idx = w = workspace.tensor
    else:
        _need(block_idx, "block_idx", torch.int32)
        _need(n_kept, "n_kept", torch.int32)
        kmax = block_idx.shape[-1]
    st = lib().kv_sparse_decode_attn(
        ctypes.byref(shape), _ptr(q), float(scale), _ptr(K), _ptr(V), _ptr(block_idx), _ptr(n_kept),
        int(kmax), _ptr(s.get("k_sum")), _ptr(s.get("v_sum")), _ptr(s.get("counts")), _ptr(s.get("k_tot")),
        _ptr(s.get("v_tot")), int(bool(use_tail_proxy)) if tok_idx is None else 0, _ptr(tok_idx), _ptr(w),
        int(m), _ptr(out), _ptr(lse), workspace.ptr(), workspace.nbytes, _stream(dev))
    _check(st)
    return out, lse


def kv_decode_step(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                   scale: float, workspace: Workspace, summaries: dict, k_top: int, force_first: bool = False,
                   force_last: bool = False, *, kmax: Optional[int] = None, use_tail_proxy: bool = True,
                   block_idx: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                   scores: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                   lse: Optional[torch.Tensor] = None, want_lse: bool = True, how: int = KV_STEP_AUTO):
    """Selection (summary mode) and attention over the kept blocks in one call;
    how = KV_STEP_FUSED asks for the single-kernel form. Returns (out, lse or None,
    block_idx, n_kept)."""
    _need(q, "q", K.dtype)
    _need(K, "K")
    _need(V, "V", K.dtype)
    shape = make_shape(q, K, seq_lens, block_size)
    dev = q.device
    NB = (shape.Ncap + block_size - 1) // block_size
    forced = int(bool(force_first)) + int(bool(force_last))
    if kmax is None:
        kmax = max(1, min(NB, k_top + forced))
    if block_idx is None:
        block_idx = torch.zeros(shape.B, shape.Hkv, kmax, dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.zeros(shape.B, shape.Hkv, dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty(shape.B, shape.Hq, shape.D, dtype=torch.float32, device=dev)
    if lse is None and want_lse:
        lse = torch.empty(shape.B, shape.Hq, dtype=torch.float32, device=dev)
    s = summaries
    _check(lib().kv_decode_step(
        ctypes.byref(shape), _ptr(q), float(scale), _ptr(K), _ptr(V), _ptr(s["k_sum"]), _ptr(s["v_sum"]),
        _ptr(s["counts"]), _ptr(s["k_tot"]), _ptr(s["v_tot"]), int(k_top), int(bool(force_first)),
        int(bool(force_last)), int(kmax), int(bool(use_tail_proxy)), _ptr(block_idx), _ptr(n_kept), _ptr(scores),
        _ptr(out), _ptr(lse), workspace.ptr(), workspace.nbytes, int(how), _stream(dev)))
    return out, lse, block_idx, n_kept


def kv_dense_decode_attn(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor,
                         block_size: int, scale: float, workspace: Workspace, *,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         want_lse: bool = True):
    """Exact attention over every cached token. Returns (out, lse or None)."""
    _need(q, "q", K.dtype)
    _need(K, "K")
    _need(V, "V", K.dtype)
    shape = make_shape(q, K, seq_lens, block_size)
    dev = q.device
    if out is None:
        out = torch.empty(shape.B, shape.Hq, shape.D, dtype=torch.float32, device=dev)
    if lse is None and want_lse:
        lse = torch.empty(shape.B, shape.Hq, dtype=torch.float32, device=dev)
    _check(lib().kv_dense_decode_attn(ctypes.byref(shape), _ptr(q), float(scale), _ptr(K), _ptr(V),
                                      _ptr(out), _ptr(lse), workspace.ptr(), workspace.nbytes,
                                      _stream(dev)))
    return out, lse


def kv_selftest_wait_timeout(status: torch.Tensor, limit_ns: int, arrive: bool) -> torch.Tensor:
    """Runs the kernels' bounded copy wait once in a one-warp kernel: with
    arrive=False it waits for bytes no copy delivers and must give up after
    limit_ns, OR-ing KV_DEV_WAIT_TIMEOUT into status (a 1-element int32 device
    tensor); with arrive=True the wait completes. Returns a 1-element device
    tensor: 1 if the wait completed, 0 if it gave up."""
    _need(status, "status", torch.int32)
    ok = torch.full((1,), 7, dtype=torch.int32, device=status.device)
    _check(lib().kv_selftest_wait_timeout(_ptr(status), _ptr(ok), ctypes.c_uint64(int(limit_ns)), 1 if arrive else 0,
                                          _stream(status.device)))
    return ok


def kv_stream_read(src: torch.Tensor, nbytes: int, sink: torch.Tensor) -> None:
    """Reads the first nbytes of src once with a plain streaming kernel (a
    measurement reference: the time one launch needs to move that many bytes)."""
    _need(sink, "sink", torch.int32)
    if nbytes > src.numel() * src.element_size():
        raise ValueError("nbytes exceeds the tensor")
    _check(lib().kv_stream_read(_ptr(src), ctypes.c_size_t(int(nbytes)), _ptr(sink), _stream(src.device)))


def kv_build_wildcat_coreset(K: torch.Tensor, seq_lens: torch.Tensor, scale: float, m: int, u: torch.Tensor,
                             workspace: Optional[torch.Tensor] = None, ctas_per_pair: int = 0):
    """Weighted coreset of every (sequence, KV head)'s keys by randomly pivoted
    Cholesky with kernel-distance weights. u: [B][Hkv][m] fp32 uniforms in (0, 1)
    on the device; ctas_per_pair: CTAs per pair (0: min(8, SMs / pairs)). Returns (tok_idx [B][Hkv][m] int32, w [B][Hkv][m] fp32, n_sel
    [B][Hkv] int32) for kv_sparse_decode_attn(tok_idx=..., w=...)."""
    _need(K, "K")
    _need(u, "u", torch.float32)
    B, Hkv, Ncap, D = K.shape
    shape = KVShape(B, Hkv, Hkv, D, Ncap, 64, _dtype_code(K.dtype), seq_lens.data_ptr())
    need = int(lib().kv_wildcat_workspace_bytes(ctypes.byref(shape), int(m)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=K.device)
    tok_idx = torch.zeros(B, Hkv, m, dtype=torch.int32, device=K.device)
    w = torch.zeros(B, Hkv, m, dtype=torch.float32, device=K.device)
    n_sel = torch.zeros(B, Hkv, dtype=torch.int32, device=K.device)
    _check(lib().kv_build_wildcat_coreset(ctypes.byref(shape), _ptr(K), float(scale), int(m), int(ctas_per_pair),
                                          _ptr(u), _ptr(tok_idx),
                                          _ptr(w), _ptr(n_sel), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(K.device)))
    return tok_idx, w, n_sel


# ----------------------------------------------------------------- stored second-order descriptor
def kv_build_query_basis(Qc: torch.Tensor, Hkv: int):
    """Eigenvectors (rows, [Hkv][D][D] fp32) and descending eigenvalues ([Hkv][D]) of
    each KV head's query second moment over calibration queries Qc [Nc][Hq][D]."""
    _need(Qc, "Qc")
    Nc, Hq, D = Qc.shape
    dev = Qc.device
    evecs = torch.empty(Hkv, D, D, dtype=torch.float32, device=dev)
    evals = torch.empty(Hkv, D, dtype=torch.float32, device=dev)
    need = int(lib().kv_query_basis_workspace_bytes(int(Hkv), int(D)))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().kv_build_query_basis(_ptr(Qc), _dtype_code(Qc.dtype), int(Nc), int(Hq), int(Hkv), int(D),
                                      _ptr(evecs), _ptr(evals), _ptr(ws), ws.numel(), _stream(dev)))
    return evecs, evals


def kv_query_subspace_rank(evals: torch.Tensor, energy: float = 0.9) -> int:
    """s from the basis eigenvalues [Hkv][D] (copied to the host for the library's
    host function)."""
    ev = evals.detach().to("cpu", torch.float32).contiguous()
    Hkv, D = ev.shape
    s = int(lib().kv_query_subspace_rank(ctypes.c_void_p(ev.data_ptr()), int(Hkv), int(D), float(energy)))
    if s < 0:
        raise KVError(KV_ERR_INVALID_ARG, "kv_query_subspace_rank: bad arguments")
    return s


def kv_build_block_cov_factors_ss(K: torch.Tensor, seq_lens: torch.Tensor, block_size: int, U: torch.Tensor,
                                  rank: int = 4, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per-block factors of the covariance within the subspace of U [Hkv][s][D]:
    [B][Hkv][NB][rank][SP] fp32, SP = s rounded up to 32 (zero past s)."""
    _need(K, "K")
    _need(seq_lens, "seq_lens", torch.int32)
    _need(U, "U", torch.float32)
    B, Hkv, Ncap, D = K.shape
    s = int(U.shape[1])
    SP = (s + 31) // 32 * 32
    NB = (Ncap + block_size - 1) // block_size
    if out is None:
        out = torch.empty(B, Hkv, NB, rank, SP, dtype=torch.float32, device=K.device)
    shape = KVShape(B, Hkv, Hkv, D, Ncap, block_size, _dtype_code(K.dtype), seq_lens.data_ptr())
    _check(lib().kv_build_block_cov_factors_ss(ctypes.byref(shape), _ptr(K), _ptr(U), s, int(rank), _ptr(out),
                                               _stream(K.device)))
    return out


def kv_quantize_fp4(x: torch.Tensor):
    """E2M1 codes of the vectors along x's last axis (a multiple of 32 long) with one
    fp32 scale each: (codes uint8 [..., len / 2], scales fp32 [...])."""
    _need(x, "x", torch.float32)
    length = int(x.shape[-1])
    nvec = x.numel() // length if length else 0
    codes = torch.empty(*x.shape[:-1], length // 2, dtype=torch.uint8, device=x.device)
    scales = torch.empty(*x.shape[:-1], dtype=torch.float32, device=x.device)
    _check(lib().kv_quantize_fp4(_ptr(x), int(nvec), length, _ptr(codes), _ptr(scales), _stream(x.device)))
    return codes, scales


def kv_select_blocks_cobs_fp4(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor, block_size: int,
                              scale: float, k_mean: torch.Tensor, counts: torch.Tensor, U: Optional[torch.Tensor],
                              codes: torch.Tensor, code_scales: torch.Tensor, rank: int, k_top: int,
                              force_first: bool = False, force_last: bool = False, kmax: Optional[int] = None,
                              block_idx: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                              scores: Optional[torch.Tensor] = None, want_scores: bool = False):
    """Kept blocks per KV head scored with the stored second-order descriptor (bf16
    means, E2M1 factors, the query subspace of U or the full space when U is None).
    Returns (block_idx [B][Hkv][kmax], n_kept [B][Hkv], scores or None)."""
    _need(q, "q", torch.bfloat16)
    _need(k_mean, "k_mean", torch.bfloat16)
    _need(counts, "counts", torch.int32)
    _need(codes, "codes", torch.uint8)
    _need(code_scales, "code_scales", torch.float32)
    if U is not None:
        _need(U, "U", torch.float32)
    shape = make_shape(q, K, seq_lens, block_size)
    s = int(U.shape[1]) if U is not None else shape.D
    NB = (shape.Ncap + block_size - 1) // block_size
    forced = int(bool(force_first)) + int(bool(force_last))
    if kmax is None:
        kmax = max(1, min(NB, k_top + forced))
    dev = q.device
    if block_idx is None:
        block_idx = torch.zeros(shape.B, shape.Hkv, kmax, dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.zeros(shape.B, shape.Hkv, dtype=torch.int32, device=dev)
    if scores is None and want_scores:
        scores = torch.empty(shape.B, shape.Hkv, NB, dtype=torch.float32, device=dev)
    _check(lib().kv_select_blocks_cobs_fp4(ctypes.byref(shape), _ptr(q), float(scale), _ptr(k_mean), _ptr(counts),
                                           _ptr(U), s, _ptr(codes), _ptr(code_scales), int(rank), int(k_top),
                                           int(bool(force_first)), int(bool(force_last)), int(kmax),
                                           _ptr(block_idx), _ptr(n_kept), _ptr(scores), _stream(dev)))
    return block_idx, n_kept, scores


# ----------------------------------------------------------------- query-guided clusters
def kv_build_qgc(K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor, P: torch.Tensor, C: int = 32,
                 iters: int = 8) -> dict:
    """Clusters of every (sequence, KV head)'s keys in the projection P [Hkv][16][D]
    and their cached mean and variance tokens (once after prefill)."""
    _need(K, "K")
    _need(V, "V", K.dtype)
    _need(P, "P", torch.float32)
    B, Hkv, Ncap, D = K.shape
    dev = K.device
    shape = KVShape(B, Hkv, Hkv, D, Ncap, 64, _dtype_code(K.dtype), seq_lens.data_ptr())
    out = dict(
        C=int(C),
        z16=torch.empty(B, Hkv, Ncap, 16, dtype=torch.bfloat16, device=dev),
        labels=torch.empty(B, Hkv, Ncap, dtype=torch.int32, device=dev),
        perm=torch.empty(B, Hkv, Ncap, dtype=torch.int32, device=dev),
        offs=torch.empty(B, Hkv, C + 1, dtype=torch.int32, device=dev),
        counts=torch.empty(B, Hkv, C, dtype=torch.int32, device=dev),
        k_sum=torch.empty(B, Hkv, C, D, dtype=torch.float32, device=dev),
        v_sum=torch.empty(B, Hkv, C, D, dtype=torch.float32, device=dev),
        k_sq=torch.empty(B, Hkv, C, D, dtype=torch.float32, device=dev),
    )
    ws = torch.empty(max(16, int(lib().kv_qgc_workspace_bytes(ctypes.byref(shape)))), dtype=torch.uint8, device=dev)
    _check(lib().kv_build_qgc(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(P), int(C), int(iters), _ptr(out["z16"]),
                              _ptr(out["labels"]), _ptr(out["perm"]), _ptr(out["offs"]), _ptr(out["counts"]),
                              _ptr(out["k_sum"]), _ptr(out["v_sum"]), _ptr(out["k_sq"]), _ptr(ws), ws.numel(),
                              _stream(dev)))
    return out


def kv_select_qgc(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                  P: torch.Tensor, qgc: dict, budget: float, max_read: Optional[int] = None,
                  workspace: Optional[torch.Tensor] = None, out: Optional[tuple] = None):
    """Error-gated read list and cluster proxies for one decode step. Returns
    (tok_idx, w, n_read, proxy_k, proxy_v, proxy_n) (written into `out` when given)."""
    _need(q, "q", K.dtype)
    B, Hkv, Ncap, D = K.shape
    Hq = q.shape[1]
    C = qgc["C"]
    dev = q.device
    if max_read is None:
        max_read = max(1, int(math.floor(budget * Ncap)))
    shape = KVShape(B, Hq, Hkv, D, Ncap, 64, _dtype_code(K.dtype), seq_lens.data_ptr())
    if out is not None:
        tok_idx, w, n_read, pk, pv, pn = out
        max_read = int(tok_idx.shape[-1])
    else:
        tok_idx = torch.empty(B, Hkv, max_read, dtype=torch.int32, device=dev)
        w = torch.empty(B, Hkv, max_read, dtype=torch.float32, device=dev)
        n_read = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
        pk = torch.empty(B, Hkv, C, D, dtype=torch.float32, device=dev)
        pv = torch.empty(B, Hkv, C, D, dtype=torch.float32, device=dev)
        pn = torch.empty(B, Hkv, C, dtype=torch.int32, device=dev)
    need = int(lib().kv_qgc_select_workspace_bytes(ctypes.byref(shape)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(16, need), dtype=torch.uint8, device=dev)
    _check(lib().kv_select_qgc(ctypes.byref(shape), _ptr(q), float(scale), _ptr(P), int(C), _ptr(qgc["z16"]),
                               _ptr(qgc["perm"]), _ptr(qgc["offs"]), _ptr(qgc["counts"]), _ptr(qgc["k_sum"]),
                               _ptr(qgc["v_sum"]), _ptr(qgc["k_sq"]), _ptr(K), _ptr(V), float(budget), int(max_read),
                               _ptr(tok_idx), _ptr(w), _ptr(n_read), _ptr(pk), _ptr(pv), _ptr(pn), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(dev)))
    return tok_idx, w, n_read, pk, pv, pn


def kv_merge_qgc_proxies(q: torch.Tensor, K: torch.Tensor, seq_lens: torch.Tensor, scale: float, C: int,
                         proxy_k: torch.Tensor, proxy_v: torch.Tensor, proxy_n: torch.Tensor, out: torch.Tensor,
                         lse: torch.Tensor) -> None:
    """Folds the cluster proxies into out / lse in place."""
    B, Hkv, Ncap, D = K.shape
    shape = KVShape(B, q.shape[1], Hkv, D, Ncap, 64, _dtype_code(K.dtype), seq_lens.data_ptr())
    _check(lib().kv_merge_qgc_proxies(ctypes.byref(shape), _ptr(q), float(scale), int(C), _ptr(proxy_k),
                                      _ptr(proxy_v), _ptr(proxy_n), _ptr(out), _ptr(lse), _stream(q.device)))


def qgc_decode(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_lens: torch.Tensor, scale: float,
               P: torch.Tensor, qgc: dict, budget: float, ws: "Workspace", out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, sel_workspace: Optional[torch.Tensor] = None,
               sel_out: Optional[tuple] = None):
    """One decode step: the error-gated read list, attention over it (weighted mode,
    weights 1) and the proxies folded in. Returns (out, lse, selection tuple)."""
    sel = kv_select_qgc(q, K, V, seq_lens, scale, P, qgc, budget, workspace=sel_workspace, out=sel_out)
    tok_idx, w = sel[0], sel[1]
    out, lse = kv_sparse_decode_attn(q, K, V, seq_lens, 64, scale, ws, tok_idx=tok_idx, w=w, out=out, lse=lse)
    kv_merge_qgc_proxies(q, K, seq_lens, scale, qgc["C"], sel[3], sel[4], sel[5], out, lse)
    return out, lse, sel
