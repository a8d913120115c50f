"""kv_sparse_decode_attn_noalloc, the entry point for callers that cannot allocate
device memory (its scratch is a fixed array inside the library), must give the
same results as kv_sparse_decode_attn with a caller workspace -- on the first call
and on the next one, which reuses the same array.

Kept in a file of its own that collects last; it builds all of its inputs itself,
so it passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import pytest
import torch

import weighted_coreset_softmax_b200 as kv
from weighted_coreset_softmax_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3  # the output tolerance of the parity tests (max row relative error)


def _noalloc_fn():
    fn = kv.lib().kv_sparse_decode_attn_noalloc
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [ctypes.POINTER(kv.KVShape), P, F, P, P, P, P, I, P, P, P, P, P, I, P, P, I, P, P, P]
    fn.restype = I
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _row_err(a, b):
    a = a.reshape(-1, a.shape[-1]).double()
    b = b.reshape(-1, b.shape[-1]).double()
    return float(((a - b).abs().amax(dim=1) / b.abs().amax(dim=1).clamp_min(1e-30)).max())


def test_noalloc_matches_workspace_entry_point_twice():
    fn = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    # block mode with the tail proxy (ragged lengths, several CTAs per head)
    wl = W.make("llama", DEV, B=3, Ncap=4160, seq_lens=[4160, 3001, 777], budget=0.05)
    sl = wl.seq_lens_tensor(DEV)
    summ = kv.kv_build_block_summaries(wl.K, wl.V, sl, wl.block_size)
    idx, nk, _ = kv.kv_select_blocks(wl.q, wl.K, sl, wl.block_size, wl.scale, summ["counts"], wl.k_top,
                                     True, True, k_sum=summ["k_sum"])
    shape = kv.make_shape(wl.q, wl.K, sl, wl.block_size)
    ws = kv.Workspace(shape, DEV)
    ref_out, ref_lse = kv.kv_sparse_decode_attn(wl.q, wl.K, wl.V, sl, wl.block_size, wl.scale, ws,
                                                block_idx=idx, n_kept=nk, summaries=summ)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = fn(ctypes.byref(shape), _p(wl.q), wl.scale, _p(wl.K), _p(wl.V), _p(idx), _p(nk),
                idx.shape[-1], _p(summ["k_sum"]), _p(summ["v_sum"]), _p(summ["counts"]),
                _p(summ["k_tot"]), _p(summ["v_tot"]), 1, None, None, 0, _p(out), _p(lse), stream)
        assert st == kv.KV_OK, kv.kv_last_error()
        torch.cuda.synchronize()
        assert _row_err(out, ref_out) <= TOL, f"call {call}: out differs"
        assert torch.allclose(lse, ref_lse, rtol=TOL, atol=TOL), f"call {call}: lse differs"

    # weighted-coreset mode, twice
    wc = W.make("llama_coreset", DEV, B=2, Ncap=3000, m=300)
    slc = wc.seq_lens_tensor(DEV)
    shape_c = kv.make_shape(wc.q, wc.K, slc, wc.block_size)
    ws_c = kv.Workspace(shape_c, DEV)
    ref_out, ref_lse = kv.kv_sparse_decode_attn(wc.q, wc.K, wc.V, slc, wc.block_size, wc.scale, ws_c,
                                                tok_idx=wc.tok_idx, w=wc.w)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = fn(ctypes.byref(shape_c), _p(wc.q), wc.scale, _p(wc.K), _p(wc.V), None, None, 0, None, None,
                None, None, None, 0, _p(wc.tok_idx), _p(wc.w), wc.tok_idx.shape[-1], _p(out), _p(lse), stream)
        assert st == kv.KV_OK, kv.kv_last_error()
        torch.cuda.synchronize()
        assert _row_err(out, ref_out) <= TOL, f"weighted call {call}: out differs"
        assert torch.allclose(lse, ref_lse, rtol=TOL, atol=TOL)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    fn = _noalloc_fn()
    sl = torch.full((4096,), 64, dtype=torch.int32, device=DEV)
    shape = kv.KVShape(4096, 64, 8, 128, 64, 64, kv.KV_BF16, sl.data_ptr())
    assert kv.kv_workspace_bytes(shape) > (16 << 20)
    st = fn(ctypes.byref(shape), None, 0.1, None, None, None, None, 1, None, None, None, None, None, 0,
            None, None, 0, None, None, None)
    assert st == kv.KV_ERR_INVALID_ARG
    assert "16 MiB" in kv.kv_last_error()
