"""The C ABI on the host: the library loads, exports every function the header
declares, and rejects bad arguments before any CUDA call (no GPU needed)."""
import ctypes
import subprocess

import pytest

import weighted_coreset_softmax_b200 as kv

FAKE = 0x7f0000100000  # 256-byte aligned address; never dereferenced by these calls


def _shape(**kw):
    d = dict(B=2, Hq=32, Hkv=8, D=128, Ncap=4096, block_size=64, dtype=kv.KV_BF16, seq_lens=FAKE)
    d.update(kw)
    return kv.KVShape(d["B"], d["Hq"], d["Hkv"], d["D"], d["Ncap"], d["block_size"], d["dtype"],
                      d["seq_lens"])


def test_exports_every_declared_function():
    names = kv.header_functions()
    for want in ("kv_build_block_summaries", "kv_select_blocks", "kv_sparse_decode_attn",
                 "kv_dense_decode_attn", "kv_workspace_bytes", "kv_workspace_init",
                 "kv_workspace_status", "kv_last_error"):
        assert want in names
    L = kv.lib()
    for n in names:
        assert getattr(L, n) is not None
    out = subprocess.run(["nm", "-D", "--defined-only", kv.library_path()], capture_output=True,
                         text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing


def test_workspace_bytes():
    L = kv.lib()
    assert L.kv_workspace_bytes(None) == 0
    a = L.kv_workspace_bytes(ctypes.byref(_shape()))
    b = L.kv_workspace_bytes(ctypes.byref(_shape(B=4)))
    c = L.kv_workspace_bytes(ctypes.byref(_shape(Hq=64)))
    assert 0 < a < b and a < c and a % 256 == 0


def _dense(shape, q=FAKE, K=FAKE, V=FAKE, out=FAKE, lse=None, ws=FAKE, nbytes=1 << 30):
    L = kv.lib()
    return L.kv_dense_decode_attn(ctypes.byref(shape) if shape is not None else None, q, 0.1, K, V, out,
                                  lse, ws, nbytes, None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(D=96), kv.KV_ERR_UNSUPPORTED, "head dim"),
    (dict(Hq=72, Hkv=8), kv.KV_ERR_UNSUPPORTED, "group size"),
    (dict(Hq=30, Hkv=8), kv.KV_ERR_INVALID_ARG, "multiple"),
    (dict(block_size=48), kv.KV_ERR_UNSUPPORTED, "block_size"),
    (dict(Ncap=64 * 4097), kv.KV_ERR_UNSUPPORTED, "NBcap"),
    (dict(B=-1), kv.KV_ERR_INVALID_ARG, "B ="),
    (dict(Ncap=0), kv.KV_ERR_INVALID_ARG, "Ncap"),
    (dict(dtype=7), kv.KV_ERR_INVALID_ARG, "dtype"),
    (dict(seq_lens=None), kv.KV_ERR_INVALID_ARG, "seq_lens"),
    (dict(seq_lens=FAKE + 2), kv.KV_ERR_INVALID_ARG, "seq_lens"),
])
def test_bad_shapes(kw, status, msg):
    assert _dense(_shape(**kw)) == status
    assert msg in kv.kv_last_error()


def test_bad_pointers_and_sizes():
    s = _shape()
    assert _dense(None) == kv.KV_ERR_INVALID_ARG
    assert _dense(s, q=None) == kv.KV_ERR_INVALID_ARG and "q is NULL" in kv.kv_last_error()
    assert _dense(s, K=FAKE + 8) == kv.KV_ERR_INVALID_ARG and "aligned" in kv.kv_last_error()
    assert _dense(s, ws=FAKE + 16) == kv.KV_ERR_INVALID_ARG
    assert _dense(s, nbytes=1024) == kv.KV_ERR_INVALID_ARG and "workspace" in kv.kv_last_error()
    L = kv.lib()
    # selection: kmax below k_top + forced blocks
    st = L.kv_select_blocks(ctypes.byref(s), FAKE, 0.1, kv.KV_SCORE_SUMMARY, FAKE, FAKE, None, 5, 1, 1,
                            6, FAKE, FAKE, None, None)
    assert st == kv.KV_ERR_INVALID_ARG and "kmax" in kv.kv_last_error()
    st = L.kv_select_blocks(ctypes.byref(s), FAKE, 0.1, 9, FAKE, FAKE, None, 5, 1, 1, 7, FAKE, FAKE, None,
                            None)
    assert st == kv.KV_ERR_INVALID_ARG
    st = L.kv_select_blocks(ctypes.byref(s), FAKE, 0.1, kv.KV_SCORE_EXACT_MASS, FAKE, FAKE, None, 5, 1, 1,
                            7, FAKE, FAKE, None, None)
    assert st == kv.KV_ERR_INVALID_ARG and "K is NULL" in kv.kv_last_error()
    st = L.kv_select_blocks(ctypes.byref(s), FAKE, float("nan"), 0, FAKE, FAKE, None, 5, 1, 1, 7, FAKE,
                            FAKE, None, None)
    assert st == kv.KV_ERR_INVALID_ARG and "scale" in kv.kv_last_error()
    # sparse attention: proxy needs the summaries; kmax beyond NBcap
    st = L.kv_sparse_decode_attn(ctypes.byref(s), FAKE, 0.1, FAKE, FAKE, FAKE, FAKE, 7, None, None, None,
                                 None, None, 1, None, None, 0, FAKE, None, FAKE, 1 << 30, None)
    assert st == kv.KV_ERR_INVALID_ARG and "k_sum" in kv.kv_last_error()
    st = L.kv_sparse_decode_attn(ctypes.byref(s), FAKE, 0.1, FAKE, FAKE, FAKE, FAKE, 65, FAKE, FAKE, FAKE,
                                 FAKE, FAKE, 1, None, None, 0, FAKE, None, FAKE, 1 << 30, None)
    assert st == kv.KV_ERR_INVALID_ARG and "kmax" in kv.kv_last_error()
    # weighted mode: negative m, missing weights
    st = L.kv_sparse_decode_attn(ctypes.byref(s), FAKE, 0.1, FAKE, FAKE, None, None, 0, None, None, None,
                                 None, None, 0, FAKE, FAKE, -1, FAKE, None, FAKE, 1 << 30, None)
    assert st == kv.KV_ERR_INVALID_ARG and "m =" in kv.kv_last_error()
    st = L.kv_sparse_decode_attn(ctypes.byref(s), FAKE, 0.1, FAKE, FAKE, None, None, 0, None, None, None,
                                 None, None, 0, FAKE, None, 4, FAKE, None, FAKE, 1 << 30, None)
    assert st == kv.KV_ERR_INVALID_ARG and "w is NULL" in kv.kv_last_error()
    # summaries and workspace helpers
    st = L.kv_build_block_summaries(ctypes.byref(s), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None)
    assert st == kv.KV_ERR_INVALID_ARG and "v_sum" in kv.kv_last_error()
    assert L.kv_workspace_init(None, 4096, None) == kv.KV_ERR_INVALID_ARG
    v = ctypes.c_uint32(0)
    assert L.kv_workspace_status(FAKE, None, None) == kv.KV_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op():
    assert _dense(_shape(B=0, seq_lens=None)) == kv.KV_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import weighted_coreset_softmax_b200 as pkg
    monkeypatch.setattr(pkg, "_lib", None)
    monkeypatch.setattr(pkg, "library_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        pkg.lib()
