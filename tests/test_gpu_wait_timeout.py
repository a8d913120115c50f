"""Failure detection on the device, without a fault: the bounded wait every
kernel uses on its copies gives up, flags KV_DEV_WAIT_TIMEOUT and returns when
the bytes it waits for never arrive (a barrier armed for 16 bytes with no copy
issued), and completes normally when the barrier's phase does complete."""
import time

import pytest
import torch

import weighted_coreset_softmax_b200 as kv

KV_DEV_WAIT_TIMEOUT = 0x10


@pytest.mark.gpu
@pytest.mark.parametrize("limit_us", [5, 200])
def test_wait_runs_out_and_flags(limit_us):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    ok = kv.kv_selftest_wait_timeout(status, limit_us * 1000, arrive=False)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(ok.item()) == 0, "the wait must give up"
    assert int(status.item()) & KV_DEV_WAIT_TIMEOUT
    assert dt < 5.0
    # the context is still usable after the timed-out wait
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2


@pytest.mark.gpu
def test_wait_completes_without_flag():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ok = kv.kv_selftest_wait_timeout(status, 1_000_000, arrive=True)
    torch.cuda.synchronize()
    assert int(ok.item()) == 1
    assert int(status.item()) == 0


@pytest.mark.gpu
def test_wait_keeps_other_status_bits():
    status = torch.full((1,), 0x4, dtype=torch.int32, device="cuda")
    kv.kv_selftest_wait_timeout(status, 2000, arrive=False)
    torch.cuda.synchronize()
    assert int(status.item()) == 0x4 | KV_DEV_WAIT_TIMEOUT


def test_wait_selftest_rejects_bad_limits():
    import ctypes
    L = kv.lib()
    dummy = ctypes.c_void_p(256)
    assert L.kv_selftest_wait_timeout(dummy, dummy, ctypes.c_uint64(0), 0, None) == kv.KV_ERR_INVALID_ARG
    assert L.kv_selftest_wait_timeout(dummy, dummy, ctypes.c_uint64(3 * 10**9), 0, None) == kv.KV_ERR_INVALID_ARG
    assert L.kv_selftest_wait_timeout(None, dummy, ctypes.c_uint64(1000), 0, None) == kv.KV_ERR_INVALID_ARG
