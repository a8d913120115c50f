import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Builds libkvsparse.so in-tree when it is missing or older than its sources
    (nvcc cross-compiles for sm_100a without a GPU)."""
    from weighted_coreset_softmax_b200 import build
    build.build()
    yield


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Reports the near ties of the selection checks: pairs checked, pairs whose
    k-th and (k+1)-th oracle scores lie within the near-tie band, and pairs whose
    GPU kept set differs from the oracle's there (allowed, reported)."""
    try:
        from gpu_helpers import NEAR_TIES, NOTES
    except Exception:  # noqa: BLE001 -- no GPU helpers imported in this session
        return
    tr = terminalreporter
    if NOTES:
        tr.section("reported figures")
        for line in NOTES:
            tr.write_line(line)
    if not NEAR_TIES:
        return
    tr.section("selection near ties (allowed mismatches, reported)")
    tot = [0, 0, 0]
    for what, n, f, m in NEAR_TIES:
        tot[0] += n
        tot[1] += f
        tot[2] += m
        if f or m:
            tr.write_line(f"{what}: {n} pairs, {f} flagged near ties, {m} kept sets differ at a near tie")
    tr.write_line(f"total: {tot[0]} pairs checked, {tot[1]} flagged near ties, {tot[2]} near-tie mismatches "
                  f"(a mismatch outside a near tie fails its test)")
