"""Host logic of bench.py for N > 1 ranks, on CPU with the gloo backend: rank
set-up from the environment, barriers, the max-over-ranks reduction of the step
time, per-rank seeds (weak scaling), and that a reference-arm rank other than 0
does no work."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    local = 1.0 + 2.5 * rank            # per-rank step time
    mx = d.max(local, torch.device("cpu"))
    seed = bench.shard_seed_offset(rank)
    ref = bench.run_reference(bench.parse_args(["--impl", "reference"]), d) if rank != 0 else "skip"
    d.barrier()
    d.close()
    q.put((rank, mx, seed, ref))


def test_two_rank_max_and_seeds():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [3.5, 3.5]           # max over ranks on every rank
    assert len({r[2] for r in res}) == world            # distinct per-rank seeds
    assert res[1][3] is None                            # reference arm: rank 1 does nothing
