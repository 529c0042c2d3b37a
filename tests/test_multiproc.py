"""Two-rank gloo test of the multi-GPU host logic of bench.py (no GPU).

Each rank runs the whole decode sweep on its own GPU; the only collectives
are a barrier and the MAX all-reduce of the per-rank step time, and the
reported value is the bytes of all ranks over the slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ms_list, q):
    import sys
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(dist, ms_list[rank], torch.device("cpu"))
        val = bench.weak_value(world, 10 ** 9, ms)
        q.put((rank, ms, val))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_timing_and_weak_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ms_list = [2.0, 5.0]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, ms_list, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, val in res:
        assert ms == 5.0                       # every rank sees the slowest rank's time
        assert val == pytest.approx(2 * 1e9 / 5e-3 / 1e9)


def test_single_process_helpers():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(None, 3.5, None) == 3.5
    assert bench.weak_value(1, 2 * 10 ** 9, 1000.0) == pytest.approx(2.0)
    # algorithmic bytes of one GEMV call: packed + fp16 s,z + X + Y
    assert bench.case_bytes(4, 16384, 16384, 128) == 16384 * 16384 // 2 + 4 * 16384 * 128 + 2 * 4 * 16384 * 2
