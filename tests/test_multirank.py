"""Host logic of the N > 1 bench path on CPU: world-size-2 gloo process group
(the bench's data path has no collective; only the step-time reduction
crosses ranks)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_workload_accounting():
    import bench
    from w4a4_rank_gemm_b200 import synth
    wl = synth.tiny()
    g = bench.groups_of(wl)
    assert [i for i, _ in g] == ["x"]
    assert bench.ops_of(2048, 4096, 4096, 128) == 2.0 * 2048 * 4096 * (4096 + 128)
