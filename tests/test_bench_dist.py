"""CPU check of the multi-rank bench plumbing with two gloo ranks: the job's
time is the slowest replica's, and the value counts every rank's bytes."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + 5.0 * rank, 20.0 - 3.0 * rank]   # rank-dependent timings
        q.put((rank, bench.max_over_ranks(mine)))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks_and_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert got[0] == got[1] == [15.0, 20.0]
    import bench
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]       # no process group: identity
    # two replicas, 1 GB each per run, slowest rank 2 ms -> 1000 GB/s for the job
    assert bench.job_value(2, 1e9, 2.0) == pytest.approx(1000.0)


def test_source_hash_ignores_comments_only():
    """The hash that ties a recorded ncu traffic figure to the kernel sources
    changes with the code, not with comments."""
    import bench
    a = "int a = 1;  // one\n/* block\n comment */\nconst char* s = \"//kept\";\n"
    b = "int a = 1;\n\nconst char* s = \"//kept\";  /* other */\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only("int a = 2;") != bench._code_only("int a = 1;")
    assert "//kept" in bench._code_only(a)
