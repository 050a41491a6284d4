"""The benchmark's multi-rank plumbing (replicas, barrier, max over ranks)
on CPU with the gloo backend and world size 2.  The data path has no
collective: each rank runs its own copy of the workload."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    elapsed = 1.0 + rank  # rank 1 is the slow one
    mx = bench.max_over_ranks(elapsed, w)
    val = bench.replica_value(100.0, w, mx)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, mx, val))


def test_two_replicas_take_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, val in res:
        assert mx == 2.0                 # max over ranks
        assert val == pytest.approx(100.0)  # 2 ranks x 100 units / 2 s


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_value(10.0, 1, 2.0) == 5.0
    assert bench.weight_bytes(4096, 4096) == 4096 * 4096 // 2 + 2 * 4096 * 64 + 4 * 4096
    assert bench.gemm_bytes(1, 4096, 4096) == bench.weight_bytes(4096, 4096) + 4096 + 4 + 8192
