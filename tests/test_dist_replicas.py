"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks run
independent replicas; the job time is the max over ranks and the throughput
counts both ranks' work (weak scaling, no data-path collective)."""
import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms_local = [2.0, 5.0][rank]
    ms, rate = bench.aggregate_replicas(ms_local, 1e6, world, dist, "cpu")
    q.put((rank, ms, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_replica_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in res:
        assert ms == 5.0                              # slowest rank
        assert abs(rate - 2 * 1e6 / 5e-3) < 1e-3     # both ranks' units over that time


def test_single_rank_needs_no_collective():
    ms, rate = bench.aggregate_replicas(4.0, 8e6, 1)
    assert ms == 4.0 and rate == 8e6 / 4e-3
