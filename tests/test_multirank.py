"""The N > 1 path of bench.py on CPU: two gloo ranks aggregate step time
(max over ranks) and tokens (sum), as the GPU run does over NCCL."""

import os
import socket

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms, tok = bench.aggregate(dist, 10.0 + rank, 8192.0 * 5, None)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, tok))


def test_two_rank_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 11.0, 81920.0), (1, 11.0, 81920.0)]


def test_single_process_aggregate_is_identity():
    import bench
    assert bench.aggregate(None, 3.5, 100.0) == (3.5, 100.0)
