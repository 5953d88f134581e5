"""Host-side logic of the multi-GPU benchmark path, run as two gloo ranks on
CPU: per-rank times are reduced to the max over ranks and the whole-job
throughput counts every rank's units (weak scaling, no data-path
collective)."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    t = bench.max_over_ranks(1.0 + rank, world)          # rank 1 is the slow one
    dist.barrier()
    q.put((rank, t, bench.job_throughput(100.0, world, t)))
    dist.destroy_process_group()


def test_two_rank_timing_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, thr in res:
        assert t == 2.0
        assert thr == 2 * 100.0 / 2.0


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(10.0, 1, 2.0) == 5.0
