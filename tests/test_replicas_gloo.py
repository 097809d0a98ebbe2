"""The N > 1 path of bench.py is "replicas only": every rank runs an
independent copy of the step and the job's time is the slowest rank's.  Two
gloo ranks on the CPU check the aggregation (no GPU)."""
import datetime
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r took 1 + r ms for 1 GB of algorithmic bytes
        ms_max, tbs = bench.replica_throughput(1.0 + rank, 1e9, dist)
        out[rank] = (ms_max, tbs)
    finally:
        dist.destroy_process_group()


def test_replica_throughput_two_gloo_ranks():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        ms_max, tbs = out[r]
        assert ms_max == 2.0  # the slowest rank
        assert abs(tbs - 2 * 1e9 / 2e-3 / 1e12) < 1e-12  # bytes of both ranks / slowest time


def test_replica_throughput_single_process():
    import bench
    ms_max, tbs = bench.replica_throughput(4.0, 2e9)
    assert ms_max == 4.0 and abs(tbs - 0.5) < 1e-12
