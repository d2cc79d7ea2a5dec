"""The multi-GPU path of bench.py is N independent replicas (one per GPU, no
data-path collective): the job's time is the slowest replica's and its
throughput counts every replica's bytes.  The rank logic is checked here with
two gloo processes on the CPU."""
import datetime
import multiprocessing as mp
import os
import socket

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank times a different duration; all must see the largest
        got = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
        again = bench.max_over_ranks(3.0 - rank, "cpu")
        out.put((rank, got, again))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 15.0, 3.0), (1, 15.0, 3.0)]


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(7.5, "cpu") == 7.5


def test_job_throughput_counts_every_replica():
    # two replicas, 1 GB per step each, 10 steps in 1 s: 20 GB/s for the job
    assert bench.job_gbs(2, 1e9, 10, 1000.0) == 20.0
    assert bench.job_gbs(1, 1e9, 10, 1000.0) == 10.0
