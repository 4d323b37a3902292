"""The multi-GPU form of the benchmark is N independent replicas (the layer has no
exchange step): the host logic that joins them -- rank/world parsing, the slowest
rank's time as the job's time, whole-job throughput -- runs here as two gloo ranks
on the CPU."""

import datetime
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_env()
        ms = bench.max_over_ranks(2.0 + 3.0 * rank, torch, "cpu", w)  # rank 1 is the slow one
        rate = bench.whole_job_rate(4096, w, ms)
        dist.barrier()
        out.put((rank, w, r, local, ms, rate))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_whole_job_rate():
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
    for rank, (r0, w, r, local, ms, rate) in enumerate(res):
        assert (r0, w, r, local) == (rank, 2, rank, rank)
        assert ms == 5.0  # the max over ranks, seen by every rank
        assert rate == 4096 * 2 / 5e-3  # all ranks' tokens over the slowest rank's time
