"""The N > 1 host path of bench.py on CPU: two gloo ranks (127.0.0.1).

bench.py under torchrun gives every rank its own full stack (weak scaling, no
collective on the data path).  What crosses ranks is the job's time: the
slowest rank's, by an all-reduce MAX.  The whole-job rate is the units of all
ranks over that time.  These tests run the same helpers over a real gloo process
group.  The reference arm prints on rank 0 only; other ranks leave at once.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 40.0][rank]
        worst = bench.reduce_max(ms, world)
        rate = bench.whole_job_rate(1000, world, worst)
        seeds = {bench.matrix_seed(rank, lid) for lid in range(224)}
        gathered = [None] * world
        dist.all_gather_object(gathered, sorted(seeds))
        class A:
            steps, warmup, gpus = 1, 0, world
        ref_rc = bench.run_reference(A, rank, world) if rank != 0 else 0
        out.put((rank, worst, rate, gathered, ref_rc))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time_and_own_distinct_stacks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, worst, rate, gathered, ref_rc = out.get(timeout=120)
        res[rank] = (worst, rate, gathered, ref_rc)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        worst, rate, gathered, ref_rc = res[rank]
        assert worst == 40.0                       # max over ranks, on every rank
        assert rate == pytest.approx(2 * 1000 / 0.040)
        assert not set(gathered[0]) & set(gathered[1])  # independent stacks
    assert res[1][3] == 0                          # reference arm: rank 1 exits 0, no work
