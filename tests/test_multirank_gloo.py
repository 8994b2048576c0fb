"""The N > 1 plumbing of bench.py on CPU: two gloo ranks, no GPU."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from exact_tiled_attention_36_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, world, "cpu")
        fi = inputs.make_fixed(inputs.TINY, seed=bench.rank_seed(inputs.TINY.seed, rank), Nq=8, Nk=8)
        digest = float(fi.q.float().sum())
        all_d = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(all_d, torch.tensor([digest], dtype=torch.float64))
        q.put((rank, m, [float(x) for x in all_d]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, digests in out:
        assert m == 15.0  # every rank sees the max
        assert digests[0] != digests[1]  # replicas draw independent batches
    # whole-job value: both ranks' work over the slowest rank's time
    assert abs(bench.job_tflops(2, 1e12, 10, 15.0) - 2 * 1e12 * 10 / 0.015 / 1e12) < 1e-9
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
