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
        # the re-measure decision: one rank throttled makes every rank re-measure
        clean = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
        hot = dict(clean, reasons=["hw_thermal_slowdown", "sw_power_cap"])
        throttled = (bench.any_rank_throttled(hot if rank == 1 else clean, world, "cpu"),
                     bench.any_rank_throttled(clean, world, "cpu"),
                     bench.any_rank_throttled(None if rank == 0 else clean, world, "cpu"))
        q.put((rank, m, [float(x) for x in all_d], throttled))
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
    for rank, m, digests, throttled in out:
        assert m == 15.0  # every rank sees the max
        assert digests[0] != digests[1]  # replicas draw independent batches
        assert throttled == (True, False, False)  # the same decision on every rank
    # whole-job value: both ranks' work over the slowest rank's time
    assert abs(bench.job_tflops(2, 1e12, 10, 15.0) - 2 * 1e12 * 10 / 0.015 / 1e12) < 1e-9
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.any_rank_throttled({"reasons": ["sw_thermal_slowdown"]}, 1, "cpu") is True
    assert bench.any_rank_throttled({"reasons": ["sw_power_cap"]}, 1, "cpu") is False


def test_reference_arm_prints_one_line_on_rank_zero_only(monkeypatch, capsys):
    """`bench.py --impl reference` under torchrun: rank 0 times the oracle and prints
    the one JSON line of the contract; every other rank exits 0 without work."""
    import argparse
    import json

    args = argparse.Namespace(gpus=2, steps=2, warmup=1)
    monkeypatch.setattr(bench, "REF_STEP_TOKENS", 64)  # a small sample keeps this test short
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    assert bench.run_reference(args) == 0
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["n_gpus"] == 2 and line["steps"] == 2 and line["warmup"] == 1
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == bench.WORKLOAD["name"] and line["config"]["sample_tokens"] == 64
