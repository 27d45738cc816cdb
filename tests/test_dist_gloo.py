"""Multi-rank host logic of the benchmark, on CPU with the gloo backend (world size 2).

With N GPUs every rank decodes its own independent batch of the same shape
(weak scaling, no collective on the data path).  What has to be right on the
host: each rank draws different values, the job is timed by its slowest rank,
and the whole-job throughput counts every rank's bytes.  The reference arm
runs on rank 0 only.
"""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        assert b.dist_env() == (rank, world, rank)
        # every rank reports its own time; the job takes the slowest
        local_ms = [12.5, 20.0][rank]
        ms = b.max_over_ranks(local_ms, world, torch.device("cpu"))
        # per-rank seeds differ, so ranks decode different batches
        seeds = [None] * world
        dist.all_gather_object(seeds, [b.rank_value_seed(479002, rank, r) for r in range(2)])
        value = b.job_throughput(1_000_000, world, ms, 10)
        q.put((rank, ms, seeds, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_timing_and_throughput_with_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=100)
    codes = [p.exitcode for p in procs]
    assert codes == [0, 0], codes
    results = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, seeds, value in results:
        assert ms == 20.0                      # max over ranks
        flat = [s for per in seeds for s in per]
        assert len(set(flat)) == len(flat)     # no two batches share a seed
        # 2 ranks x 1 MB per step, 10 steps in 20 ms -> 1 GB/s
        assert value == pytest.approx(1.0)


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert b.job_throughput(2e9, 1, 1000.0, 1) == pytest.approx(2.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    b = _bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload, steps, warmup, gpus, ref_seconds = 2, 1, 0, 2, 1.0
    assert b.run_reference(Args()) is None
    assert capsys.readouterr().out == ""
