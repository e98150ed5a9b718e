"""The N > 1 path of bench.py on CPU: two ranks on the gloo backend (one process each, started
with spawn).  The path shards independent problems over ranks (replicas, weak scaling), so the
only exchange is the timing reduction: the job's step time is the slowest rank's, and the job's
throughput is every rank's work over that time.  Each rank draws its own inputs (seed + rank)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports (total, attention, quantize) sums; rank 1 is the slow one in total
        # and attention, rank 0 in quantize
        mine = [10.0 + 5.0 * rank, 8.0 + 5.0 * rank, 2.0 - rank]
        got = bench.max_over_ranks(mine, world, "cpu")
        # each rank's inputs: the workload's generator with its own seed
        w = wl.WORKLOADS["int8_tiny"].scaled(seed=wl.WORKLOADS["int8_tiny"].seed + rank)
        q = wl.make_inputs(w, calib=False)["q"]
        torch.save({"got": got, "q": q}, os.path.join(out_dir, f"rank{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank_and_distinct_inputs(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r0 = torch.load(tmp_path / "rank0.pt")
    r1 = torch.load(tmp_path / "rank1.pt")
    assert r0["got"] == r1["got"] == [15.0, 13.0, 2.0]
    assert not torch.equal(r0["q"], r1["q"])


def test_job_value_is_weak_scaling_over_the_slowest_rank():
    # one rank: 1e12 FLOP per step in 2 ms -> 500 TFLOP/s; two ranks, each with its own 1e12,
    # and the slower rank taking 2 ms -> 1000 TFLOP/s
    assert bench.job_value(1e12, 2.0, 1, "TFLOP/s") == pytest.approx(500.0)
    assert bench.job_value(1e12, 2.0, 2, "TFLOP/s") == pytest.approx(1000.0)
    assert bench.job_value(1e9, 1.0, 4, "GB/s") == pytest.approx(4000.0)
    assert bench.max_over_ranks([1, 2, 3], 1, "cpu") == [1.0, 2.0, 3.0]
