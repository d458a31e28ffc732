"""The multi-GPU path on CPU: two gloo ranks run the benchmark's rank logic.

On one node the path shards by (batch, head) with no data-path collective.
Each rank gets its own seeded shard, the step time is the maximum over ranks,
and the reported value is the whole job's work over that time. These host
parts are what differ at N > 1, and they are checked here with world size 2."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(workloads.C5, rank)
        elapsed = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        q, _, _, _ = workloads.make_inputs(
            workloads.small("shard", 1, 2, 2, 16, 64, True, seed=w.seed))
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"seed": w.seed, "elapsed": elapsed,
                       "q0": float(q.float().flatten()[0])}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(2)]
    assert r[0]["seed"] != r[1]["seed"]                 # distinct data shards
    assert r[0]["q0"] != r[1]["q0"]
    assert r[0]["elapsed"] == r[1]["elapsed"] == 15.0   # max over ranks on every rank


def test_job_throughput_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_throughput(1e12, 10, 1, 1000.0)
    assert one == pytest.approx(10.0)
    assert bench.job_throughput(1e12, 10, 4, 1000.0) == pytest.approx(40.0)
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
