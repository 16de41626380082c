"""The N > 1 path of bench.py on CPU: world-size-2 gloo process groups.

The linear has no exchange step, so N GPUs run N independent replicas; what
the ranks share is the barrier, the max-over-ranks device time and the
aggregate throughput.  These tests run that logic as two gloo ranks on the
host, and check that the reference arm runs on rank 0 alone.
"""
import io
import json
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    sys.path.insert(0, ROOT)
    import datetime

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        tops = bench.aggregate_tops(world, 1.0e12, 10, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "tops": tops}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo(tmp_path):
    world = 2
    times = [12.5, 20.0]
    mp.start_processes(_rank_main, args=(world, _free_port(), times, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["ms"] == max(times)
        # 2 replicas x 1e12 ops x 10 steps over the slowest rank's 20 ms
        assert r["tops"] == pytest.approx(2 * 1e12 * 10 / 0.020 / 1e12)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    assert bench.aggregate_tops(1, 2.0e12, 4, 8.0) == pytest.approx(2.0e12 * 4 / 0.008 / 1e12)


def test_reference_arm_only_rank0_works(oracle):
    sys.path.insert(0, ROOT)
    import bench

    args = types.SimpleNamespace(workload="small", steps=2, warmup=1, gpus=2)
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, rank=1, world=2) == 0
    assert buf.getvalue() == ""
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, rank=0, world=2) == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == "small"
