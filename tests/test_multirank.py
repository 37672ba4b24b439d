"""Multi-rank host logic of bench.py on CPU: two gloo processes (no GPU).

bench.py runs N independent replicas; the only cross-rank steps are the barrier, the
max-over-ranks step time and the whole-job throughput, and the reference arm runs on rank 0
alone. These are exercised here with world size 2 over gloo on 127.0.0.1.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_dir):
    import datetime
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t_max = bench.max_over_ranks(times[rank], dist, "cpu")
        value = bench.job_value(1.0e9, world, t_max)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{t_max!r} {value!r}\n")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo(tmp_path):
    world, times = 2, [3.25, 7.5]
    mp.spawn(_worker, args=(world, _free_port(), times, str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        t_max, value = (float(v) for v in (tmp_path / f"rank{r}.txt").read_text().split())
        assert t_max == max(times)                        # every rank sees the slowest rank's time
        assert value == pytest.approx(1.0e9 * world / (max(times) * 1e-3) / 1e9)


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks(2.5, None, "cpu") == 2.5
    assert bench.job_value(2.0e9, 1, 1.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    import argparse
    import bench
    args = argparse.Namespace(steps=1, warmup=0, cpu_sample_rows=2)
    assert bench.run_reference(args, rank=1, world=2) is None      # other ranks do no work
    line = bench.run_reference(args, rank=0, world=2)
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
