"""Multi-process (world_size 2, gloo, CPU) checks of bench.py's replica path.

The path does not shard: every rank runs the same step on its own GPU and the
job's time is the slowest rank's.  These tests run the host logic of that
path on CPU ranks: the max-over-ranks reduction every rank must agree on, the
whole-job value built from it, a barrier-bracketed timing on ranks of uneven
speed, and the reference arm's rule that only rank 0 prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime
    import time
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # 1. every rank gets the same maximum
        local = [3.5, 7.25][rank]
        got = bench.max_over_ranks_of(torch, dist, local, "cpu")
        # 2. a barrier-bracketed region on ranks of uneven speed: rank 1 sleeps longer
        dist.barrier()
        t0 = time.perf_counter()
        time.sleep(0.05 * (rank + 1))
        ms_local = (time.perf_counter() - t0) * 1e3
        dist.barrier()
        ms = bench.max_over_ranks_of(torch, dist, ms_local, "cpu")
        value = bench.whole_job_value(world, 1e9, 10, ms, 1e9)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"got": got, "ms_local": ms_local, "ms": ms, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_replica_timing_is_max_over_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    assert r[0]["got"] == r[1]["got"] == 7.25
    # both ranks report the slowest rank's time, and the value is built from it
    assert r[0]["ms"] == r[1]["ms"] == max(r[0]["ms_local"], r[1]["ms_local"])
    assert r[1]["ms_local"] > r[0]["ms_local"]
    expect = world * 1e9 * 10 / (r[0]["ms"] / 1e3) / 1e9
    assert r[0]["value"] == pytest.approx(expect) and r[1]["value"] == pytest.approx(expect)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks_of(torch, None, 1.25, "cpu") == 1.25
    assert bench.whole_job_value(1, 2e9, 4, 2.0, 1e9) == pytest.approx(4000.0)


def test_whole_job_value_scales_with_replicas():
    one = bench.whole_job_value(1, 436879360, 100, 13.65, 1e9)
    eight = bench.whole_job_value(8, 436879360, 100, 13.65, 1e9)
    assert eight == pytest.approx(8 * one)


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "kproj"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1", "--workload", "kproj"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["metric"] == bench.METRIC and line["config"]["key"] == "kproj"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == bench.host_threads()
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
