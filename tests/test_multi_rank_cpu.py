"""The multi-replica path of bench.py on CPU: two gloo ranks.

The step shards by request, so a multi-GPU run is independent replicas
whose figures are combined once: times by the max over ranks, committed
tokens by the sum. These tests run that combination with two real gloo
ranks and check that the reference arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out_path):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        # rank r: step times 10 + r and 3 - r ms, tokens 100 * (r + 1) and 7
        times, toks = bench.reduce_over_ranks([10.0 + rank, 3.0 - rank], [100 * (rank + 1), 7], ws,
                                              "cpu")
        if rank == 0:
            with open(out_path, "w") as f:
                json.dump({"times": times, "tokens": toks}, f)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    out = tmp_path / "r.json"
    mp.spawn(_rank_main, args=(2, _free_port(), str(out)), nprocs=2, join=True)
    got = json.loads(out.read_text())
    assert got["times"] == [11.0, 3.0]           # max over ranks
    assert got["tokens"] == [300.0, 14.0]        # sum over ranks


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    times, toks = bench.reduce_over_ranks([2.5], [9], 1, "cpu")
    assert times == [2.5] and toks == [9.0]


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_prints_the_gpu_arms_metric_and_config():
    """Both arms describe the same workload: the reference line's metric,
    unit, direction and config are the ones the GPU arm prints."""
    sys.path.insert(0, ROOT)
    import bench
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.metric_name("tiny")
    assert line["config"] == bench.workload_config("tiny", 1)
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["e2e"]["value"] == line["value"] == line["cpu_baseline"]["value"]
    head = bench.workload_config("qwen3_8b_b64", 1)
    assert head["global_batch"] == 64 and head["rows_per_step"] == 448
    assert head["l2"].startswith("inputs larger than L2")
