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
