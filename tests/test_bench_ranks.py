"""Multi-process plumbing of bench.py on the CPU: world size 2 over gloo.

The decode path shards as independent replicas (no data-path collective); the only
cross-rank steps are the timing reduction (slowest rank's time, all ranks' bytes) and
the reference arm's rule that rank 0 alone runs and prints.
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.25, 5.5][rank]
        nbytes = [1000, 2500][rank]
        got = bench.reduce_over_ranks(dist, ms, nbytes, torch.device("cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(got, f)


def test_reduce_over_ranks_gloo_world2(tmp_path):
    mp.spawn(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        ms_max, bytes_sum = json.load(open(tmp_path / f"rank{r}.json"))
        assert ms_max == 5.5 and bytes_sum == 3500.0, (r, ms_max, bytes_sum)


def test_reduce_over_ranks_single_process():
    import bench
    assert bench.reduce_over_ranks(None, 2.0, 7, torch.device("cpu")) == (2.0, 7.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
