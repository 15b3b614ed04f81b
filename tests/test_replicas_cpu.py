"""The N>1 path of bench.py on CPU with gloo, world size 2.

The hot path does not shard: N GPUs run N independent replicas of the layer
step, each on its own token stream, with no data-path collective.  What N>1
adds is host logic: a barrier around the timed region, the slowest rank's
time (max over ranks) for the whole-job rate, and rank 0 alone printing.
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


def _rank_main(rank, world, port, out_path):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    mx = bench.sync_max(world, "cpu", 1.0 + 2.5 * rank)   # rank 1 is the slow one
    mn = bench.sync_max(world, "cpu", 10.0 - rank)        # rank 0 is the slow one
    bench.barrier(world)
    with open(f"{out_path}.{rank}", "w") as f:
        json.dump({"max": mx, "max2": mn, "base": bench.rank_token_base(10_000_000, rank)}, f)
    dist.destroy_process_group()


def test_max_over_ranks_and_disjoint_token_streams(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    out = str(tmp_path / "r")
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    r = [json.load(open(f"{out}.{i}")) for i in range(2)]
    assert r[0]["max"] == r[1]["max"] == 3.5
    assert r[0]["max2"] == r[1]["max2"] == 10.0
    b0, b1 = r[0]["base"], r[1]["base"]
    assert abs(b1 - b0) >= 10_000_000  # streams of fewer than 10^7 tokens never overlap


def test_reference_arm_under_torchrun_prints_once():
    """Two ranks of the reference arm: rank 0 alone runs the oracle and prints
    one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "c0", "--gpus", "2", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
