"""Host logic of bench.py's multi-GPU (replicas) path, on CPU with gloo.

Every rank runs one replica of the layer; the whole-job figures are the max
over ranks of the device-timed step and the bytes summed over ranks.  These
tests run that reduction with world size 2 on the gloo backend, and check
that the reference arm does its work on rank 0 alone.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: step 1.0 + r ms, end-to-end 2.0 + 3r ms, 100 (r + 1) bytes
        out = bench.combine_ranks(1.0 + rank, 2.0 + 3 * rank, 100 * (rank + 1), world, "cpu")
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_combine_ranks_single():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(1.5, 2.5, 7, 1, "cpu") == (1.5, 2.5, 7.0)


def test_combine_ranks_gloo_world2():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, out = q.get(timeout=120)
        res[r] = out
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the same whole-job figures
    for r in range(2):
        assert res[r] == (2.0, 5.0, 300.0)


@pytest.mark.parametrize("rank", ["1"])
def test_reference_arm_other_ranks_exit(rank):
    """Under torchrun the reference arm runs on rank 0 only: other ranks
    exit 0 at once with no output."""
    env = dict(os.environ, RANK=rank, WORLD_SIZE="2", LOCAL_RANK=rank)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line():
    """The reference arm (the oracle on the host cores) prints one JSON line
    with the same metric and unit as the GPU arm, plus its CPU baseline and
    an end-to-end figure with no host-device copies."""
    import json
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--T", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == "GB/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["T"] == 2
    # one whole layer per step, and the steps reported are the steps run
    assert d["steps"] == 1 and d["ms_per_step"] > 0
    assert "whole layer" in d["cpu_baseline"]["sample"]
