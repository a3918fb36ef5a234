"""The N>1 host logic of the benchmark on CPU: two gloo ranks on 127.0.0.1.
Each rank is an independent replica (the path has no exchange step); the
whole-job throughput is all ranks' tokens over the slowest rank's time, and
the reference arm prints from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        total_ms = 100.0 * (rank + 1)          # rank 1 is the slowest
        value, slowest = bench.aggregate_throughput(dist, 1000, 10, total_ms, cpu)
        m = bench.max_over_ranks(dist, float(rank), cpu)
        q.put((rank, value, slowest, m))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(ws))
    for rank, value, slowest, m in res:
        assert slowest == 200.0                 # max over ranks
        assert m == 1.0
        assert value == pytest.approx(2 * 1000 * 10 / 0.2)   # all tokens / slowest time


def test_reference_arm_rank_zero_only():
    """Under torchrun-style env, rank 1 of the reference arm exits 0 silently."""
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "3", "--warmup", "3", "--workload", "tiny"],
                         capture_output=True, text=True, env=env, cwd=ROOT, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "3", "--warmup", "3", "--workload", "tiny"],
                         capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"]
