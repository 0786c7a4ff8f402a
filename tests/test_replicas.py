"""Multi-process (replica) path of the benchmark, on CPU with gloo.

The decoder step has no data exchange: N GPUs run N independent videos. What
the N > 1 path adds is host-side: barriers around the timed region, the time
taken as the max over ranks, the work summed over ranks, and the reference arm
running on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    bench.barrier(dist)
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    frames = 7 + rank
    mx = bench.max_over_ranks(dist, ms)
    tot = bench.sum_over_ranks(dist, frames)
    value = bench.replica_throughput(4, tot, mx)
    bench.barrier(dist)
    dist.destroy_process_group()
    q.put((rank, mx, tot, value))


def test_replica_timing_is_max_and_work_is_sum_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, tot, value in res:
        assert mx == 15.0 and tot == 15.0
        assert value == pytest.approx(4 * 15 / 0.015)


def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny_fp32",
           "--gpus", "2", "--steps", "2", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
