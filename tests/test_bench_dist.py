"""The multi-process side of bench.py on CPU (gloo, world size 2): each rank
times its own replica, the job time is the maximum over ranks and the value
counts every rank's bytes; the reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = [12.5, 20.0][rank]                    # rank 1 is the slow one
        job_ms = bench.max_over_ranks(ms, world, torch.device("cpu"))
        gbs = bench.job_gbs(1e9, world, 10, job_ms * 1e-3)
        out.put((rank, job_ms, gbs))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(2))
    for rank, job_ms, gbs in got:
        assert job_ms == 20.0, "every rank sees the slowest rank's time"
        # 2 ranks x 10 steps x 1 GB in 20 ms
        assert gbs == pytest.approx(2 * 10 * 1e9 / 0.020 / 1e9)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.job_gbs(2e9, 1, 4, 2.0) == pytest.approx(4.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "3", "--warmup", "3"],
                         env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0
    assert res.stdout.strip() == "", "ranks other than 0 print nothing"


def test_reference_arm_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "3", "--warmup", "3", "--workload", "tiny"],
                         env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
