"""The multi-rank path of bench.py on CPU (gloo, world size 2, 127.0.0.1).

The pipeline has no exchange step, so N GPUs run N independent replicas; the
only cross-rank logic is the timing aggregation (max over ranks) and the
per-call value over all ranks' calls, and the reference arm printing on
rank 0 only.  No GPU is needed."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(values[rank], dist)
        out_q.put((rank, ms, bench.us_per_call(ms, steps=10, calls_per_step=12, world=world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_value_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    values = [3.5, 7.25]
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [7.25, 7.25]           # every rank sees the slowest rank's time
    assert res[0][2] == res[1][2] == pytest.approx(7.25 * 1000 / (10 * 12 * 2))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.0, None) == 4.0
    assert bench.us_per_call(12.0, 100, 12, 1) == pytest.approx(10.0)


def _reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--gpus", str(world), "--steps", "1", "--warmup", "3"],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_on_rank_zero_only():
    r1 = _reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _reference(0, 2)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "µs/call" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["value"] > 0
