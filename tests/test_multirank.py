"""The multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1)."""
from __future__ import annotations

import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        m = bench.max_over_ranks(ms[rank], world)
        out.put((rank, m, bench.job_throughput(1000, world, 10, m)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_maximum_time_and_count_both_ranks_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ms = [3.0, 5.0]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, ms, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [m for _, m, _ in res] == [5.0, 5.0]
    assert all(v == 1000 * 2 * 10 / 5e-3 for _, _, v in res)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.5, 1) == 4.5
    assert bench.job_throughput(7, 1, 3, 2.0) == 7 * 3 / 2e-3


def test_rank_weight_sets_are_disjoint():
    layers = 32
    seeds = [{bench.rank_layer_seed(l, r, layers) for l in range(layers)} for r in range(8)]
    for a in range(8):
        for b in range(a + 1, 8):
            assert not seeds[a] & seeds[b]


def test_reference_arm_on_a_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.timeout(600)
def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
